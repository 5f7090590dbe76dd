"""KV-sharded decode on one GPU, against the fp64 oracle.

Each shard's attention call and split merge run one after another on the same
GPU (no kernel waits on another), their results are stacked in shard order as
the GPUs' all-gather would deliver them, and ``mla_combine_shards`` merges
them.  The merged output must match the oracle over each sequence's whole
row range, and the unsharded GPU result."""
import math
import zlib

import numpy as np
import pytest

import latent_attention_decode_absorbed_b200 as mla
import oracle
from latent_attention_decode_absorbed_b200 import sharded
from test_gpu_kernels import DT, _pool, _random_cache
from workloads import round_bf16
from workloads.device import to_device, to_host_f64

pytestmark = pytest.mark.gpu
torch = pytest.importorskip("torch")

CASES = [
    # (name, cache_dt, lens, T, world, split_tokens)
    ("bf16_t1_3shards", "bf16", [2000, 700, 1025], 1, 3, 256),
    ("bf16_t2_2shards", "bf16", [1500, 513], 2, 2, 512),
    ("bf16_t1_8shards", "bf16", [4096, 600], 1, 8, 64),
    ("e4m3_t2_4shards", "e4m3", [1100, 400], 2, 4, 128),
]


@pytest.mark.parametrize("case", CASES, ids=lambda c: c[0])
def test_sharded_decode_matches_oracle(case):
    name, cache_dt, lens, T, world, st = case
    g = np.random.default_rng(zlib.crc32(name.encode()))
    bt, num_pages = _pool(lens, spare=1, seed=len(name))
    cache, scale, vals = _random_cache(g, num_pages, cache_dt)
    B, H = len(lens), 128
    q = round_bf16(g.standard_normal((B * T, H, 576)).astype(np.float32) * 0.25)
    q_dev = to_device(q, "bf16")
    scale_f = 1 / math.sqrt(192)
    plan = sharded.plan_shards(lens, T, world)
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    o_all = torch.full((world, B * T, H, 512), float("nan"), device="cuda")
    l_all = torch.full((world, B * T, H), float("nan"), device="cuda")
    for s in range(world):
        table, ln = sharded.shard_inputs(plan, s, bt)
        S = -(-table.shape[1] * 64 // st)
        o_part = torch.empty((B * T, H, S, 512), device="cuda")
        lse_part = torch.empty((B * T, H, S), device="cuda")
        sharded.decode_shard(q_dev, cache, scale, DT[cache_dt], num_pages, torch.from_numpy(table).cuda(),
                             torch.from_numpy(ln).cuda(), H, st, scale_f, o_part, lse_part, o_all[s], l_all[s], err)
    o_lat = torch.empty((B * T, H, 512), device="cuda")
    lse = torch.empty((B * T, H), device="cuda")
    sharded.merge_shards(o_all, l_all, o_lat, mla.MLA_F32, lse)
    # the unsharded GPU path on the same inputs
    S1 = -(-bt.shape[1] * 64 // st)
    o1 = torch.empty((B * T, H, S1, 512), device="cuda"); l1 = torch.empty((B * T, H, S1), device="cuda")
    mla.mla_decode_fwd(q_dev, mla.MLA_BF16, cache, scale, DT[cache_dt], num_pages, torch.from_numpy(bt).cuda(),
                       bt.shape[1], 64, torch.tensor(lens, dtype=torch.int32).cuda(), B, T, H, S1, st, scale_f,
                       o1, l1, err)
    o_un = torch.empty((B * T, H, 512), device="cuda"); l_un = torch.empty((B * T, H), device="cuda")
    mla.mla_combine(o1, l1, B * T, H, S1, o_un, mla.MLA_F32, l_un)
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    got_o, got_l = to_host_f64(o_lat), to_host_f64(lse)
    for b, L in enumerate(lens):
        slots = bt[b, np.arange(L) // 64].astype(np.int64) * 64 + np.arange(L) % 64
        rows = vals[slots]
        qq = q[b * T:(b + 1) * T].astype(np.float64)
        ref_o, ref_l = oracle.attention_partials(qq[..., :512], qq[..., 512:], rows[:, :512], rows[:, 512:],
                                                 64 * -(-L // 64), 1)
        go, gl = got_o[b * T:(b + 1) * T], got_l[b * T:(b + 1) * T]
        assert oracle.normwise_rel_err(go, ref_o[:, :, 0]) < 5e-3, f"seq {b} o_lat"
        np.testing.assert_allclose(gl, ref_l[:, :, 0], rtol=0, atol=2e-3)
    assert oracle.normwise_rel_err(got_o, to_host_f64(o_un)) < 5e-3
    np.testing.assert_allclose(got_l, to_host_f64(l_un), rtol=0, atol=2e-3)


def test_combine_shards_skips_shards_that_saw_nothing():
    """A shard with lse = -inf for a (row, head) is not read (its o is NaN
    here); a (row, head) no shard saw gives o = 0 and lse = -inf."""
    g = np.random.default_rng(5)
    G, rows, H = 3, 4, 16
    o = g.standard_normal((G, rows, H, 512)).astype(np.float32)
    lse = g.standard_normal((G, rows, H)).astype(np.float32)
    lse[1, 0, :] = -np.inf; o[1, 0, :] = np.nan
    lse[:, 2, 3] = -np.inf
    # the oracle's convention for a part that saw nothing: o = 0
    o_seen = np.where(np.isfinite(lse)[..., None], o, 0.0).astype(np.float64)
    ref_o, ref_l = oracle.combine_partials(np.moveaxis(o_seen, 0, 2), np.moveaxis(lse.astype(np.float64), 0, 2))
    o_lat = torch.empty((rows, H, 512), device="cuda"); l_out = torch.empty((rows, H), device="cuda")
    mla.mla_combine_shards(torch.from_numpy(o).cuda(), torch.from_numpy(lse).cuda(), G, rows, H, o_lat,
                           mla.MLA_F32, l_out)
    torch.cuda.synchronize()
    got_o, got_l = to_host_f64(o_lat), to_host_f64(l_out)
    fin = np.isfinite(ref_l)
    assert np.all(np.isneginf(got_l[~fin])) and np.all(got_o[~fin] == 0)
    assert oracle.normwise_rel_err(got_o[fin], ref_o[fin]) < 1e-6
    np.testing.assert_allclose(got_l[fin], ref_l[fin], rtol=0, atol=1e-5)
