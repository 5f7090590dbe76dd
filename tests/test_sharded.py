"""KV-sharded decode on CPU: the shard plan, the per-shard attention inputs
and the exchange, with the fp64 oracle standing in for each shard's kernels.

The merge of shard results must reproduce the unsharded result exactly (up to
fp64 rounding): the softmax sum decomposes over disjoint row ranges.  The
exchange runs over two gloo ranks, as the GPUs' all-gather would."""
import os
import socket
import sys

import numpy as np
import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import oracle  # noqa: E402
from latent_attention_decode_absorbed_b200 import sharded  # noqa: E402


def _problem(lens, T, H, seed):
    """Seeded paged pool (fp64 rows), block table and absorbed queries."""
    g = np.random.default_rng(seed)
    npg = [-(-L // 64) for L in lens]
    ids = g.permutation(sum(npg) + 3)
    bt = np.full((len(lens), max(npg)), -1, np.int32)
    off = 0
    for b, n in enumerate(npg):
        bt[b, :n] = ids[off:off + n]
        off += n
    pool = g.standard_normal((len(ids) * 64, 576))
    q = 0.25 * g.standard_normal((len(lens) * T, H, 576))
    return bt, pool, q


def _seq_rows(pool, bt, b, L):
    pages = bt[b, :-(-L // 64)].astype(np.int64)
    return np.concatenate([pool[p * 64:(p + 1) * 64] for p in pages])[:L]


def _oracle_unsharded(lens, T, bt, pool, q):
    H = q.shape[1]
    o = np.zeros((len(lens) * T, H, 512)); lse = np.zeros((len(lens) * T, H))
    for b, L in enumerate(lens):
        rows = _seq_rows(pool, bt, b, L)
        op, lp = oracle.attention_partials(q[b * T:(b + 1) * T, :, :512], q[b * T:(b + 1) * T, :, 512:],
                                           rows[:, :512], rows[:, 512:], 64 * -(-L // 64), 1)
        o[b * T:(b + 1) * T], lse[b * T:(b + 1) * T] = op[:, :, 0], lp[:, :, 0]
    return o, lse


def _oracle_shard(plan, g, bt, pool, q):
    """Shard g's result through its own attention inputs: each query row is a
    sequence of lens[r] rows whose pages are table[r] (all rows visible)."""
    table, lens = sharded.shard_inputs(plan, g, bt)
    H = q.shape[1]
    o = np.zeros((table.shape[0], H, 512)); lse = np.full((table.shape[0], H), -np.inf)
    for r in range(table.shape[0]):
        n = int(lens[r])
        assert n >= 1
        rows = np.concatenate([pool[int(p) * 64:(int(p) + 1) * 64] for p in table[r] if p >= 0])[:n]
        op, lp = oracle.attention_partials(q[r:r + 1, :, :512], q[r:r + 1, :, 512:], rows[:, :512],
                                           rows[:, 512:], 64 * -(-n // 64), 1)
        o[r], lse[r] = op[0, :, 0], lp[0, :, 0]
    return o, lse


def _merge(o_all, lse_all):
    # shard-major [G, rows, H, 512] -> the oracle's [..., parts, 512] convention
    return oracle.combine_partials(np.moveaxis(o_all, 0, 2), np.moveaxis(lse_all, 0, 2))


@pytest.mark.parametrize("world", [1, 2, 3, 5])
@pytest.mark.parametrize("T", [1, 2, 3])
def test_plan_covers_every_row_once(world, T):
    lens = [320, 321, 383, 384, 1000, 64 * world + T]
    plan = sharded.plan_shards(lens, T, world)
    for b, L in enumerate(lens):
        r = [plan.ranges[g][b] for g in range(world)]
        assert r[0][0] == 0 and r[-1][1] == L
        for g in range(world):
            lo, hi = r[g]
            assert lo < hi, "every shard holds rows of every sequence"
            assert lo % 64 == 0 and (hi % 64 == 0 or g == world - 1)
            if g + 1 < world:
                assert hi == r[g + 1][0]
        assert r[-1][0] <= L - T, "the new rows lie in the last shard"


def test_plan_rejects_what_cannot_shard():
    with pytest.raises(ValueError):
        sharded.plan_shards([128], 1, 3)                     # 2 pages, 3 shards
    with pytest.raises(ValueError):
        sharded.plan_shards([65], 2, 2)                      # new rows straddle the only boundary
    with pytest.raises(ValueError):
        sharded.plan_shards([1], 2, 1)                       # shorter than q_len


@pytest.mark.parametrize("T", [1, 2])
def test_shard_inputs_see_exactly_the_causal_rows(T):
    lens = [700, 130, 257]
    world = 2
    bt, pool, _ = _problem(lens, T, 4, seed=3)
    plan = sharded.plan_shards(lens, T, world)
    for g in range(world):
        table, ln = sharded.shard_inputs(plan, g, bt)
        for b, L in enumerate(lens):
            lo, hi = plan.ranges[g][b]
            for t in range(T):
                r = b * T + t
                want = [j for j in range(lo, hi) if j <= L - T + t]        # causal rule, brute force
                assert ln[r] == len(want)
                pages = [int(p) for p in table[r] if p >= 0]
                got_slots = [p * 64 + i for p in pages for i in range(64)][:ln[r]]
                want_slots = [int(bt[b, j // 64]) * 64 + j % 64 for j in want]
                assert got_slots == want_slots


@pytest.mark.parametrize("world,T", [(1, 1), (2, 1), (3, 2), (4, 1)])
def test_merged_shards_equal_unsharded(world, T):
    lens = [1000, 300, 64 * 4 + 1]
    bt, pool, q = _problem(lens, T, 8, seed=world * 10 + T)
    plan = sharded.plan_shards(lens, T, world)
    parts = [_oracle_shard(plan, g, bt, pool, q) for g in range(world)]
    o, lse = _merge(np.stack([p[0] for p in parts]), np.stack([p[1] for p in parts]))
    ref_o, ref_l = _oracle_unsharded(lens, T, bt, pool, q)
    assert oracle.normwise_rel_err(o, ref_o) < 1e-12
    np.testing.assert_allclose(lse, ref_l, rtol=0, atol=1e-12)


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _rank_main(rank, world, port, out):
    import datetime
    import torch
    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        lens, T = [900, 200], 2
        bt, pool, q = _problem(lens, T, 4, seed=7)            # same seed: every rank has the whole problem
        plan = sharded.plan_shards(lens, T, world)
        o_g, l_g = _oracle_shard(plan, rank, bt, pool, q)     # this rank's rows only
        o_all, l_all = sharded.gather_shards(torch.from_numpy(o_g), torch.from_numpy(l_g))
        o, lse = _merge(o_all.numpy(), l_all.numpy())
        out[rank] = (o_all.numpy()[rank] - o_g, o, lse)
    finally:
        dist.destroy_process_group()


def test_exchange_over_two_gloo_ranks():
    world = 2
    mgr = mp.get_context("spawn").Manager()
    out = mgr.dict()
    mp.spawn(_rank_main, args=(world, _free_port(), out), nprocs=world, join=True)
    lens, T = [900, 200], 2
    bt, pool, q = _problem(lens, T, 4, seed=7)
    ref_o, ref_l = _oracle_unsharded(lens, T, bt, pool, q)
    for rank in range(world):
        own_diff, o, lse = out[rank]
        assert np.all(own_diff == 0), "the gathered tensor holds each rank's result at its rank"
        assert oracle.normwise_rel_err(o, ref_o) < 1e-12
        np.testing.assert_allclose(lse, ref_l, rtol=0, atol=1e-12)
