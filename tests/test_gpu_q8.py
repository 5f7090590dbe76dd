"""The 8-bit tensor-core decode over an e4m3 cache, on the GPU through the C
ABI: mla_split_q_e4m3 (the query's two-term e4m3 form) against the oracle's
split_query_e4m3 bit for bit, and mla_decode_fwd_q8's partials against the
oracle's exact attention over the dequantised cache.

Tolerances come from the arithmetic: the query and the softmax weights each
carry about 8 significant bits (two e4m3 terms, 2^-8 relative per value), the
products are exact and accumulate in fp32, so the partial's normwise error is
a few 2^-9 at most: the same 5e-3 (o_part) and 2e-3 (lse) bounds as the
widened e4m3 form (f16 operands) of mla_decode_fwd."""
import math
import zlib

import numpy as np
import pytest

import latent_attention_decode_absorbed_b200 as mla
import oracle
from test_gpu_kernels import _pool, _random_cache
from workloads import round_bf16
from workloads.device import to_device, to_host_f64

pytestmark = pytest.mark.gpu
torch = pytest.importorskip("torch")


def _split(q_dev, rows, H):
    q8 = torch.full((rows, 2, H, 576), 0xAB, dtype=torch.uint8, device="cuda")
    qs = torch.full((rows, H), float("nan"), device="cuda")
    mla.mla_split_q_e4m3(q_dev, rows, H, q8, qs)
    return q8, qs


@pytest.mark.parametrize("rows,H", [(3, 128), (1, 65), (7, 96), (2, 16)])
def test_split_q_matches_oracle_bit_exact(rows, H):
    g = np.random.default_rng(rows * 1000 + H)
    q = g.standard_normal((rows, H, 576)) * np.exp(g.uniform(-12, 12, (rows, H, 1)))
    q[0, H // 2] = 0.0                                     # a zero vector: codes 0, scale 0
    q[-1, 0, 7] = 3.0e4                                    # one large value among small ones
    q = round_bf16(q.astype(np.float32))
    q8, qs = _split(to_device(q, "bf16"), rows, H)
    torch.cuda.synchronize()
    hi, lo, sc = oracle.split_query_e4m3(q)
    got = q8.cpu().numpy()
    assert np.array_equal(got[:, 0], hi), "hi codes"
    assert np.array_equal(got[:, 1], lo), "lo codes"
    assert np.array_equal(qs.cpu().numpy().view(np.uint32), sc.astype(np.float32).view(np.uint32)), "scales"


def _decode_q8(q, cache, scale, num_pages, bt, lens, T, H, st, err=None):
    B = len(lens)
    q8, qs = _split(to_device(q, "bf16"), B * T, H)
    S = -(-bt.shape[1] * 64 // st)
    o_part = torch.full((B * T, H, S, 512), float("nan"), device="cuda")
    lse_part = torch.full((B * T, H, S), float("nan"), device="cuda")
    if err is None:
        err = torch.zeros(1, dtype=torch.int32, device="cuda")
    mla.mla_decode_fwd_q8(q8, qs, cache, scale, num_pages, torch.from_numpy(bt).cuda(), bt.shape[1], 64,
                          torch.tensor(lens, dtype=torch.int32).cuda(), B, T, H, S, st, 1 / math.sqrt(192),
                          o_part, lse_part, err)
    torch.cuda.synchronize()
    return o_part, lse_part, err, S


CASES = [
    # (name, lens, T, H, split_tokens)
    ("ragged_mtp", [5, 400, 1025], 2, 128, 256),
    ("multi_tile_mtp", [1100, 600], 2, 128, 1024),
    ("long_split", [5000], 1, 128, 4096),
    ("heads96_mtp", [700, 65, 2], 2, 96, 128),
    ("heads65", [129], 1, 65, 64),
    ("many_units_mtp", [1500] * 6 + [7000], 2, 128, 128),
]


@pytest.mark.parametrize("case", CASES, ids=lambda c: c[0])
def test_decode_q8_partials(case):
    name, lens, T, H, st = case
    g = np.random.default_rng(zlib.crc32(("q8" + name).encode()))
    bt, num_pages = _pool(lens, spare=2, seed=len(name))
    cache, scale, vals = _random_cache(g, num_pages, "e4m3")
    B = len(lens)
    q = round_bf16(g.standard_normal((B * T, H, 576)).astype(np.float32) * 0.25)
    o_part, lse_part, err, S = _decode_q8(q, cache, scale, num_pages, bt, lens, T, H, st)
    assert int(err.item()) == 0
    got_o, got_l = to_host_f64(o_part), to_host_f64(lse_part)
    for b, L in enumerate(lens):
        slots = bt[b, np.arange(L) // 64].astype(np.int64) * 64 + np.arange(L) % 64
        rows = vals[slots]
        qq = q[b * T:(b + 1) * T].astype(np.float64)
        ref_o, ref_l = oracle.attention_partials(qq[..., :512], qq[..., 512:], rows[:, :512], rows[:, 512:],
                                                 st, S, 1 / math.sqrt(192))
        go, gl = got_o[b * T:(b + 1) * T], got_l[b * T:(b + 1) * T]
        # runs of merged splits: each finite lse starts a run ending at the next
        assert np.all(np.isneginf(gl[~np.isfinite(ref_l)])), f"seq {b}: empty splits must report -inf"
        for t in range(T):
            for h in range(H):
                starts = np.nonzero(np.isfinite(gl[t, h]))[0]
                assert starts.size and starts[0] == 0, f"seq {b}: the first split must hold a partial"
                for s0, s1 in zip(starts, list(starts[1:]) + [S]):
                    mo, ml = oracle.combine_partials(ref_o[t, h, s0:s1], ref_l[t, h, s0:s1])
                    ref_o[t, h, s0], ref_l[t, h, s0] = mo, ml
                    ref_l[t, h, s0 + 1:s1] = -np.inf
        fin = np.isfinite(gl)
        assert np.array_equal(fin, np.isfinite(ref_l)), f"seq {b}: runs of merged splits"
        assert oracle.normwise_rel_err(go[fin], ref_o[fin]) < 5e-3, f"seq {b} o_part"
        np.testing.assert_allclose(gl[fin], ref_l[fin], rtol=0, atol=2e-3)


def test_decode_q8_flags_a_page_outside_the_pool():
    lens, T, H, st = [300, 130], 1, 128, 128
    g = np.random.default_rng(77)
    bt, num_pages = _pool(lens, spare=1, seed=3)
    bt[1, 1] = num_pages + 5
    cache, scale, _ = _random_cache(g, num_pages, "e4m3")
    q = round_bf16(g.standard_normal((2, H, 576)).astype(np.float32) * 0.25)
    o_part, lse_part, err, _ = _decode_q8(q, cache, scale, num_pages, bt, lens, T, H, st)
    assert int(err.item()) & mla.MLA_DEVERR_PAGE
    lse = lse_part.cpu().numpy()
    assert not np.isnan(lse).any()


def test_decode_q8_wait_bound_runs_out_then_next_launch_is_correct():
    lens, T, H, st = [300, 1000, 64], 1, 128, 256
    g = np.random.default_rng(78)
    bt, num_pages = _pool(lens, spare=0, seed=4)
    cache, scale, vals = _random_cache(g, num_pages, "e4m3")
    q = round_bf16(g.standard_normal((3, H, 576)).astype(np.float32) * 0.25)
    try:
        mla.mla_test_set_decode_wait(2_000_000, withhold_q_load=True)
        _, _, err, _ = _decode_q8(q, cache, scale, num_pages, bt, lens, T, H, st)
        assert int(err.item()) & mla.MLA_DEVERR_TIMEOUT
    finally:
        mla.mla_test_set_decode_wait(0, withhold_q_load=False)
    o_part, lse_part, err, S = _decode_q8(q, cache, scale, num_pages, bt, lens, T, H, st)
    assert int(err.item()) == 0
    o_lat = torch.empty((3, H, 512), device="cuda")
    lse = torch.empty((3, H), device="cuda")
    mla.mla_combine(o_part, lse_part, 3, H, S, o_lat, mla.MLA_F32, lse)
    torch.cuda.synchronize()
    got = to_host_f64(o_lat)
    for b, L in enumerate(lens):
        slots = bt[b, np.arange(L) // 64].astype(np.int64) * 64 + np.arange(L) % 64
        rows = vals[slots]
        qq = q[b:b + 1].astype(np.float64)
        o, l = oracle.attention_partials(qq[..., :512], qq[..., 512:], rows[:, :512], rows[:, 512:], st, S,
                                         1 / math.sqrt(192))
        oc, _ = oracle.combine_partials(o, l)
        assert oracle.normwise_rel_err(got[b:b + 1], oc) < 5e-3


def test_decode_q8_rejects_unsupported_heads():
    x = torch.zeros(64, dtype=torch.uint8, device="cuda")
    f = torch.zeros(64, device="cuda")
    i = torch.zeros(4, dtype=torch.int32, device="cuda")
    with pytest.raises(mla.MlaError) as e:
        mla.mla_decode_fwd_q8(x, f, x, f, 1, i, 1, 64, i, 1, 1, 64, 1, 64, 0.1, f, f)
    assert e.value.status == mla.MLA_ERR_UNSUPPORTED
