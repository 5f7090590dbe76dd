"""The non-absorbed ("level 2") decode against the oracle, on the GPU through
the C ABI: mla_decompress_kv (k^C = W_UK c, v^C = W_UV c per head, stored
bf16) and mla_attend_naive (standard attention per head over them).

Tolerances come from the arithmetic: the decompressed keys and values are
fp32 sums of bf16 products rounded once to bf16 (relative 2^-9 per element);
the attention then runs in fp32 over those bf16 values and stores bf16, so the
per-head output is within the bf16 gate (normwise 1e-2) of the fp64 oracle,
and within the same gate of the absorbed path."""
import math
import zlib

import numpy as np
import pytest

import latent_attention_decode_absorbed_b200 as mla
import oracle
from workloads import round_bf16
from workloads.device import to_device, to_host_f64

pytestmark = pytest.mark.gpu
torch = pytest.importorskip("torch")


def _pool(lens, spare, seed):
    g = np.random.default_rng(seed)
    npg = [(L + 63) // 64 for L in lens]
    total = sum(npg) + spare
    ids = g.permutation(total)
    bt = np.full((len(lens), max(npg)), -1, np.int32)
    off = 0
    for b, n in enumerate(npg):
        bt[b, :n] = ids[off:off + n]
        off += n
    return bt, total


def _weights(g, H):
    w_uk = round_bf16((g.standard_normal((H, 128, 512)) / math.sqrt(512)).astype(np.float32))
    w_uv = round_bf16((g.standard_normal((H, 128, 512)) / math.sqrt(512)).astype(np.float32))
    return w_uk, w_uv


@pytest.mark.parametrize("num_pages,H", [(5, 128), (8, 16), (1, 65)])
def test_decompress_matches_oracle(num_pages, H):
    g = np.random.default_rng(num_pages * 100 + H)
    rows = round_bf16(g.standard_normal((num_pages * 64, 576)).astype(np.float32))
    cache = mla.pack_cache_rows(to_device(rows, "bf16"))
    w_uk, w_uv = _weights(g, H)
    k_c = torch.full((num_pages, 64, H, 128), float("nan"), dtype=torch.bfloat16, device="cuda")
    v_c = torch.full_like(k_c, float("nan"))
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    mla.mla_decompress_kv(cache, mla.MLA_BF16, num_pages, 64, to_device(w_uk, "bf16"), to_device(w_uv, "bf16"), H,
                          k_c, v_c, err)
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    ref_k, ref_v = oracle.decompress_kv(rows[:, :512].astype(np.float64), w_uk.astype(np.float64),
                                        w_uv.astype(np.float64))
    got_k = to_host_f64(k_c).reshape(num_pages * 64, H, 128)
    got_v = to_host_f64(v_c).reshape(num_pages * 64, H, 128)
    for got, ref in ((got_k, ref_k), (got_v, ref_v)):
        assert np.all(np.isfinite(got)), "rows left unwritten"
        # each element: one bf16 rounding of an fp32 sum (bf16 half-ulp 2^-9, plus fp32 sum error)
        np.testing.assert_allclose(got, ref, rtol=2 ** -8, atol=1e-5)
        assert oracle.normwise_rel_err(got, ref) < 4e-3


def _random_step(name, lens, T, H):
    g = np.random.default_rng(zlib.crc32(name.encode()))
    bt, num_pages = _pool(lens, spare=2, seed=len(name))
    rows = round_bf16(g.standard_normal((num_pages * 64, 576)).astype(np.float32))
    B = len(lens)
    q_nope = round_bf16(g.standard_normal((B * T, H, 128)).astype(np.float32))
    q_pe = round_bf16(g.standard_normal((B * T, H, 64)).astype(np.float32))
    w_uk, w_uv = _weights(g, H)
    return bt, num_pages, rows, q_nope, q_pe, w_uk, w_uv


def _run_naive(bt, num_pages, rows, q_nope, q_pe, w_uk, w_uv, lens, T, H, scale):
    B = len(lens)
    cache = mla.pack_cache_rows(to_device(rows, "bf16"))
    k_c = torch.empty((num_pages, 64, H, 128), dtype=torch.bfloat16, device="cuda")
    v_c = torch.empty_like(k_c)
    out = torch.full((B * T, H, 128), float("nan"), dtype=torch.bfloat16, device="cuda")
    lse = torch.full((B * T, H), float("nan"), device="cuda")
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    bt_d = torch.from_numpy(bt).cuda()
    lens_d = torch.tensor(lens, dtype=torch.int32).cuda()
    mla.mla_decompress_kv(cache, mla.MLA_BF16, num_pages, 64, to_device(w_uk, "bf16"), to_device(w_uv, "bf16"), H,
                          k_c, v_c, err)
    mla.mla_attend_naive(to_device(q_nope, "bf16"), to_device(q_pe, "bf16"), cache, mla.MLA_BF16, k_c, v_c,
                         num_pages, bt_d, bt.shape[1], 64, lens_d, B, T, H, scale, out, lse, err)
    torch.cuda.synchronize()
    return cache, out, lse, err


NAIVE_CASES = [
    ("ragged_t1", [1, 65, 300], 1, 128),
    ("mtp_t2", [2, 190, 129], 2, 128),
    ("heads16", [700], 1, 16),
    ("heads65_t2", [64, 3], 2, 65),
]


@pytest.mark.parametrize("case", NAIVE_CASES, ids=lambda c: c[0])
def test_attend_naive_matches_oracle_and_absorbed(case):
    name, lens, T, H = case
    scale = 1 / math.sqrt(192)
    bt, num_pages, rows, q_nope, q_pe, w_uk, w_uv = _random_step(name, lens, T, H)
    cache, out, lse, err = _run_naive(bt, num_pages, rows, q_nope, q_pe, w_uk, w_uv, lens, T, H, scale)
    assert int(err.item()) == 0
    got = to_host_f64(out).reshape(len(lens), T, H, 128)
    got_lse = lse.cpu().numpy().astype(np.float64).reshape(len(lens), T, H)
    for b, L in enumerate(lens):
        slots = (bt[b, np.arange(L) // 64].astype(np.int64) * 64 + np.arange(L) % 64)
        c_hat, k_r = rows[slots, :512].astype(np.float64), rows[slots, 512:].astype(np.float64)
        ref = oracle.attention_naive(q_nope[b * T:(b + 1) * T].astype(np.float64),
                                     q_pe[b * T:(b + 1) * T].astype(np.float64), w_uk.astype(np.float64),
                                     w_uv.astype(np.float64), c_hat, k_r, scale)
        assert oracle.normwise_rel_err(got[b], ref) < 1e-2, f"{name} seq {b}"
        # lse: the log-normaliser of the same scores (absorbed form, same values)
        q_lat = oracle.absorb_q(q_nope[b * T:(b + 1) * T], w_uk.astype(np.float64))
        for t in range(T):
            n_vis = L - T + t + 1
            z = (np.einsum("hc,jc->hj", q_lat[t], c_hat[:n_vis]) +
                 np.einsum("hr,jr->hj", q_pe[b * T + t].astype(np.float64), k_r[:n_vis])) * scale
            zm = z.max(axis=1)
            ref_lse = zm + np.log(np.exp(z - zm[:, None]).sum(axis=1))
            np.testing.assert_allclose(got_lse[b, t], ref_lse, atol=0.05)
    # the absorbed path on the same cache and queries gives the same per-head output
    B = len(lens)
    q_abs = torch.empty((B * T, H, 576), dtype=torch.bfloat16, device="cuda")
    mla.mla_absorb_q(to_device(q_nope, "bf16"), to_device(q_pe, "bf16"), to_device(w_uk, "bf16"), q_abs, B * T, H,
                     mla.MLA_BF16)
    S = -(-bt.shape[1] * 64 // 256)
    o_part = torch.empty((B * T, H, S, 512), device="cuda")
    lse_part = torch.empty((B * T, H, S), device="cuda")
    mla.mla_decode_fwd(q_abs, mla.MLA_BF16, cache, None, mla.MLA_BF16, num_pages, torch.from_numpy(bt).cuda(),
                       bt.shape[1], 64, torch.tensor(lens, dtype=torch.int32).cuda(), B, T, H, S, 256, scale, o_part,
                       lse_part, err)
    o_lat = torch.empty((B * T, H, 512), dtype=torch.bfloat16, device="cuda")
    mla.mla_combine(o_part, lse_part, B * T, H, S, o_lat, mla.MLA_BF16, None)
    out_abs = torch.empty((B * T, H, 128), dtype=torch.bfloat16, device="cuda")
    mla.mla_out_uv(o_lat, to_device(w_uv, "bf16"), out_abs, B * T, H, mla.MLA_BF16)
    torch.cuda.synchronize()
    assert oracle.normwise_rel_err(to_host_f64(out).reshape(B * T, H, 128),
                                   to_host_f64(out_abs).reshape(B * T, H, 128)) < 1e-2


def test_attend_naive_flags_a_page_outside_the_pool():
    lens, T, H = [130], 1, 16
    bt, num_pages, rows, q_nope, q_pe, w_uk, w_uv = _random_step("badpage", lens, T, H)
    bt[0, 1] = num_pages + 7
    _, out, _, err = _run_naive(bt, num_pages, rows, q_nope, q_pe, w_uk, w_uv, lens, T, H, 1 / math.sqrt(192))
    assert int(err.item()) & mla.MLA_DEVERR_PAGE
    assert np.all(np.isfinite(to_host_f64(out)))


def test_naive_path_rejects_an_e4m3_cache():
    x = torch.zeros((1, 9, 64, 64), dtype=torch.uint8, device="cuda")
    k = torch.zeros((1, 64, 16, 128), dtype=torch.bfloat16, device="cuda")
    w = torch.zeros((16, 128, 512), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(mla.MlaError) as e:
        mla.mla_decompress_kv(x, mla.MLA_E4M3, 1, 64, w, w, 16, k, k)
    assert e.value.status == mla.MLA_ERR_UNSUPPORTED
