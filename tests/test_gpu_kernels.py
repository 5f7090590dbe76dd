"""Each C-ABI call against the oracle on the GPU, on seeded inputs.

Append and its page indexing must be exact; projections, attention partials
and the combine must meet tolerances derived from their arithmetic."""
import math
import zlib

import numpy as np
import pytest

import latent_attention_decode_absorbed_b200 as mla
import oracle
from gpu_common import bf16_exact_or_boundary
from workloads import round_bf16
from workloads.device import to_device, to_host_f64

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")
DT = {"f32": mla.MLA_F32, "bf16": mla.MLA_BF16, "e4m3": mla.MLA_E4M3}
TDT = {"f32": torch.float32, "bf16": torch.bfloat16, "e4m3": torch.uint8}


def _rope_tables(n, theta=10000.0):
    cos = np.empty((n, 32), np.float32); sin = np.empty_like(cos)
    mla.mla_rope_table(theta, n, cos, sin)
    return torch.from_numpy(cos).cuda(), torch.from_numpy(sin).cuda()


def _pool(lens, spare, seed):
    """Permuted page pool with `spare` pages nobody owns."""
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


# ------------------------------------------------------------------ append
@pytest.mark.parametrize("cache_dt", ["f32", "bf16", "e4m3"])
@pytest.mark.parametrize("kv_dt", ["f32", "bf16"])
def test_append_exact(cache_dt, kv_dt):
    lens = [70, 130, 5, 64]
    bt, num_pages = _pool(lens, spare=3, seed=1)
    g = np.random.default_rng(2)
    seq = np.concatenate([np.full(L, b) for b, L in enumerate(lens)]).astype(np.int32)
    pos = np.concatenate([np.arange(L) for L in lens]).astype(np.int32)
    order = g.permutation(len(seq))
    seq, pos = seq[order], pos[order]
    kv = g.standard_normal((len(seq), 576)).astype(np.float32) * 2.0
    if kv_dt == "bf16":
        kv = round_bf16(kv)
    gain = (1.0 + 0.3 * g.standard_normal(512)).astype(np.float32)
    eps = 1e-6
    max_pos = 200
    cos, sin = _rope_tables(max_pos)
    cache = torch.zeros((num_pages, 9, 64, 64), dtype=TDT[cache_dt], device="cuda")
    cache.view(torch.uint8).fill_(0xFF)                     # sentinel: every byte 0xFF
    scale = torch.full((num_pages, 64), float("nan"), device="cuda") if cache_dt == "e4m3" else None
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    mla.mla_cache_append(to_device(kv, kv_dt), DT[kv_dt], len(seq), torch.from_numpy(seq).cuda(),
                         torch.from_numpy(pos).cuda(), torch.from_numpy(bt).cuda(), len(lens), bt.shape[1], 64,
                         torch.from_numpy(gain).cuda(), eps, cos, sin, max_pos, cache, scale, DT[cache_dt],
                         num_pages, err)
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    rows_dev = mla.unpack_cache_rows(cache)                  # logical rows [num_pages*64, 576]
    raw = rows_dev.contiguous().view(torch.uint8).cpu().numpy().reshape(num_pages * 64, -1)
    slot = bt[seq, pos // 64].astype(np.int64) * 64 + pos % 64
    # indexing: exactly the appended slots changed
    touched = np.zeros(num_pages * 64, bool); touched[slot] = True
    assert np.all(raw[~touched] == 0xFF)
    assert not np.any(np.all(raw[touched] == 0xFF, axis=1))
    ref = oracle.cache_rows(kv, pos, gain, eps)              # fp64 [n, 576]
    if cache_dt == "f32":
        got = rows_dev.cpu().numpy().astype(np.float64)[slot]
        np.testing.assert_allclose(got, ref, rtol=2e-6, atol=1e-6)
    elif cache_dt == "bf16":
        got = rows_dev.to(torch.float64).cpu().numpy()[slot]
        bad = bf16_exact_or_boundary(got, ref)
        assert not bad.any(), f"{bad.sum()} bf16 values off (first at {np.argwhere(bad)[:3]})"
    else:
        codes = rows_dev.cpu().numpy()[slot]
        sc = scale.view(-1).cpu().numpy().astype(np.float64)
        assert np.all(np.isnan(np.delete(sc, slot)))
        ref_codes, ref_scale = oracle.quantize_rows_e4m3(ref)
        np.testing.assert_allclose(sc[slot], ref_scale, rtol=2e-6)
        diff = codes != ref_codes
        if diff.any():
            # only where x*448/a sits within fp32 error of a rounding tie
            y = ref * (448.0 / np.max(np.abs(ref), axis=1, keepdims=True))
            a, bq = oracle.e4m3_decode(codes[diff]), oracle.e4m3_decode(ref_codes[diff])
            mid = 0.5 * (a + bq)
            assert np.all(np.abs(y[diff] - mid) <= 1e-5 * np.abs(y[diff])), "e4m3 codes differ away from a tie"
            assert diff.mean() < 1e-3


def test_append_bad_indices_are_skipped_and_flagged():
    lens = [64, 64]
    bt, num_pages = _pool(lens, spare=0, seed=3)
    bt[1, 0] = num_pages + 5                                # a page outside the pool
    cos, sin = _rope_tables(128)
    cache = torch.zeros((num_pages, 9, 64, 64), dtype=torch.bfloat16, device="cuda")
    cache.view(torch.uint8).fill_(0xFF)
    kv = to_device(round_bf16(np.ones((4, 576), np.float32)), "bf16")
    for seq, pos, flag in [([0, 0, 0, 0], [0, 1, 64, 2], mla.MLA_DEVERR_POSITION),   # 64 is past the table
                           ([0, 2, 0, 0], [0, 1, 5, 6], mla.MLA_DEVERR_POSITION),    # sequence 2 does not exist
                           ([1, 0, 0, 0], [3, 1, 5, 6], mla.MLA_DEVERR_PAGE)]:       # page outside the pool
        cache.view(torch.uint8).fill_(0xFF)
        err = torch.zeros(1, dtype=torch.int32, device="cuda")
        mla.mla_cache_append(kv, mla.MLA_BF16, 4, torch.tensor(seq, dtype=torch.int32, device="cuda"),
                             torch.tensor(pos, dtype=torch.int32, device="cuda"), torch.from_numpy(bt).cuda(),
                             2, bt.shape[1], 64, None, 1e-6, cos, sin, 128, cache, None, mla.MLA_BF16,
                             num_pages, err)
        torch.cuda.synchronize()
        assert int(err.item()) & flag
        raw = mla.unpack_cache_rows(cache).contiguous().view(torch.uint8).cpu().numpy()
        good = [(s, p) for s, p in zip(seq, pos) if s < 2 and p < 64 and not (s == 1)]
        n_written = int(np.sum(~np.all(raw == 0xFF, axis=1)))
        assert n_written == len(good)


# ------------------------------------------------------------------ projections
@pytest.mark.parametrize("dt", ["f32", "bf16"])
@pytest.mark.parametrize("rows,H", [(1, 128), (7, 16), (9, 128), (256, 128), (3, 48)])
def test_absorb_q(dt, rows, H):
    g = np.random.default_rng(rows * 1000 + H)
    cast = round_bf16 if dt == "bf16" else (lambda x: x)
    qn = cast(g.standard_normal((rows, H, 128)).astype(np.float32))
    qp = cast(g.standard_normal((rows, H, 64)).astype(np.float32))
    wuk = cast((g.standard_normal((H, 128, 512)) / math.sqrt(512)).astype(np.float32))
    q_abs = torch.empty((rows, H, 576), dtype=TDT[dt], device="cuda")
    mla.mla_absorb_q(to_device(qn, dt), to_device(qp, dt), to_device(wuk, dt), q_abs, rows, H, DT[dt])
    got = to_host_f64(q_abs)
    ref = oracle.absorb_q(qn, wuk)
    tol = 1e-5 if dt == "f32" else 6e-3
    assert oracle.normwise_rel_err(got[..., :512], ref) < tol
    assert np.array_equal(got[..., 512:], qp.astype(np.float64))        # q_pe copied bit for bit


@pytest.mark.parametrize("dt", ["f32", "bf16"])
@pytest.mark.parametrize("rows,H", [(1, 128), (8, 16), (13, 128), (256, 128)])
def test_out_uv(dt, rows, H):
    g = np.random.default_rng(rows * 7 + H)
    cast = round_bf16 if dt == "bf16" else (lambda x: x)
    o = cast(g.standard_normal((rows, H, 512)).astype(np.float32) * 0.1)
    wuv = cast((g.standard_normal((H, 128, 512)) / math.sqrt(512)).astype(np.float32))
    out = torch.empty((rows, H, 128), dtype=TDT[dt], device="cuda")
    mla.mla_out_uv(to_device(o, dt), to_device(wuv, dt), out, rows, H, DT[dt])
    tol = 1e-5 if dt == "f32" else 6e-3
    assert oracle.normwise_rel_err(to_host_f64(out), oracle.out_uv(o, wuv)) < tol


# ------------------------------------------------------------------ combine
@pytest.mark.parametrize("S", [1, 2, 7, 64])
@pytest.mark.parametrize("dt", ["f32", "bf16"])
def test_combine(S, dt):
    g = np.random.default_rng(S)
    rows, H = 5, 128
    o = g.standard_normal((rows, H, S, 512)).astype(np.float32)
    lse = (g.standard_normal((rows, H, S)) * 3).astype(np.float32)
    if S > 1:
        lse[:, :, 1] = -np.inf                               # an empty split
    lse[0, 0, :] = -np.inf                                   # a head that saw nothing
    lse[0, 0, 0] = 2.0 if S == 1 else lse[0, 0, 0]
    o_lat = torch.empty((rows, H, 512), dtype=TDT[dt], device="cuda")
    lse_out = torch.empty((rows, H), dtype=torch.float32, device="cuda")
    mla.mla_combine(torch.from_numpy(o).cuda(), torch.from_numpy(lse).cuda(), rows, H, S, o_lat, DT[dt], lse_out)
    ref_o, ref_l = oracle.combine_partials(o, lse)
    got_o, got_l = to_host_f64(o_lat), to_host_f64(lse_out)
    fin = np.isfinite(ref_l)
    tol = 1e-5 if dt == "f32" else 4e-3
    assert oracle.normwise_rel_err(got_o[fin], ref_o[fin]) < tol
    np.testing.assert_allclose(got_l[fin], ref_l[fin], rtol=1e-5, atol=1e-5)
    assert np.all(np.isneginf(got_l[~fin])) and np.all(got_o[~fin] == 0)


@pytest.mark.parametrize("rows,H,S", [(1, 128, 32), (3, 16, 7), (8, 128, 1), (2, 65, 64)])
def test_combine_out_uv(rows, H, S):
    """The merge and W_UV in one launch: o_lat bit-identical to mla_combine,
    out against the oracle (out_uv of the merged partials) and the two-launch
    path."""
    g = np.random.default_rng(rows * 100 + S)
    o = g.standard_normal((rows, H, S, 512)).astype(np.float32)
    lse = (g.standard_normal((rows, H, S)) * 3).astype(np.float32)
    if S > 1:
        lse[:, :, 1] = -np.inf                               # an empty split
    lse[0, 0, :] = -np.inf                                   # a head that saw nothing
    if S == 1:
        lse[0, 0, 0] = 2.0
    w_uv = round_bf16((g.standard_normal((H, 128, 512)) / np.sqrt(512)).astype(np.float32))
    od, ld, wd = torch.from_numpy(o).cuda(), torch.from_numpy(lse).cuda(), to_device(w_uv, "bf16")
    o_lat = torch.full((rows, H, 512), float("nan"), dtype=torch.bfloat16, device="cuda")
    out = torch.full((rows, H, 128), float("nan"), dtype=torch.bfloat16, device="cuda")
    lse_out = torch.empty((rows, H), dtype=torch.float32, device="cuda")
    mla.mla_combine_out_uv(od, ld, rows, H, S, wd, o_lat, out, lse_out)
    o_lat2 = torch.empty_like(o_lat)
    out2 = torch.empty_like(out)
    lse2 = torch.empty_like(lse_out)
    mla.mla_combine(od, ld, rows, H, S, o_lat2, mla.MLA_BF16, lse2)
    mla.mla_out_uv(o_lat2, wd, out2, rows, H, mla.MLA_BF16)
    torch.cuda.synchronize()
    assert torch.equal(o_lat, o_lat2) and torch.equal(lse_out, lse2)
    ref_o, _ = oracle.combine_partials(o, lse)
    ref_out = oracle.out_uv(oracle.round_to_bf16(np.nan_to_num(ref_o)), w_uv.astype(np.float64))
    got = to_host_f64(out)
    assert np.all(np.isfinite(got))
    seen = np.isfinite(lse).any(axis=2)                      # (row, head) pairs with a visible row
    assert np.all(got[~seen] == 0)
    assert oracle.normwise_rel_err(got[seen][:, None, :], ref_out[seen][:, None, :]) < 4e-3
    # the same products as the tensor-core out_uv up to fp32 summation order and one bf16 rounding
    np.testing.assert_allclose(got, to_host_f64(out2), rtol=2 ** -7, atol=1e-3)


# ------------------------------------------------------------------ attention partials
def _random_cache(g, num_pages, cache_dt):
    """Seeded cache contents straight from the generator: a valid input to the
    attention op whatever produced it.  Returns (device tensors, fp64 values)."""
    x = g.standard_normal((num_pages * 64, 576)).astype(np.float32)
    if cache_dt == "bf16":
        v = round_bf16(x)
        return mla.pack_cache_rows(to_device(v, "bf16")), None, v.astype(np.float64)
    if cache_dt == "f32":
        return mla.pack_cache_rows(to_device(x, "f32")), None, x.astype(np.float64)
    codes = torch.from_numpy(np.clip(x * 100, -440, 440)).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    sc = (g.uniform(0.002, 0.02, num_pages * 64)).astype(np.float32)
    vals = oracle.e4m3_decode(codes) * sc.astype(np.float64)[:, None]
    return (mla.pack_cache_rows(torch.from_numpy(codes).cuda()), torch.from_numpy(sc).cuda(), vals)


CASES = [
    # (name, cache_dt, lens, T, H, split_tokens)
    ("ragged_bf16", "bf16", [1, 65, 700, 129], 1, 128, 256),
    ("single_split_bf16", "bf16", [300, 1000], 1, 128, 1024),
    ("many_splits_bf16", "bf16", [2048, 777], 1, 128, 64),
    ("mtp_bf16", "bf16", [2, 190, 513], 2, 128, 128),
    ("heads16_bf16", "bf16", [333, 64], 1, 16, 128),
    ("heads64_mtp_bf16", "bf16", [260], 2, 64, 128),
    ("heads48_bf16", "bf16", [200, 513], 1, 48, 256),
    ("long_split_bf16", "bf16", [5000], 1, 128, 4096),
    # head counts that pad the pair's second half, and more units than CTA pairs
    ("heads96_bf16", "bf16", [500, 90], 1, 96, 256),
    ("heads80_mtp_bf16", "bf16", [300], 2, 80, 128),
    ("heads65_bf16", "bf16", [129], 1, 65, 64),
    ("many_units_bf16", "bf16", [1500] * 6 + [7000], 1, 128, 128),
    ("ragged_e4m3", "e4m3", [5, 400, 1025], 2, 128, 256),
    ("heads64_e4m3", "e4m3", [300, 70], 1, 64, 128),
    ("heads16_many_splits_e4m3", "e4m3", [700], 1, 16, 64),
    ("multi_tile_e4m3", "e4m3", [1100, 600], 2, 128, 1024),
    ("long_split_e4m3", "e4m3", [5000], 1, 128, 4096),
    # the e4m3 cache on the head-split pair: padded heads, two tokens, merged runs
    ("heads96_mtp_e4m3", "e4m3", [700, 65, 2], 2, 96, 128),
    ("heads65_e4m3", "e4m3", [129], 1, 65, 64),
    ("many_units_mtp_e4m3", "e4m3", [1500] * 6 + [7000], 2, 128, 128),
    ("tiny_f32", "f32", [256, 37], 1, 16, 64),
]


@pytest.mark.parametrize("case", CASES, ids=lambda c: c[0])
def test_decode_partials(case):
    name, cache_dt, lens, T, H, st = case
    g = np.random.default_rng(zlib.crc32(name.encode()))
    bt, num_pages = _pool(lens, spare=2, seed=len(name))
    q_dt = "f32" if cache_dt == "f32" else "bf16"
    cache, scale, vals = _random_cache(g, num_pages, cache_dt)
    B = len(lens)
    q = g.standard_normal((B * T, H, 576)).astype(np.float32) * 0.25
    q = round_bf16(q) if q_dt == "bf16" else q
    S = -(-bt.shape[1] * 64 // st)
    o_part = torch.full((B * T, H, S, 512), float("nan"), device="cuda")
    lse_part = torch.full((B * T, H, S), float("nan"), device="cuda")
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    scale_f = 1 / math.sqrt(192)
    mla.mla_decode_fwd(to_device(q, q_dt), DT[q_dt], cache, scale, DT[cache_dt], num_pages,
                       torch.from_numpy(bt).cuda(), bt.shape[1], 64, torch.tensor(lens, dtype=torch.int32).cuda(),
                       B, T, H, S, st, scale_f, o_part, lse_part, err)
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    got_o, got_l = to_host_f64(o_part), to_host_f64(lse_part)
    tol_o = 1e-5 if cache_dt == "f32" else 5e-3
    tol_l = 1e-5 if cache_dt == "f32" else 2e-3
    for b, L in enumerate(lens):
        slots = bt[b, np.arange(L) // 64].astype(np.int64) * 64 + np.arange(L) % 64
        rows = vals[slots]
        qq = q[b * T:(b + 1) * T].astype(np.float64)
        ref_o, ref_l = oracle.attention_partials(qq[..., :512], qq[..., 512:], rows[:, :512], rows[:, 512:],
                                                 st, S, scale_f)
        go, gl = got_o[b * T:(b + 1) * T], got_l[b * T:(b + 1) * T]
        # A kernel may merge a run of consecutive splits into the run's first
        # split (the others then report lse = -inf): each finite lse_part[s]
        # starts a run that ends at the next finite split, and must equal the
        # oracle's partials merged over that run.  Splits that see no row are
        # -inf in every case.
        fin_ref = np.isfinite(ref_l)
        assert np.all(np.isneginf(gl[~fin_ref])), f"seq {b}: empty splits must report -inf"
        for t in range(T):
            for h in range(H):
                starts = np.nonzero(np.isfinite(gl[t, h]))[0]
                assert starts.size and starts[0] == 0, f"seq {b}: the first split must hold a partial"
                ends = list(starts[1:]) + [S]
                for s0, s1 in zip(starts, ends):
                    mo, ml = oracle.combine_partials(ref_o[t, h, s0:s1], ref_l[t, h, s0:s1])
                    ref_o[t, h, s0], ref_l[t, h, s0] = mo, ml
                    ref_l[t, h, s0 + 1:s1] = -np.inf
        fin = np.isfinite(gl)
        assert np.array_equal(fin, np.isfinite(ref_l)), f"seq {b}: runs of merged splits"
        assert oracle.normwise_rel_err(go[fin], ref_o[fin]) < tol_o, f"seq {b} o_part"
        np.testing.assert_allclose(gl[fin], ref_l[fin], rtol=0, atol=tol_l)


def test_decode_bad_page_is_skipped_and_flagged():
    lens = [256]
    bt, num_pages = _pool(lens, spare=0, seed=9)
    g = np.random.default_rng(10)
    cache, _, vals = _random_cache(g, num_pages, "bf16")
    q = round_bf16(g.standard_normal((1, 128, 576)).astype(np.float32) * 0.25)
    bt_bad = bt.copy(); bt_bad[0, 2] = num_pages + 3          # rows 128..191 point outside the pool
    o_part = torch.empty((1, 128, 1, 512), device="cuda"); lse_part = torch.empty((1, 128, 1), device="cuda")
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    mla.mla_decode_fwd(to_device(q, "bf16"), mla.MLA_BF16, cache, None, mla.MLA_BF16, num_pages,
                       torch.from_numpy(bt_bad).cuda(), bt.shape[1], 64, torch.tensor(lens, dtype=torch.int32).cuda(),
                       1, 1, 128, 1, 256, 1 / math.sqrt(192), o_part, lse_part, err)
    torch.cuda.synchronize()
    assert int(err.item()) & mla.MLA_DEVERR_PAGE
    keep = np.r_[0:128, 192:256]
    slots = bt[0, keep // 64].astype(np.int64) * 64 + keep % 64
    rows = vals[slots]
    qq = q.astype(np.float64)
    ref_o, ref_l = oracle.attention_partials(qq[..., :512], qq[..., 512:], rows[:, :512], rows[:, 512:], 256, 1,
                                             1 / math.sqrt(192))
    assert oracle.normwise_rel_err(to_host_f64(o_part), ref_o) < 5e-3


def test_decode_split_invariance_and_paging_bit_identity():
    """The result does not depend on the split count (within rounding), and a
    permuted page pool gives bit-identical partials to a contiguous one."""
    lens = [1500, 900]
    g = np.random.default_rng(11)
    B, H = 2, 128
    npg = [(L + 63) // 64 for L in lens]
    num_pages = sum(npg)
    cache, _, vals = _random_cache(g, num_pages, "bf16")
    q = to_device(round_bf16(g.standard_normal((B, H, 576)).astype(np.float32) * 0.25), "bf16")
    contig = np.full((B, max(npg)), -1, np.int32)
    off = 0
    for b, n in enumerate(npg):
        contig[b, :n] = np.arange(off, off + n); off += n
    perm = g.permutation(num_pages)
    cache_p = torch.empty_like(cache)
    cache_p[torch.from_numpy(perm).cuda().long()] = cache    # page i moves to slot perm[i]
    paged = np.where(contig >= 0, perm[np.maximum(contig, 0)], -1).astype(np.int32)
    lens_t = torch.tensor(lens, dtype=torch.int32).cuda()

    def run(tab, cch, st):
        S = -(-tab.shape[1] * 64 // st)
        o = torch.empty((B, H, S, 512), device="cuda"); l = torch.empty((B, H, S), device="cuda")
        mla.mla_decode_fwd(q, mla.MLA_BF16, cch, None, mla.MLA_BF16, num_pages, torch.from_numpy(tab).cuda(),
                           tab.shape[1], 64, lens_t, B, 1, H, S, st, 1 / math.sqrt(192), o, l)
        ol = torch.empty((B, H, 512), device="cuda"); ll = torch.empty((B, H), device="cuda")
        mla.mla_combine(o, l, B, H, S, ol, mla.MLA_F32, ll)
        torch.cuda.synchronize()
        return o, l, ol, ll

    o1, l1, ol1, ll1 = run(contig, cache, 256)
    o2, l2, ol2, ll2 = run(paged, cache_p, 256)
    # splits with no visible row (lse = -inf) leave o_part unwritten
    fin = torch.isfinite(l1)
    assert torch.equal(l1, l2) and torch.equal(o1[fin], o2[fin])
    assert not bool(fin.all()), "the case must include empty splits"
    assert bool(torch.isneginf(l1[~fin]).all())
    base = to_host_f64(ol1)
    for st in [64, 512, 2048]:
        _, _, ol, ll = run(contig, cache, st)
        assert oracle.normwise_rel_err(to_host_f64(ol), base) < 5e-3
        np.testing.assert_allclose(to_host_f64(ll), to_host_f64(ll1), atol=2e-3)
