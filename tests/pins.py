"""Pins that tie the oracle to something other than itself.

Each ``pin_*`` function raises AssertionError when the oracle disagrees with
what the pages print, a closed form, an invariant, an independent library
routine or brute force on tiny inputs.  ``test_oracle.py`` runs them all;
``test_oracle_mutations.py`` plants plausible mistakes in the oracle and
checks that at least one pin catches each.
"""
from __future__ import annotations

import json
import math
import os

import numpy as np

import oracle

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")
SCALE = 1.0 / math.sqrt(192.0)


def _rng(seed):
    return np.random.default_rng(seed)


def _problem(seed, T=1, H=3, L=5):
    g = _rng(seed)
    q_nope = g.standard_normal((T, H, 128))
    q_pe = g.standard_normal((T, H, 64))
    w_uk = g.standard_normal((H, 128, 512)) / math.sqrt(512)
    w_uv = g.standard_normal((H, 128, 512)) / math.sqrt(512)
    c = oracle.rms_norm(g.standard_normal((L, 512)))
    kr = g.standard_normal((L, 64))
    return q_nope, q_pe, w_uk, w_uv, c, kr


# ---------------------------------------------------------------- printed values
def pin_cache_arithmetic():
    """Every cache size the pages print, from the oracle's arithmetic."""
    with open(os.path.join(GOLDEN, "cache_arithmetic.json")) as f:
        items = json.load(f)["items"]
    mla = oracle.mla_cache_numbers_per_token()
    for it in items:
        k = it["kind"]
        if k == "mla_numbers":
            v = mla
        elif k == "mha_numbers":
            v = oracle.mha_cache_numbers_per_token(it["n_h"], it["d_h"])
        elif k == "ratio_mha_mla":
            v = oracle.mha_cache_numbers_per_token(it["n_h"], it["d_h"]) / mla
        elif k == "ratio_gqa_mla":
            v = oracle.gqa_cache_numbers_per_token(it["n_g"], it["d_h"]) / mla
        elif k == "mha_bytes":
            v = oracle.cache_bytes_per_token(oracle.mha_cache_numbers_per_token(it["n_h"], it["d_h"]),
                                             it["layers"], it["bytes"]) / it["unit"]
        elif k == "mla_bytes":
            v = oracle.cache_bytes_per_token(mla, it["layers"], it["bytes"]) / it["unit"]
        elif k == "mla_seq_bytes":
            v = oracle.cache_bytes_per_token(mla, it["layers"], it["bytes"]) * it["tokens"] / it["unit"]
        elif k == "mha_seq_bytes":
            v = oracle.cache_bytes_per_token(oracle.mha_cache_numbers_per_token(it["n_h"], it["d_h"]),
                                             it["layers"], it["bytes"]) * it["tokens"] / it["unit"]
        elif k == "latent_compression":
            v = oracle.mha_cache_numbers_per_token(it["n_h"], it["d_h"]) / oracle.D_C
        elif k == "reduction_pct":
            v = 100.0 * (1.0 - mla / oracle.mha_cache_numbers_per_token(it["n_h"], it["d_h"]))
        else:
            raise AssertionError(f"unknown kind {k}")
        assert round(v, it["digits"]) == it["printed"], (it["what"], v, it["printed"])
    # exact byte counts behind the rounded figures
    assert oracle.cache_bytes_per_token(mla, 61, 2) == 70272
    assert oracle.cache_bytes_per_token(mla, 61, 2) * 131072 == 9_210_691_584


# ---------------------------------------------------------------- RMSNorm
def pin_rmsnorm():
    g = _rng(1)
    c = g.standard_normal((7, 512)) * 3.0
    eps = 1e-6
    y = oracle.rms_norm(c, None, eps)
    ms = np.mean(c * c, axis=1)
    # mean of squares after the norm is 1 / (1 + eps / mean(c^2)), in closed form
    np.testing.assert_allclose(np.mean(y * y, axis=1), 1.0 / (1.0 + eps / ms), rtol=1e-13)
    # with eps = 0 the norm is scale invariant and keeps direction
    np.testing.assert_allclose(oracle.rms_norm(5.0 * c, None, 0.0), oracle.rms_norm(c, None, 0.0), rtol=1e-13)
    cos = np.sum(y * c, axis=1) / np.linalg.norm(y, axis=1) / np.linalg.norm(c, axis=1)
    np.testing.assert_allclose(cos, 1.0, rtol=1e-13)
    gain = g.standard_normal(512)
    np.testing.assert_allclose(oracle.rms_norm(c, gain, eps), y * gain, rtol=1e-13)
    # a constant row x = a normalises to a / sqrt(a^2 + eps)
    z = oracle.rms_norm(np.full((1, 512), 2.0), None, eps)
    np.testing.assert_allclose(z, 2.0 / math.sqrt(4.0 + eps), rtol=1e-15)


# ---------------------------------------------------------------- RoPE
def pin_rope():
    theta = 10000.0
    # channel pair 0 turns at 1 rad per position; pair i at theta^(-2i/64)
    e0 = np.zeros((1, 64)); e0[0, 0] = 1.0
    y = oracle.rope(e0, np.array([3]), theta)
    expect = np.zeros(64); expect[0] = math.cos(3.0); expect[1] = math.sin(3.0)
    np.testing.assert_allclose(y[0], expect, atol=1e-15)
    e3 = np.zeros((1, 64)); e3[0, 3] = 1.0          # second channel of pair 1
    a = 7.0 * theta ** (-2.0 / 64.0)
    y = oracle.rope(e3, np.array([7]), theta)
    expect = np.zeros(64); expect[2] = -math.sin(a); expect[3] = math.cos(a)
    np.testing.assert_allclose(y[0], expect, atol=1e-15)
    g = _rng(2)
    x = g.standard_normal((5, 64))
    pos = np.array([0, 1, 17, 4095, 131071])
    y = oracle.rope(x, pos, theta)
    np.testing.assert_allclose(y[0], x[0], rtol=0, atol=0)          # position 0 is the identity
    pn = lambda v: np.hypot(v[..., 0::2], v[..., 1::2])
    np.testing.assert_allclose(pn(y), pn(x), rtol=1e-13)            # pair norms kept
    # <RoPE_m q, RoPE_n k> depends on n - m only
    q, k = g.standard_normal(64), g.standard_normal(64)
    d1 = oracle.rope(q[None], np.array([5]))[0] @ oracle.rope(k[None], np.array([12]))[0]
    d2 = oracle.rope(q[None], np.array([1005]))[0] @ oracle.rope(k[None], np.array([1012]))[0]
    np.testing.assert_allclose(d1, d2, rtol=1e-10)


# ---------------------------------------------------------------- e4m3 codec
def pin_e4m3():
    import torch
    codes = np.arange(256, dtype=np.uint8)
    ref = torch.from_numpy(codes.copy()).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    mine = oracle.e4m3_decode(codes)
    assert np.array_equal(np.isnan(ref), np.isnan(mine))
    fin = ~np.isnan(ref)
    assert np.array_equal(ref[fin], mine[fin])
    # every finite code survives decode -> encode (zero keeps its sign bit)
    assert np.array_equal(oracle.e4m3_encode(mine[fin]), codes[fin])
    # encode agrees with torch's float8_e4m3fn rounding inside the finite range
    g = _rng(3)
    pos_vals = np.unique(mine[fin][mine[fin] > 0])
    mids = 0.5 * (pos_vals[1:] + pos_vals[:-1])                 # exact ties
    x = np.concatenate([g.standard_normal(20000) * 50, g.uniform(-448, 448, 20000),
                        g.standard_normal(5000) * 2.0 ** -7, mine[fin], mids, -mids])
    t = torch.from_numpy(x).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(oracle.e4m3_encode(x), t)
    # ties go to the even mantissa; the top of the range saturates to 448
    assert oracle.e4m3_encode(np.array([0.5 * 2.0 ** -9]))[0] == 0x00
    assert oracle.e4m3_encode(np.array([1.5 * 2.0 ** -9]))[0] == 0x02
    assert oracle.e4m3_encode(np.array([1.0 + 1.0 / 16]))[0] == 0x38
    assert oracle.e4m3_encode(np.array([1.0 + 3.0 / 16]))[0] == 0x3A
    assert oracle.e4m3_encode(np.array([448.0, 500.0, -1e9]))[0] == 0x7E
    assert oracle.e4m3_encode(np.array([-1e9]))[0] == 0xFE
    # per-token quantisation: the absmax element maps to +-448 exactly
    rows = g.standard_normal((9, 576))
    c, s = oracle.quantize_rows_e4m3(rows)
    am = np.argmax(np.abs(rows), axis=1)
    assert np.all(np.abs(oracle.e4m3_decode(c[np.arange(9), am])) == 448.0)
    np.testing.assert_allclose(s, np.max(np.abs(rows), axis=1) / 448.0, rtol=1e-15)
    deq = oracle.dequantize_rows_e4m3(c, s)
    # relative error of one e4m3 rounding is at most 2^-4 for normal values
    big = np.abs(rows) > 2.0 ** -6 * s[:, None]
    assert np.all(np.abs(deq - rows)[big] <= 2.0 ** -4 * np.abs(rows)[big] + 1e-300)
    z, zs = oracle.quantize_rows_e4m3(np.zeros((1, 576)))
    assert np.all(z == 0) and zs[0] == 0.0


def pin_split_query_e4m3():
    """hi is a nearest e4m3 value to y = fp32(q * fp32(448 / max|q|)) and lo a
    nearest to y - hi, checked by exhaustive search over every finite code
    (tie-breaking is pinned by pin_e4m3); the absmax element maps to +-448;
    hi + lo carries y to max(2^-8 |y|, 2^-10)."""
    g = _rng(41)
    vals = oracle.e4m3_decode(np.arange(256, dtype=np.uint8))
    table = vals[~np.isnan(vals)]

    def nearest_dist(x):
        return np.min(np.abs(x[:, None] - table[None, :]), axis=1)

    q = (g.standard_normal((3, 5, 576)) * np.exp(g.uniform(-4, 4, (3, 5, 1)))).astype(np.float32)
    q[0, 1, :] = 0.0                                   # a zero (row, head)
    hi, lo, sc = oracle.split_query_e4m3(q)
    assert hi.shape == q.shape and lo.shape == q.shape and sc.shape == (3, 5)
    a = np.abs(q).max(-1)
    inv = np.where(a > 0, np.float32(448.0) / np.where(a > 0, a, np.float32(1)), np.float32(0)).astype(np.float32)
    yf = (q * inv[..., None]).astype(np.float32).astype(np.float64).reshape(-1)
    vh, vl = oracle.e4m3_decode(hi).reshape(-1), oracle.e4m3_decode(lo).reshape(-1)
    assert np.all(np.abs(yf - vh) <= nearest_dist(yf) + 1e-12)
    r = yf - vh
    assert np.all(np.abs(r - vl) <= nearest_dist(r) + 1e-15)
    err = np.abs(yf - vh - vl)
    assert np.all(err <= np.maximum(2.0 ** -8 * np.abs(yf), 2.0 ** -10))
    am = np.argmax(np.abs(q), axis=-1)
    top = np.take_along_axis(np.abs(oracle.e4m3_decode(hi)), am[..., None], -1)[..., 0]
    assert np.all(top[a > 0] == 448.0)
    np.testing.assert_allclose(sc, a / 448.0, rtol=2.0 ** -23)
    assert np.all(hi[0, 1] == 0) and np.all(lo[0, 1] == 0) and sc[0, 1] == 0.0
    # q ~ scale * (hi + lo) to about 2^-8 of max|q| per element
    rec = sc[..., None].astype(np.float64) * (oracle.e4m3_decode(hi) + oracle.e4m3_decode(lo))
    assert np.max(np.abs(rec - q) / np.maximum(a[..., None], 1e-30)) <= 2.0 ** -8 * 1.01

def pin_bf16_rounding():
    import torch
    g = _rng(4)
    x = np.concatenate([g.standard_normal(50000) * 10.0 ** g.integers(-8, 8, 50000)])
    # exact fp64 -> bf16 with ties to even, compared where fp32 keeps all the
    # information needed (values exactly representable in fp32)
    x32 = x.astype(np.float32).astype(np.float64)
    ref = torch.from_numpy(x32).to(torch.float32).to(torch.bfloat16).to(torch.float64).numpy()
    assert np.array_equal(oracle.round_to_bf16(x32), ref)
    # a midpoint between two bf16 numbers rounds to the even one
    assert oracle.round_to_bf16(np.array([1.0 + 2.0 ** -8]))[0] == 1.0
    assert oracle.round_to_bf16(np.array([1.0 + 3 * 2.0 ** -8]))[0] == 1.0 + 2.0 ** -6


# ---------------------------------------------------------------- attention
def pin_naive_equals_absorbed():
    """Distributive property: folding W_UK into q and W_UV after the sum gives
    the naive result ([V2-C] Optimization Note)."""
    for seed, (T, H, L) in enumerate([(1, 3, 5), (2, 4, 9), (1, 2, 64), (2, 2, 65), (1, 1, 1)]):
        args = _problem(10 + seed, T, H, L)
        a = oracle.attention_naive(*args)
        b, _, _ = oracle.attention_absorbed(*args)
        assert oracle.normwise_rel_err(b, a) < 1e-12, (T, H, L)


def pin_single_row():
    """L = 1: softmax weight 1, out = W_UV c_0 exactly."""
    q_nope, q_pe, w_uk, w_uv, c, kr = _problem(20, 1, 4, 1)
    expect = np.stack([w_uv[h] @ c[0] for h in range(4)])[None]
    assert oracle.normwise_rel_err(oracle.attention_naive(q_nope, q_pe, w_uk, w_uv, c, kr), expect) < 1e-14
    assert oracle.normwise_rel_err(oracle.attention_absorbed(q_nope, q_pe, w_uk, w_uv, c, kr)[0], expect) < 1e-14


def pin_uniform_scores():
    """q = 0: every score equal, out = W_UV mean(c)."""
    q_nope, q_pe, w_uk, w_uv, c, kr = _problem(21, 1, 3, 37)
    q_nope[:] = 0; q_pe[:] = 0
    expect = np.stack([w_uv[h] @ c.mean(axis=0) for h in range(3)])[None]
    for f in (oracle.attention_naive, lambda *a: oracle.attention_absorbed(*a)[0]):
        assert oracle.normwise_rel_err(f(q_nope, q_pe, w_uk, w_uv, c, kr), expect) < 1e-13


def pin_two_rows_sigmoid():
    """L = 2: out = (1 - s) v_0 + s v_1 with s = sigmoid(z_1 - z_0) and
    z_j = (q^C . W_UK c_j + q^R . k^R_j) / sqrt(192)."""
    q_nope, q_pe, w_uk, w_uv, c, kr = _problem(22, 1, 3, 2)
    out_n = oracle.attention_naive(q_nope, q_pe, w_uk, w_uv, c, kr)
    out_a = oracle.attention_absorbed(q_nope, q_pe, w_uk, w_uv, c, kr)[0]
    for h in range(3):
        z = [(q_nope[0, h] @ (w_uk[h] @ c[j]) + q_pe[0, h] @ kr[j]) / math.sqrt(192.0) for j in range(2)]
        s = 1.0 / (1.0 + math.exp(-(z[1] - z[0])))
        expect = (1 - s) * (w_uv[h] @ c[0]) + s * (w_uv[h] @ c[1])
        np.testing.assert_allclose(out_n[0, h], expect, rtol=1e-12)
        np.testing.assert_allclose(out_a[0, h], expect, rtol=1e-12)


def pin_row_permutation():
    """The softmax sum runs over a set: permuting cached rows (latent and rope
    key together) leaves the output unchanged when every row is visible."""
    q_nope, q_pe, w_uk, w_uv, c, kr = _problem(23, 1, 2, 50)
    perm = _rng(5).permutation(50)
    a = oracle.attention_absorbed(q_nope, q_pe, w_uk, w_uv, c, kr)[0]
    b = oracle.attention_absorbed(q_nope, q_pe, w_uk, w_uv, c[perm], kr[perm])[0]
    assert oracle.normwise_rel_err(a, b) < 1e-13


def pin_causal():
    """With T = 2, query 0 sits at L-2 and does not see row L-1; query 1 does."""
    q_nope, q_pe, w_uk, w_uv, c, kr = _problem(24, 2, 2, 9)
    c2, kr2 = c.copy(), kr.copy()
    c2[-1] = -c2[-1] * 3; kr2[-1] += 5
    for f in (oracle.attention_naive, lambda *a: oracle.attention_absorbed(*a)[0]):
        a = f(q_nope, q_pe, w_uk, w_uv, c, kr)
        b = f(q_nope, q_pe, w_uk, w_uv, c2, kr2)
        np.testing.assert_allclose(a[0], b[0], rtol=1e-13)
        assert np.max(np.abs(a[1] - b[1])) > 1e-3
    # query 0 equals a T = 1 problem on the first L-1 rows
    a0 = oracle.attention_naive(q_nope[:1], q_pe[:1], w_uk, w_uv, c[:-1], kr[:-1])
    np.testing.assert_allclose(oracle.attention_naive(q_nope, q_pe, w_uk, w_uv, c, kr)[0], a0[0], rtol=1e-13)


def _brute(q_nope, q_pe, w_uk, w_uv, c, kr):
    """Appendix-C formulas with scalar Python loops only."""
    T, H = len(q_nope), len(q_nope[0])
    L = len(c)
    out = [[[0.0] * 128 for _ in range(H)] for _ in range(T)]
    for t in range(T):
        nv = L - T + t + 1
        for h in range(H):
            kc = [[sum(w_uk[h][a][b] * c[j][b] for b in range(512)) for a in range(128)] for j in range(nv)]
            vc = [[sum(w_uv[h][a][b] * c[j][b] for b in range(512)) for a in range(128)] for j in range(nv)]
            z = []
            for j in range(nv):
                dot = sum(q_nope[t][h][a] * kc[j][a] for a in range(128))
                dot += sum(q_pe[t][h][r] * kr[j][r] for r in range(64))
                z.append(dot / math.sqrt(128 + 64))
            m = max(z)
            e = [math.exp(v - m) for v in z]
            s = sum(e)
            for a in range(128):
                out[t][h][a] = sum(e[j] / s * vc[j][a] for j in range(nv))
    return np.array(out)


def pin_brute_force():
    for seed, (T, H, L) in enumerate([(1, 1, 3), (2, 1, 3)]):
        args = _problem(30 + seed, T, H, L)
        ref = _brute(*[a.tolist() for a in args])
        assert oracle.normwise_rel_err(oracle.attention_naive(*args), ref) < 1e-12
        assert oracle.normwise_rel_err(oracle.attention_absorbed(*args)[0], ref) < 1e-12


def pin_split_combine():
    """Log-sum-exp combine of split partials equals the unsplit softmax."""
    q_nope, q_pe, w_uk, w_uv, c, kr = _problem(40, 2, 3, 200)
    out, o_lat, lse = oracle.attention_absorbed(q_nope, q_pe, w_uk, w_uv, c, kr)
    q_lat = oracle.absorb_q(q_nope, w_uk)
    for S, st in [(1, 256), (2, 128), (7, 29), (64, 4), (4, 64)]:
        o, l = oracle.attention_partials(q_lat, q_pe, c, kr, st, S)
        oc, lc = oracle.combine_partials(o, l)
        np.testing.assert_allclose(oc, o_lat, rtol=1e-12, atol=1e-14)
        np.testing.assert_allclose(lc, lse, rtol=1e-12)
        np.testing.assert_allclose(oracle.out_uv(oc, w_uv), out, rtol=1e-11, atol=1e-14)
    # lse is the log of the softmax normaliser: exp(lse) = sum_j exp(z_j)
    z = (q_lat[0, 0] @ c[:199].T + q_pe[0, 0] @ kr[:199].T) / math.sqrt(192.0)
    np.testing.assert_allclose(lse[0, 0], math.log(np.sum(np.exp(z))), rtol=1e-13)


def pin_cache_rows():
    """A cache row is [RMSNorm(latent); RoPE(rope key)] of the 576-wide row."""
    g = _rng(6)
    kv = g.standard_normal((4, 576))
    pos = np.array([0, 3, 64, 9999])
    rows = oracle.cache_rows(kv, pos)
    assert rows.shape == (4, 576)
    np.testing.assert_allclose(rows[:, :512], oracle.rms_norm(kv[:, :512]), rtol=1e-15)
    np.testing.assert_allclose(rows[0, 512:], kv[0, 512:], rtol=0)     # position 0
    pn = lambda v: np.hypot(v[..., 0::2], v[..., 1::2])
    np.testing.assert_allclose(pn(rows[:, 512:]), pn(kv[:, 512:]), rtol=1e-13)


def pin_normwise_rel_err():
    """The parity gate: max over (t, h) of ||got - ref||_2 / ||ref||_2 over the
    last axis, checked on hand-computed values.  Head 0 of token 0 has ref
    (3, 4), norm 5, and error (0, 1): ratio 0.2; head 1 has ref (1, 0) and
    error (0.5, 0): ratio 0.5; token 1 has ratios 0.25 and 0.6.  The answer
    is 0.6.  A mean (0.3875), the norm taken over the wrong axis, a
    denominator taken from `got`, one global norm ratio (0.44) or a constant 0
    all give something else."""
    ref = np.array([[[3.0, 4.0], [1.0, 0.0]],
                    [[0.0, 2.0], [5.0, 0.0]]])
    got = np.array([[[3.0, 5.0], [1.5, 0.0]],
                    [[0.0, 2.5], [5.0, 3.0]]])
    # token 1: head 0 error 0.5 over norm 2 -> 0.25; head 1 error 3 over norm 5 -> 0.6
    err = oracle.normwise_rel_err(got, ref)
    assert abs(err - 0.6) < 1e-15, err
    assert oracle.normwise_rel_err(ref, ref) == 0.0
    # scale invariance, and the argument order matters (ref is the denominator)
    assert abs(oracle.normwise_rel_err(7.0 * got, 7.0 * ref) - 0.6) < 1e-15
    swapped = oracle.normwise_rel_err(ref, got)
    assert abs(swapped - max(1 / np.hypot(3, 5), 0.5 / 1.5, 0.5 / np.hypot(0, 2.5), 3 / np.hypot(5, 3))) < 1e-15
    # one (t, h) far off dominates however many are exact
    big = np.ones((3, 5, 16)); off = big.copy(); off[2, 4, 0] += 16.0
    assert abs(oracle.normwise_rel_err(off, big) - 4.0) < 1e-15


def pin_out_projection():
    """u = W_O [o_1; ...; o_H]: identity W_O gives the heads concatenated in
    head order; a one-hot row of W_O picks out exactly one (head, element);
    scalar loops agree; and W_O composed with W_UV per head (the value
    up-projection combined with the output projection) gives the same u."""
    g = _rng(71)
    T, H = 2, 3
    out = g.standard_normal((T, H, 128))
    # identity: u[t] = [out[t,0,:], out[t,1,:], out[t,2,:]]
    u = oracle.out_projection(out, np.eye(H * 128))
    np.testing.assert_array_equal(u, np.concatenate([out[:, h, :] for h in range(H)], axis=1))
    # one-hot rows: row j of W_O selects element i of head h at column h*128 + i
    sel = [(0, 5), (1, 0), (2, 127), (1, 77)]
    w = np.zeros((len(sel), H * 128))
    for j, (h, i) in enumerate(sel):
        w[j, h * 128 + i] = 1.0
    u = oracle.out_projection(out, w)
    for j, (h, i) in enumerate(sel):
        np.testing.assert_array_equal(u[:, j], out[:, h, i])
    # scalar loops on a small non-square W_O
    d = 5
    w = g.standard_normal((d, H * 128))
    u = oracle.out_projection(out, w)
    for t in range(T):
        for j in range(d):
            ref = 0.0
            for h in range(H):
                for i in range(128):
                    ref += w[j, h * 128 + i] * out[t, h, i]
            assert abs(u[t, j] - ref) <= 1e-12 * (1 + abs(ref))
    # folding: sum_h (W_O[:, h] W_UV[h]) o_lat[h] == W_O [W_UV o_lat]
    q_nope, q_pe, w_uk, w_uv, c, kr = _problem(72, T, H, 40)
    o, o_lat, _ = oracle.attention_absorbed(q_nope, q_pe, w_uk, w_uv, c, kr)
    u1 = oracle.out_projection(o, w)
    u2 = sum(o_lat[:, h, :] @ (w[:, h * 128:(h + 1) * 128] @ w_uv[h]).T for h in range(H))
    np.testing.assert_allclose(u1, u2, rtol=1e-11, atol=1e-13)


def pin_kv_a_projection():
    """[c; k~R] = W_kv,a h: identity W gives h back; a one-hot row picks one
    hidden channel; scalar loops agree; and the cache rows built from h go
    through the same [512, 64] split, RMSNorm and RoPE as cache_rows."""
    g = _rng(73)
    n = 3
    h = g.standard_normal((n, 576))
    np.testing.assert_array_equal(oracle.kv_a_projection(h, np.eye(576)), h)
    d = 40
    h = g.standard_normal((n, d))
    w = np.zeros((576, d))
    w[0, 7] = 1.0; w[511, 0] = 1.0; w[512, 39] = 1.0; w[575, 3] = 1.0
    kv = oracle.kv_a_projection(h, w)
    np.testing.assert_array_equal(kv[:, 0], h[:, 7]); np.testing.assert_array_equal(kv[:, 511], h[:, 0])
    np.testing.assert_array_equal(kv[:, 512], h[:, 39]); np.testing.assert_array_equal(kv[:, 575], h[:, 3])
    w = g.standard_normal((576, d))
    kv = oracle.kv_a_projection(h, w)
    for t in range(n):
        for j in (0, 100, 511, 512, 575):
            ref = sum(w[j, k] * h[t, k] for k in range(d))
            assert abs(kv[t, j] - ref) <= 1e-12 * (1 + abs(ref))
    pos = np.array([0, 5, 4095])
    np.testing.assert_allclose(oracle.cache_rows_from_hidden(h, w, pos), oracle.cache_rows(kv, pos), rtol=0, atol=0)
    # the latent half is RMS-normalised, the rope half keeps its pair norms
    rows = oracle.cache_rows_from_hidden(h, w, pos)
    np.testing.assert_allclose(np.mean(rows[:, :512] ** 2, axis=1),
                               1.0 / (1.0 + 1e-6 / np.mean(kv[:, :512] ** 2, axis=1)), rtol=1e-12)
    pn = lambda v: np.hypot(v[..., 0::2], v[..., 1::2])
    np.testing.assert_allclose(pn(rows[:, 512:]), pn(kv[:, 512:]), rtol=1e-13)


def pin_decompress_kv():
    """k^C = W^UK c, v^C = W^UV c per head: one-hot rows of W pick single
    latent components; W^UK and W^UV are not swapped; scalar loops agree."""
    g = _rng(83)
    L, H = 3, 2
    c = g.standard_normal((L, 512))
    w_uk = np.zeros((H, 128, 512))
    w_uv = np.zeros((H, 128, 512))
    # head h, output i picks latent component (7 i + h) mod 512 for keys, (5 i + 3 h + 1) mod 512 for values
    for h in range(H):
        for i in range(128):
            w_uk[h, i, (7 * i + h) % 512] = 1.0
            w_uv[h, i, (5 * i + 3 * h + 1) % 512] = 1.0
    k_c, v_c = oracle.decompress_kv(c, w_uk, w_uv)
    assert k_c.shape == (L, H, 128) and v_c.shape == (L, H, 128)
    for h in range(H):
        for i in range(128):
            np.testing.assert_array_equal(k_c[:, h, i], c[:, (7 * i + h) % 512])
            np.testing.assert_array_equal(v_c[:, h, i], c[:, (5 * i + 3 * h + 1) % 512])
    # scalar loops with dense weights
    w_uk = g.standard_normal((H, 128, 512)) / 20
    w_uv = g.standard_normal((H, 128, 512)) / 20
    k_c, v_c = oracle.decompress_kv(c, w_uk, w_uv)
    for j in range(L):
        for h in range(H):
            for i in (0, 63, 127):
                rk = sum(w_uk[h, i, m] * c[j, m] for m in range(512))
                rv = sum(w_uv[h, i, m] * c[j, m] for m in range(512))
                assert abs(k_c[j, h, i] - rk) <= 1e-12 * (1 + abs(rk))
                assert abs(v_c[j, h, i] - rv) <= 1e-12 * (1 + abs(rv))


ALL_PINS = [pin_cache_arithmetic, pin_rmsnorm, pin_rope, pin_e4m3, pin_bf16_rounding,
            pin_naive_equals_absorbed, pin_single_row, pin_uniform_scores, pin_two_rows_sigmoid,
            pin_row_permutation, pin_causal, pin_brute_force, pin_split_combine, pin_cache_rows,
            pin_normwise_rel_err, pin_out_projection, pin_kv_a_projection, pin_decompress_kv,
            pin_split_query_e4m3]
