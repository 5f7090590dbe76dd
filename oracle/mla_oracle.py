"""Plain fp64 CPU oracle of absorbed Multi-head Latent Attention (MLA) decode.

TEST INFRASTRUCTURE ONLY: imported by ``tests/``, ``__graft_entry__.smoke()``
and ``bench.py``'s cpu-baseline leg, never by the product path.

It is written to be checked by eye against the pages it follows, with no
blocking, fusion or reordering beyond what their formulas state.  Sources
(page title, then the section or equation used):

  [V2-C]   "DeepSeek-V2: MLA Explained" (mibrahim.dev), section "MLA Full
           Formulas": 1. Query Compression, 2. Key-Value Joint Compression,
           3. Attention Calculation; "Caching Strategy"; "Optimization Note".
  [V3-KV]  "KV Compression - DeepSeek-V3" (ai-engineer-exhaustive), sections
           "How it works" (Eq. (1), the 576-wide wkv_a map, RMSNorm on the
           latent) and "Official code" (kv_norm, kv_cache / pe_cache).
  [CURIO]  "Latent Attention." (llm.curionode.com), "Compress, then rebuild":
           cache arithmetic for DeepSeek-V3's shape.
  [DENIZ]  "DeepSeek'in MLA'si latent attention ile KV cache'i %93
           sikistiriyor" (deniz.in): sections on the latent vector, decoupled
           RoPE and absorption.
  [OCP-FP8] the OCP 8-bit floating point specification, E4M3 format (bias 7,
           max 448, no infinities, NaN = S.1111.111); used for the e4m3 cache
           with one fp32 scale per token (absmax/448).

Readings where the pages are silent:
  * RoPE pairs channels (2i, 2i+1), angle = pos * theta^(-2i/64), theta=1e4,
    rotation [x0 cos - x1 sin, x0 sin + x1 cos].
  * RMSNorm(x) = x / sqrt(mean(x^2) + eps) * gain, eps = 1e-6.
  * The cache stores the normalised latent and the rotated rope key (576
    numbers per token, one contiguous row).
  * q_pe arrives already rotated (RoPE is applied upstream of the path).
  * The attention sum over j <= t includes the current token; a step's T new
    tokens are appended before attending; query t of a sequence with L cached
    rows (new rows included) sits at position L - T + t.
  * W_UK, W_UV are stored [H, 128, 512]: k^C_h = W_UK[h] c, v^C_h = W_UV[h] c.
  * The attention core ends at the per-head 128-d outputs; the output
    projection u = W_O [o_1; ...; o_H] (out_projection) and the wkv_a
    projection that produces the cached rows (kv_a_projection) are the
    steps on either side of it.  W_O is [d, H*128] with head h's element i
    at column h*128 + i; W_kv,a is [576, d].
  * e4m3 cache: one fp32 scale per token over all 576 values, scale = a/448
    with a = max |x|; code = RNE-satfinite(x * 448 / a); a = 0 -> all zero.
  * 8-bit tensor-core MMAs over an e4m3 cache take the query as two e4m3
    terms on one fp32 scale per (row, head) (split_query_e4m3); the pages
    fix no such encoding, and the attention itself is still checked against
    the exact formulas above.
"""
from __future__ import annotations

import math
from typing import Optional, Tuple

import numpy as np

D_C, D_R, D_N, D_V = 512, 64, 128, 128
D_ROW = D_C + D_R


# --------------------------------------------------------------------------
# cache arithmetic  [CURIO] "Compress, then rebuild"; [V3-KV] "How it works";
# [DENIZ] latent-vector and absorption sections
# --------------------------------------------------------------------------
def mla_cache_numbers_per_token(d_c: int = D_C, d_r: int = D_R) -> int:
    """Numbers cached per token per layer by MLA: latent plus shared rope key."""
    return d_c + d_r


def mha_cache_numbers_per_token(n_h: int, d_h: int) -> int:
    """Numbers cached per token per layer by multi-head attention: K and V."""
    return 2 * n_h * d_h


def gqa_cache_numbers_per_token(n_g: int, d_h: int) -> int:
    """Grouped-query attention with n_g key-value heads."""
    return 2 * n_g * d_h


def cache_bytes_per_token(numbers_per_layer: int, layers: int, bytes_per_number: int) -> int:
    return numbers_per_layer * layers * bytes_per_number


# --------------------------------------------------------------------------
# storage rounding
# --------------------------------------------------------------------------
def round_to_bf16(x: np.ndarray) -> np.ndarray:
    """Round fp64 values to the nearest bfloat16 (8 significant bits), ties to
    even, directly from fp64 (no intermediate fp32 rounding)."""
    x = np.asarray(x, dtype=np.float64)
    out = np.zeros_like(x)
    nz = (x != 0) & np.isfinite(x)
    e = np.floor(np.log2(np.abs(x[nz])))
    q = np.ldexp(1.0, (e - 7).astype(np.int64))           # spacing in that binade
    out[nz] = np.rint(x[nz] / q) * q                       # rint: half to even
    out[~np.isfinite(x)] = x[~np.isfinite(x)]
    return out


def round_to_f32(x: np.ndarray) -> np.ndarray:
    return np.asarray(x, dtype=np.float64).astype(np.float32).astype(np.float64)


# --------------------------------------------------------------------------
# OCP FP8 E4M3 codec  [OCP-FP8]
# --------------------------------------------------------------------------
E4M3_MAX = 448.0


def e4m3_decode(codes: np.ndarray) -> np.ndarray:
    """Value of each 8-bit E4M3 code: sign bit 7, exponent bits 6..3 (bias 7),
    mantissa bits 2..0; exponent 0 is subnormal (m * 2^-9); S.1111.111 is NaN;
    there are no infinities."""
    c = np.asarray(codes, dtype=np.int64) & 0xFF
    s = np.where(c & 0x80, -1.0, 1.0)
    e = (c >> 3) & 0xF
    m = c & 0x7
    val = np.where(e == 0, m * 2.0 ** -9, (1.0 + m / 8.0) * np.ldexp(1.0, (e - 7).astype(np.int64)))
    val = s * val
    return np.where((e == 0xF) & (m == 0x7), np.nan, val)


def e4m3_encode(x: np.ndarray) -> np.ndarray:
    """Nearest E4M3 code (ties to even mantissa), saturating to +-448."""
    x = np.asarray(x, dtype=np.float64)
    sign = (np.signbit(x)).astype(np.int64) << 7
    a = np.minimum(np.abs(x), E4M3_MAX)
    e = np.floor(np.log2(np.where(a > 0, a, 1.0)))
    e = np.clip(e, -6, 8)                                  # subnormals share 2^-6's spacing
    q = np.ldexp(1.0, (e - 3).astype(np.int64))             # 3 mantissa bits
    r = np.rint(a / q) * q                                  # half to even
    r = np.minimum(r, E4M3_MAX)
    # re-derive the code of the rounded magnitude
    er = np.floor(np.log2(np.where(r > 0, r, 1.0)))
    sub = r < 2.0 ** -6
    code_sub = np.rint(r / 2.0 ** -9).astype(np.int64)
    er_c = np.clip(er, -6, 8).astype(np.int64)
    mant = np.rint((r / np.ldexp(1.0, er_c) - 1.0) * 8).astype(np.int64)
    code_norm = ((er_c + 7) << 3) | mant
    code = np.where(sub, code_sub, code_norm)
    code = np.where(r == 0, 0, code)
    return (code | sign).astype(np.uint8)


def quantize_rows_e4m3(rows: np.ndarray) -> Tuple[np.ndarray, np.ndarray]:
    """Per-token e4m3 quantisation of cache rows [n, 576] (fp64).

    scale = max|x| / 448 (one fp32 per token); code = e4m3(x * 448 / max|x|).
    Returns (codes uint8 [n, 576], scale float64 [n])."""
    a = np.max(np.abs(rows), axis=1)
    inv = np.where(a > 0, E4M3_MAX / np.where(a > 0, a, 1.0), 0.0)
    codes = e4m3_encode(rows * inv[:, None])
    scale = a / E4M3_MAX
    return codes, scale


def dequantize_rows_e4m3(codes: np.ndarray, scale: np.ndarray) -> np.ndarray:
    return e4m3_decode(codes) * np.asarray(scale, dtype=np.float64)[:, None]


def split_query_e4m3(q: np.ndarray) -> Tuple[np.ndarray, np.ndarray, np.ndarray]:
    """Two-term e4m3 form of absorbed queries q [..., 576] (fp32 values):
    the query operand of the 8-bit tensor-core decode over an e4m3 cache.

    Not a step of the pages: with an e4m3 cache ([DENIZ] cache section,
    [OCP-FP8]) both operands of an 8-bit MMA are 8-bit, so the query is
    carried as two e4m3 terms on one fp32 scale per (row, head), in fp32:
        a = max |q|;  inv = fp32(448 / a) (0 when a = 0);  y = fp32(q * inv)
        hi = e4m3(y);  lo = e4m3(y - hi)   (y - hi is exact in fp32)
        scale = fp32(a / 448)
    so that q ~ scale * (hi + lo) to about 2^-8 relative.
    Returns (hi codes, lo codes) uint8 [..., 576] and scale float32 [...]."""
    q32 = np.asarray(q, dtype=np.float32)
    a = np.max(np.abs(q32), axis=-1)
    inv = np.where(a > 0, np.float32(E4M3_MAX) / np.where(a > 0, a, np.float32(1)), np.float32(0)).astype(np.float32)
    y = (q32 * inv[..., None]).astype(np.float32)
    hi = e4m3_encode(y.astype(np.float64))
    lo = e4m3_encode(y.astype(np.float64) - e4m3_decode(hi))
    scale = (a / np.float32(E4M3_MAX)).astype(np.float32)
    return hi, lo, scale


# --------------------------------------------------------------------------
# cache write: RMSNorm on the latent, RoPE on the shared rope key
# --------------------------------------------------------------------------
def rms_norm(c: np.ndarray, gain: Optional[np.ndarray] = None, eps: float = 1e-6) -> np.ndarray:
    """c_hat = RMSNorm(c_KV)  [V3-KV] "How it works" / "Official code" (kv_norm).
    Rows of c: x / sqrt(mean(x^2) + eps) * gain."""
    c = np.asarray(c, dtype=np.float64)
    ms = np.mean(c * c, axis=-1, keepdims=True)
    y = c / np.sqrt(ms + eps)
    if gain is not None:
        y = y * np.asarray(gain, dtype=np.float64)
    return y


def rope_angles(pos: np.ndarray, theta: float = 10000.0, d: int = D_R) -> np.ndarray:
    """Rotation angle of pair i at position p: p * theta^(-2i/d), [n, d/2]."""
    i = np.arange(d // 2, dtype=np.float64)
    inv_freq = theta ** (-2.0 * i / d)
    return np.asarray(pos, dtype=np.float64)[:, None] * inv_freq[None, :]


def rope(x: np.ndarray, pos: np.ndarray, theta: float = 10000.0) -> np.ndarray:
    """k^R_t = RoPE(W^KR h_t)  [V2-C] §2; pairs (2i, 2i+1) rotated by the angle
    of pair i at the row's position."""
    x = np.asarray(x, dtype=np.float64)
    ang = rope_angles(pos, theta, x.shape[-1])
    cs, sn = np.cos(ang), np.sin(ang)
    x0, x1 = x[..., 0::2], x[..., 1::2]
    y = np.empty_like(x)
    y[..., 0::2] = x0 * cs - x1 * sn
    y[..., 1::2] = x0 * sn + x1 * cs
    return y


def cache_rows(kv_a: np.ndarray, pos: np.ndarray, gain=None, eps: float = 1e-6,
               theta: float = 10000.0) -> np.ndarray:
    """One cache row per token from the 576-wide wkv_a output  [V3-KV] "How it
    works": split [512, 64], RMSNorm the latent, RoPE the rope key; [V2-C]
    "Caching Strategy": only (c_KV, k^R) are cached.  Returns fp64 [n, 576]."""
    kv_a = np.asarray(kv_a, dtype=np.float64)
    c = rms_norm(kv_a[:, :D_C], gain, eps)
    kr = rope(kv_a[:, D_C:], pos, theta)
    return np.concatenate([c, kr], axis=1)


def kv_a_projection(h: np.ndarray, w_kva: np.ndarray) -> np.ndarray:
    """The joint down-projection that feeds the cache  [V3-KV] "How it works",
    Eq. (1) and the widened official map: [c_t^KV ; k~_t^R] = W_kv,a h_t, one
    576-wide row per token (512 latent channels, then the 64 rope channels
    before RoPE).  h [n, d], w_kva [576, d] -> fp64 [n, 576]."""
    h = np.asarray(h, np.float64); w_kva = np.asarray(w_kva, np.float64)
    if w_kva.shape[0] != D_ROW or w_kva.shape[1] != h.shape[1]:
        raise ValueError("kv_a_projection: w_kva must be [576, d] for h [n, d]")
    return h @ w_kva.T


def cache_rows_from_hidden(h: np.ndarray, w_kva: np.ndarray, pos: np.ndarray, gain=None, eps: float = 1e-6,
                           theta: float = 10000.0) -> np.ndarray:
    """Cache rows straight from the hidden states: the wkv_a projection, then
    the split / RMSNorm / RoPE of cache_rows  [V3-KV] "How it works" and
    "Official code" (split(wkv_a(x), [512, 64]), kv_norm)."""
    return cache_rows(kv_a_projection(h, w_kva), pos, gain, eps, theta)


def stored_rows(rows: np.ndarray, cache_dtype: str):
    """What a cache of the given storage dtype holds for fp64 rows.
    Returns (values fp64 [n, 576], codes or None, scale or None)."""
    if cache_dtype == "f32":
        return round_to_f32(rows), None, None
    if cache_dtype == "bf16":
        return round_to_bf16(rows), None, None
    if cache_dtype == "e4m3":
        codes, scale = quantize_rows_e4m3(rows)
        scale32 = round_to_f32(scale)
        return dequantize_rows_e4m3(codes, scale32), codes, scale32
    raise ValueError(cache_dtype)


# --------------------------------------------------------------------------
# attention, naive form  [V2-C] §1-§3 (Appendix C formulas)
# --------------------------------------------------------------------------
def decompress_kv(c_hat, w_uk, w_uv):
    """Per-head keys and values of cached latents, [V2-C] §2 ("up-project"):
    k^C_{j,i} = W^UK_i c_j and v^C_{j,i} = W^UV_i c_j.  c_hat [L, 512],
    w_uk / w_uv [H, 128, 512]; returns k_c, v_c [L, H, 128].  This is the
    "decompress" step of the non-absorbed (level 2) decode."""
    c_hat = np.asarray(c_hat, np.float64)
    k_c = np.einsum("lc,hkc->lhk", c_hat, np.asarray(w_uk, np.float64))
    v_c = np.einsum("lc,hkc->lhk", c_hat, np.asarray(w_uv, np.float64))
    return k_c, v_c


def attention_naive(q_nope, q_pe, w_uk, w_uv, c_hat, k_r, softmax_scale=None):
    """Per-head output o_{t,i} of one sequence, naive form.

    q_nope [T, H, 128], q_pe [T, H, 64]: q^C_{t,i} and q^R_{t,i} ([V2-C] §1);
    w_uk, w_uv [H, 128, 512]; c_hat [L, 512], k_r [L, 64]: the cached rows.
    Query t sits at position L - T + t and sees rows j = 0 .. L - T + t.

      k^C_{j,i} = W^UK_i c_j,  v^C_{j,i} = W^UV_i c_j          [V2-C] §2
      k_{j,i} = [k^C_{j,i}; k^R_j],  q_{t,i} = [q^C_{t,i}; q^R_{t,i}]
      o_{t,i} = sum_j softmax_j(q_{t,i}^T k_{j,i} / sqrt(d_h + d_h^R)) v^C_{j,i}   [V2-C] §3
    """
    q_nope = np.asarray(q_nope, np.float64); q_pe = np.asarray(q_pe, np.float64)
    w_uk = np.asarray(w_uk, np.float64); w_uv = np.asarray(w_uv, np.float64)
    c_hat = np.asarray(c_hat, np.float64); k_r = np.asarray(k_r, np.float64)
    T, H, _ = q_nope.shape
    L = c_hat.shape[0]
    scale = 1.0 / math.sqrt(D_N + D_R) if softmax_scale is None else softmax_scale
    out = np.zeros((T, H, D_V))
    k_all, v_all = decompress_kv(c_hat, w_uk, w_uv)  # [L, H, 128]: row j = W^UK_i c_j, W^UV_i c_j
    for i in range(H):
        k_c, v_c = k_all[:, i], v_all[:, i]
        k = np.concatenate([k_c, k_r], axis=1)       # [L, 192]
        for t in range(T):
            n_vis = L - T + t + 1
            q = np.concatenate([q_nope[t, i], q_pe[t, i]])   # [192]
            z = (k[:n_vis] @ q) * scale
            p = np.exp(z - z.max())
            p = p / p.sum()
            out[t, i] = p @ v_c[:n_vis]
    return out


# --------------------------------------------------------------------------
# attention, absorbed form  [V2-C] "Optimization Note"; [DENIZ] absorption
# section; [CURIO] "folded into the query and output projections"
# --------------------------------------------------------------------------
def absorb_q(q_nope, w_uk):
    """Latent query q_lat[t, i] = W^UK_i^T q^C_{t,i}  ([T, H, 512]): since
    q^C . (W^UK c) = (W^UK^T q^C) . c, the key up-projection folds into q."""
    return np.einsum("thk,hkc->thc", np.asarray(q_nope, np.float64), np.asarray(w_uk, np.float64))


def attention_absorbed(q_nope, q_pe, w_uk, w_uv, c_hat, k_r, softmax_scale=None):
    """Same output as attention_naive, computed in latent space.

      z_j = scale * (q_lat . c_j + q^R . k^R_j)
      o_lat = sum_j softmax_j(z) c_j,   lse = log sum_j exp(z_j)
      out = W^UV_i o_lat                 (value up-projection after the sum)
    Returns (out [T,H,128], o_lat [T,H,512], lse [T,H])."""
    q_pe = np.asarray(q_pe, np.float64)
    c_hat = np.asarray(c_hat, np.float64); k_r = np.asarray(k_r, np.float64)
    T, H, _ = q_pe.shape
    L = c_hat.shape[0]
    scale = 1.0 / math.sqrt(D_N + D_R) if softmax_scale is None else softmax_scale
    q_lat = absorb_q(q_nope, w_uk)
    z = ((q_lat.reshape(T * H, D_C) @ c_hat.T + q_pe.reshape(T * H, D_R) @ k_r.T) * scale).reshape(T, H, L)
    for t in range(T):
        z[t, :, L - T + t + 1:] = -np.inf
    m = z.max(axis=-1, keepdims=True)
    e = np.exp(z - m)
    s = e.sum(axis=-1, keepdims=True)
    p = e / s
    o_lat = (p.reshape(T * H, L) @ c_hat).reshape(T, H, D_C)
    lse = (m + np.log(s))[..., 0]
    out = np.einsum("thc,hvc->thv", o_lat, np.asarray(w_uv, np.float64))
    return out, o_lat, lse


# --------------------------------------------------------------------------
# split-KV partials and their log-sum-exp combine (exact decomposition of the
# softmax sum of [V2-C] §3 over disjoint token ranges)
# --------------------------------------------------------------------------
def attention_partials(q_lat, q_pe, c_hat, k_r, split_tokens: int, num_splits: int,
                       softmax_scale=None):
    """Per split s (rows [s*split_tokens, (s+1)*split_tokens) that the query
    sees): o_s = softmax-weighted mean of c over the split, lse_s = log of the
    split's sum of exp(z).  A split with no visible row has lse = -inf, o = 0.
    q_lat [T, H, 512], q_pe [T, H, 64] -> (o [T, H, S, 512], lse [T, H, S])."""
    q_lat = np.asarray(q_lat, np.float64); q_pe = np.asarray(q_pe, np.float64)
    c_hat = np.asarray(c_hat, np.float64); k_r = np.asarray(k_r, np.float64)
    T, H, _ = q_lat.shape
    L = c_hat.shape[0]
    scale = 1.0 / math.sqrt(D_N + D_R) if softmax_scale is None else softmax_scale
    o = np.zeros((T, H, num_splits, D_C))
    lse = np.full((T, H, num_splits), -np.inf)
    for t in range(T):
        n_vis = L - T + t + 1
        for s in range(num_splits):
            lo, hi = s * split_tokens, min((s + 1) * split_tokens, n_vis)
            if lo >= hi:
                continue
            z = (q_lat[t] @ c_hat[lo:hi].T + q_pe[t] @ k_r[lo:hi].T) * scale   # [H, n]
            m = z.max(axis=1, keepdims=True)
            e = np.exp(z - m)
            ssum = e.sum(axis=1, keepdims=True)
            o[t, :, s] = (e / ssum) @ c_hat[lo:hi]
            lse[t, :, s] = (m + np.log(ssum))[:, 0]
    return o, lse


def combine_partials(o_part, lse_part):
    """Merge split partials: M = max_s lse_s, w_s = exp(lse_s - M),
    o = sum_s w_s o_s / sum_s w_s, lse = M + log sum_s w_s.
    When no split saw a row (every lse_s = -inf): o = 0, lse = -inf.
    o_part [..., S, 512], lse_part [..., S] -> (o [..., 512], lse [...])."""
    o_part = np.asarray(o_part, np.float64); lse_part = np.asarray(lse_part, np.float64)
    M = lse_part.max(axis=-1, keepdims=True)
    seen = np.isfinite(M)                                  # some split saw a row
    Ms = np.where(seen, M, 0.0)
    w = np.where(np.isfinite(lse_part), np.exp(lse_part - Ms), 0.0)
    ws = w.sum(axis=-1, keepdims=True)
    o = (w[..., None] * o_part).sum(axis=-2) / np.where(seen, ws, 1.0)
    lse = np.where(seen, Ms + np.log(np.where(seen, ws, 1.0)), -np.inf)
    return o, lse[..., 0]


def out_uv(o_lat, w_uv):
    """out[t, i] = W^UV_i o_lat[t, i]  (value up-projection, [V2-C] §2, moved
    after the softmax sum)."""
    return np.einsum("thc,hvc->thv", np.asarray(o_lat, np.float64), np.asarray(w_uv, np.float64))


def out_projection(out, w_o):
    """u_t = W_O [o_{t,1}; o_{t,2}; ...; o_{t,n_h}]  ([V2-C] §3, "Concatenate
    all heads and project"): the heads' 128-wide outputs are concatenated in
    head order (element i of head h at h*128 + i) and multiplied by W_O.
    out [T, H, 128], w_o [d, H*128] -> fp64 [T, d]."""
    out = np.asarray(out, np.float64); w_o = np.asarray(w_o, np.float64)
    T, H, dv = out.shape
    if w_o.shape[1] != H * dv:
        raise ValueError("out_projection: w_o must be [d, H*128]")
    return out.reshape(T, H * dv) @ w_o.T


# --------------------------------------------------------------------------
# whole decode step of one sequence, from raw inputs
# --------------------------------------------------------------------------
def sequence_cache(kv_a_rows, cache_dtype: str, gain=None, eps=1e-6, theta=10000.0):
    """Cache contents (as stored) of one sequence whose rows sit at positions
    0..L-1.  Returns (c_hat [L,512], k_r [L,64]) fp64 values as stored."""
    L = kv_a_rows.shape[0]
    rows = cache_rows(kv_a_rows, np.arange(L), gain, eps, theta)
    vals, _, _ = stored_rows(rows, cache_dtype)
    return vals[:, :D_C], vals[:, D_C:]


def decode_step_sequence(q_nope, q_pe, w_uk, w_uv, kv_a_rows, cache_dtype: str,
                         gain=None, eps=1e-6, theta=10000.0, form: str = "absorbed"):
    """Output [T, H, 128] of one sequence's decode step (naive or absorbed)."""
    c_hat, k_r = sequence_cache(kv_a_rows, cache_dtype, gain, eps, theta)
    if form == "naive":
        return attention_naive(q_nope, q_pe, w_uk, w_uv, c_hat, k_r)
    return attention_absorbed(q_nope, q_pe, w_uk, w_uv, c_hat, k_r)[0]


def normwise_rel_err(got, ref) -> float:
    """max over (t, h) of ||got - ref||_2 / ||ref||_2 over the last axis."""
    got = np.asarray(got, np.float64); ref = np.asarray(ref, np.float64)
    num = np.linalg.norm(got - ref, axis=-1)
    den = np.linalg.norm(ref, axis=-1)
    return float(np.max(num / np.maximum(den, 1e-300)))
