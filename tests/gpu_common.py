"""Helpers for the GPU tests: oracle references of seeded workloads and the
error measures the parity gates use."""
from __future__ import annotations

import numpy as np

import oracle
import workloads as W

# parity gates: max normwise relative error of each 128-d head output
TOL = {"bf16": 1e-2, "e4m3": 3e-2, "f32": 1e-4}


def reference_sequence(w: W.Workload, b: int, gain=None, heads=None, form="absorbed"):
    """Oracle output of sequence b: (out [T,H,128], o_lat [T,H,512], lse [T,H]).
    form='naive' returns (out, None, None) for the listed heads only."""
    kv = W.kv_rows(w, b)
    qn, qp = W.queries(w)
    wuk, wuv = W.weights(w)
    rows = slice(b * w.q_len, (b + 1) * w.q_len)
    qn, qp = qn[rows], qp[rows]
    c_hat, k_r = oracle.sequence_cache(kv, w.cache_dtype, gain, w.eps, w.theta)
    if form == "naive":
        hs = list(range(w.n_heads)) if heads is None else list(heads)
        out = oracle.attention_naive(qn[:, hs], qp[:, hs], wuk[hs], wuv[hs], c_hat, k_r)
        return out, None, None
    return oracle.attention_absorbed(qn, qp, wuk, wuv, c_hat, k_r)


def gpu_rows(t, b, q_len):
    from workloads.device import to_host_f64
    return to_host_f64(t[b * q_len:(b + 1) * q_len])


def bf16_exact_or_boundary(gpu: np.ndarray, ref64: np.ndarray, rel=4e-6) -> np.ndarray:
    """True where the GPU's bf16 value is the correctly rounded oracle value,
    or where the oracle value lies within `rel` (the fp32 arithmetic error of
    the kernel) of the rounding boundary between the two.  Returns the mask of
    violating elements."""
    r = oracle.round_to_bf16(ref64)
    bad = gpu != r
    if not bad.any():
        return bad
    mid = 0.5 * (gpu + r)
    near = np.abs(ref64 - mid) <= rel * np.abs(ref64)
    one_ulp = np.abs(gpu - r) <= np.abs(r) * 2.0 ** -7 + 1e-300
    return bad & ~(near & one_ulp)
