"""Seeded synthetic inputs for absorbed-MLA decode.

This module is shared by the oracle side (tests, cpu baseline) and the GPU
side (tests, bench, smoke).  It holds *no* arithmetic of the method: it only
draws random numbers, casts them to the storage dtype a workload names, and
lays out lengths and page tables.  RMSNorm, RoPE, quantisation, absorption and
attention live in ``oracle/`` (CPU, fp64) and in the CUDA library, separately.

Workloads (DeepSeek-V3 head shape: d_nope = d_v = 128, d_rope = 64, d_c = 512):

  tiny      B=1,   T=1, H=16,  L=256,              fp32, contiguous
  v3_b1     B=1,   T=1, H=128, L=4096,             bf16, contiguous
  serving   B=64,  T=1, H=128, L~U[1024,8192],     bf16, paged, permuted pages
  long      B=8,   T=1, H=128, L=131072,           bf16, paged, 64 splits x 2048
  fp8_mtp   B=128, T=2, H=128, L=4096,             e4m3 cache + per-token scale,
                                                   bf16 queries/weights, paged

Value distributions: q_nope, q_pe ~ N(0,1); W_UK, W_UV ~ N(0, 1/512); the raw
kv_a projection rows (512 latent + 64 rope channels) ~ N(0,1).  The cache is
built from those raw rows by the append step (RMSNorm on the latent, RoPE at
the row's position on the rope channels), on each side independently.

Every tensor draws from its own numpy Philox stream keyed by
(seed, tensor id, sequence index), so one sequence can be regenerated alone.
"""
from __future__ import annotations

import dataclasses
from typing import Dict, List, Optional

import numpy as np

D_C = 512        # joint KV latent width (kv_lora_rank)
D_R = 64         # decoupled rope key width (qk_rope_head_dim)
D_N = 128        # per-head nope query/key width (qk_nope_head_dim)
D_V = 128        # per-head value width (v_head_dim)
D_ROW = D_C + D_R  # 576 numbers cached per token per layer
PAGE = 64        # tokens per cache page

# tensor ids for the Philox key
_T_KVA, _T_QN, _T_QP, _T_WUK, _T_WUV, _T_LEN, _T_PERM, _T_GAIN = range(8)


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    batch: int
    q_len: int            # T: query tokens per sequence (new tokens this step)
    n_heads: int
    seq_len: Optional[int]  # fixed L (None: drawn per sequence)
    len_range: Optional[tuple]  # (lo, hi) inclusive when seq_len is None
    dtype: str            # "f32" | "bf16": queries, weights, raw kv rows
    cache_dtype: str      # "f32" | "bf16" | "e4m3"
    paged: bool           # True: permuted page pool; False: identity table
    split_tokens: int     # split-KV chunk length (multiple of PAGE)
    seed: int = 0
    theta: float = 10000.0
    eps: float = 1e-6

    @property
    def softmax_scale(self) -> float:
        return 1.0 / float(np.sqrt(D_N + D_R))


WORKLOADS: Dict[str, Workload] = {
    "tiny": Workload("tiny", 1, 1, 16, 256, None, "f32", "f32", False, 64),
    "v3_b1": Workload("v3_b1", 1, 1, 128, 4096, None, "bf16", "bf16", False, 128),
    "serving": Workload("serving", 64, 1, 128, None, (1024, 8192), "bf16", "bf16", True, 2048),
    "long": Workload("long", 8, 1, 128, 131072, None, "bf16", "bf16", True, 2048),
    "fp8_mtp": Workload("fp8_mtp", 128, 2, 128, 4096, None, "bf16", "e4m3", True, 2048),
}
WORKLOAD_ORDER: List[str] = ["tiny", "v3_b1", "serving", "long", "fp8_mtp"]


def _rng(seed: int, tensor: int, index: int = 0) -> np.random.Generator:
    return np.random.Generator(np.random.Philox(key=[seed * 1000 + tensor, index]))


def round_bf16(x: np.ndarray) -> np.ndarray:
    """Round float32 values to the nearest bfloat16 (ties to even); returns
    float32 holding bf16-representable values.  Storage cast of an input."""
    u = np.array(x, dtype=np.float32, copy=True).view(np.uint32)
    if not np.isfinite(u.view(np.float32)).all():
        raise ValueError("round_bf16: non-finite input")
    # finite inputs: u + 0x8000 stays below 2**32, so 32-bit arithmetic is exact
    lsb = (u >> 16) & 1
    u += np.uint32(0x7FFF)
    u += lsb
    u &= np.uint32(0xFFFF0000)
    return u.view(np.float32)


def bf16_bits(x: np.ndarray) -> np.ndarray:
    """bf16-representable float32 -> raw uint16 bit patterns."""
    return (np.ascontiguousarray(x, dtype=np.float32).view(np.uint32) >> 16).astype(np.uint16)


def cast(x: np.ndarray, dtype: str) -> np.ndarray:
    x = np.asarray(x, dtype=np.float32)
    if dtype == "f32":
        return x
    if dtype == "bf16":
        return round_bf16(x)
    raise ValueError(dtype)


def seq_lens(w: Workload) -> np.ndarray:
    if w.seq_len is not None:
        return np.full(w.batch, w.seq_len, dtype=np.int32)
    lo, hi = w.len_range
    return _rng(w.seed, _T_LEN).integers(lo, hi + 1, size=w.batch).astype(np.int32)


def pages_per_seq(lens: np.ndarray) -> np.ndarray:
    return (lens.astype(np.int64) + PAGE - 1) // PAGE


def block_table(w: Workload, lens: Optional[np.ndarray] = None):
    """Return (block_table [B, max_pages] int32, num_pages).

    Contiguous workloads hand out pages in order (sequence b owns a run of
    consecutive pages, so the cache bytes equal a dense [L, 576] array).
    Paged workloads hand out a seeded Fisher-Yates permutation of one global
    pool.  Unused table entries are -1."""
    lens = seq_lens(w) if lens is None else lens
    npg = pages_per_seq(lens)
    total = int(npg.sum())
    ids = np.arange(total, dtype=np.int64)
    if w.paged:
        ids = _rng(w.seed, _T_PERM).permutation(total)
    maxp = int(npg.max())
    bt = np.full((w.batch, maxp), -1, dtype=np.int32)
    off = 0
    for b in range(w.batch):
        bt[b, : npg[b]] = ids[off: off + npg[b]]
        off += npg[b]
    return bt, total


def kv_rows(w: Workload, b: int, lo: int = 0, hi: Optional[int] = None) -> np.ndarray:
    """Raw kv_a projection rows [hi-lo, 576] of sequence b (positions lo..hi-1),
    cast to the workload dtype.  Drawn in blocks of 4096 positions so any
    window is reproducible without drawing the whole sequence."""
    L = int(seq_lens(w)[b])
    hi = L if hi is None else hi
    out = np.empty((hi - lo, D_ROW), dtype=np.float32)
    blk = 4096
    for s in range(lo // blk, (hi + blk - 1) // blk):
        g = _rng(w.seed, _T_KVA, b * 100000 + s)
        rows = g.standard_normal((blk, D_ROW), dtype=np.float32)
        a, e = max(lo, s * blk), min(hi, (s + 1) * blk)
        out[a - lo: e - lo] = rows[a - s * blk: e - s * blk]
    return cast(out, w.dtype)


def queries(w: Workload):
    """(q_nope [B*T, H, 128], q_pe [B*T, H, 64]) in the workload dtype."""
    r = w.batch * w.q_len
    qn = _rng(w.seed, _T_QN).standard_normal((r, w.n_heads, D_N), dtype=np.float32)
    qp = _rng(w.seed, _T_QP).standard_normal((r, w.n_heads, D_R), dtype=np.float32)
    return cast(qn, w.dtype), cast(qp, w.dtype)


def weights(w: Workload):
    """(W_UK, W_UV), each [H, 128, 512] ~ N(0, 1/512), in the workload dtype."""
    std = 1.0 / np.sqrt(D_C)
    wuk = _rng(w.seed, _T_WUK).standard_normal((w.n_heads, D_N, D_C), dtype=np.float32) * np.float32(std)
    wuv = _rng(w.seed, _T_WUV).standard_normal((w.n_heads, D_V, D_C), dtype=np.float32) * np.float32(std)
    return cast(wuk, w.dtype), cast(wuv, w.dtype)


def norm_gain(w: Workload, kind: str = "ones") -> np.ndarray:
    """RMSNorm gain [512] fp32: all ones (the workloads) or a seeded draw
    around 1 (used by tests that must see the gain applied)."""
    if kind == "ones":
        return np.ones(D_C, dtype=np.float32)
    return (1.0 + 0.25 * _rng(w.seed, _T_GAIN).standard_normal(D_C)).astype(np.float32)


def new_token_positions(w: Workload, lens: Optional[np.ndarray] = None):
    """(seq_ids, positions) int32 of the T new tokens per sequence, in the
    row order of the step's query rows (r = b*T + t -> position L_b - T + t)."""
    lens = seq_lens(w) if lens is None else lens
    sid = np.repeat(np.arange(w.batch, dtype=np.int32), w.q_len)
    pos = np.concatenate([np.arange(L - w.q_len, L, dtype=np.int32) for L in lens])
    return sid, pos


def with_overrides(w: Workload, **kw) -> Workload:
    return dataclasses.replace(w, **kw)
