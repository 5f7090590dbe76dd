"""One layer's decode step over a paged latent cache, as five library calls.

``DecodeStep`` owns the device buffers of one layer (cache, page table,
rope tables, workspace and outputs, as torch tensors) and runs

    mla_cache_append -> mla_absorb_q -> mla_decode_fwd -> mla_combine -> mla_out_uv

on one stream (over an e4m3 cache with 65..128 heads: mla_absorb_q then
mla_split_q_e4m3, and mla_decode_fwd_q8 for the attention).  It only allocates and marshals; every step runs in libmla.
``DecodeStep.capture`` records the same calls as CUDA graphs, for steps whose
device work is shorter than the host time of five marshalled calls.
"""
from __future__ import annotations

import math

import numpy as np

from . import (D_C, D_R, D_ROW, D_V, MLA_BF16, MLA_E4M3, MLA_F32, PAGE, mla_absorb_q, mla_cache_append,
               mla_combine, mla_combine_out_uv, mla_decode_fwd, mla_decode_fwd_q8, mla_split_q_e4m3, mla_kv_proj_append, mla_kv_proj_workspace_bytes, mla_out_proj,
               mla_out_uv, mla_rope_table)

_DT = {"f32": MLA_F32, "bf16": MLA_BF16, "e4m3": MLA_E4M3}


def _torch_dtype(code):
    import torch
    return {MLA_F32: torch.float32, MLA_BF16: torch.bfloat16, MLA_E4M3: torch.uint8}[code]


class DecodeStep:
    """Device state of one layer for `batch` sequences with `q_len` new tokens.

    block_table: int32 [batch, max_pages] (host array or tensor); num_pages:
    size of the page pool; split_tokens: split-KV chunk (multiple of 64).
    q8: with an e4m3 cache, bf16 queries and 65..128 heads the attention runs
    on 8-bit MMAs (mla_split_q_e4m3 in absorb, mla_decode_fwd_q8 in attend)
    unless q8=False, which keeps mla_decode_fwd's widened f16 operands."""

    def __init__(self, *, batch, q_len, n_heads, dtype, cache_dtype, block_table, num_pages,
                 split_tokens, max_pos=None, theta=10000.0, eps=1e-6, norm_gain=None,
                 softmax_scale=None, device="cuda", q8=None):
        import torch
        self.torch = torch
        self.batch, self.q_len, self.n_heads = int(batch), int(q_len), int(n_heads)
        self.dtype, self.cache_dtype = _DT[dtype], _DT[cache_dtype]
        self.device = torch.device(device)
        bt = torch.as_tensor(np.asarray(block_table, dtype=np.int32))
        self.block_table = bt.to(self.device)
        self.max_pages = int(bt.shape[1])
        self.num_pages = int(num_pages)
        self.split_tokens = int(split_tokens)
        self.num_splits = int(math.ceil(self.max_pages * PAGE / self.split_tokens))
        self.eps = float(eps)
        self.softmax_scale = float(softmax_scale if softmax_scale is not None else 1.0 / math.sqrt(192.0))
        self.max_pos = int(max_pos if max_pos is not None else self.max_pages * PAGE)
        cos = np.empty((self.max_pos, D_R // 2), np.float32)
        sin = np.empty_like(cos)
        mla_rope_table(theta, self.max_pos, cos, sin)
        self.rope_cos = torch.from_numpy(cos).to(self.device)
        self.rope_sin = torch.from_numpy(sin).to(self.device)
        self.norm_gain = None if norm_gain is None else torch.as_tensor(
            np.asarray(norm_gain, np.float32)).to(self.device)
        dev = self.device
        # zero-filled: the tensor-core decode reads whole pages (see mla_decode_fwd)
        self.cache = torch.zeros((self.num_pages, D_ROW // 64, PAGE, 64), dtype=_torch_dtype(self.cache_dtype),
                                 device=dev)
        self.cache_scale = (torch.zeros((self.num_pages, PAGE), dtype=torch.float32, device=dev)
                            if self.cache_dtype == MLA_E4M3 else None)
        rows = self.batch * self.q_len
        qdt = _torch_dtype(self.dtype)
        self.q_abs = torch.empty((rows, self.n_heads, D_ROW), dtype=qdt, device=dev)
        # e4m3 cache, bf16 queries, 65..128 heads: both GEMMs on 8-bit MMAs from
        # the query's two-term e4m3 form (q8=False keeps the widened f16 operands)
        q8_ok = self.cache_dtype == MLA_E4M3 and self.dtype == MLA_BF16 and 64 < self.n_heads <= 128
        if q8 and not q8_ok:
            raise ValueError("q8 needs an e4m3 cache, bf16 queries and 65..128 heads")
        self.q8 = q8_ok if q8 is None else bool(q8)
        self.q_e4m3 = (torch.empty((rows, 2, self.n_heads, D_ROW), dtype=torch.uint8, device=dev)
                       if self.q8 else None)
        self.q_scale = torch.empty((rows, self.n_heads), dtype=torch.float32, device=dev) if self.q8 else None
        self.o_part = torch.empty((rows, self.n_heads, self.num_splits, D_C), dtype=torch.float32, device=dev)
        self.lse_part = torch.empty((rows, self.n_heads, self.num_splits), dtype=torch.float32, device=dev)
        self.o_lat = torch.empty((rows, self.n_heads, D_C), dtype=qdt, device=dev)
        self.lse = torch.empty((rows, self.n_heads), dtype=torch.float32, device=dev)
        self.out = torch.empty((rows, self.n_heads, D_V), dtype=qdt, device=dev)
        self.err = torch.zeros(1, dtype=torch.int32, device=dev)
        self.seq_lens = torch.zeros(self.batch, dtype=torch.int32, device=dev)

    # -- individual calls ------------------------------------------------
    def append(self, kv_a, seq_ids, positions, stream=None):
        mla_cache_append(kv_a, _DT["f32"] if kv_a.dtype == self.torch.float32 else MLA_BF16,
                         kv_a.shape[0], seq_ids, positions, self.block_table, self.batch, self.max_pages,
                         PAGE, self.norm_gain, self.eps, self.rope_cos, self.rope_sin, self.max_pos,
                         self.cache, self.cache_scale, self.cache_dtype, self.num_pages, self.err, stream)

    def absorb(self, q_nope, q_pe, w_uk, stream=None):
        """q_abs = [W_UK^T q_nope; q_pe]; with q8 also its two-term e4m3 form."""
        mla_absorb_q(q_nope, q_pe, w_uk, self.q_abs, self.batch * self.q_len, self.n_heads, self.dtype, stream)
        if self.q8:
            mla_split_q_e4m3(self.q_abs, self.batch * self.q_len, self.n_heads, self.q_e4m3, self.q_scale, stream)

    def attend(self, stream=None):
        if self.q8:
            mla_decode_fwd_q8(self.q_e4m3, self.q_scale, self.cache, self.cache_scale, self.num_pages,
                              self.block_table, self.max_pages, PAGE, self.seq_lens, self.batch, self.q_len,
                              self.n_heads, self.num_splits, self.split_tokens, self.softmax_scale, self.o_part,
                              self.lse_part, self.err, stream)
            return
        mla_decode_fwd(self.q_abs, self.dtype, self.cache, self.cache_scale, self.cache_dtype, self.num_pages,
                       self.block_table, self.max_pages, PAGE, self.seq_lens, self.batch, self.q_len,
                       self.n_heads, self.num_splits, self.split_tokens, self.softmax_scale, self.o_part,
                       self.lse_part, self.err, stream)

    def combine(self, stream=None):
        mla_combine(self.o_part, self.lse_part, self.batch * self.q_len, self.n_heads, self.num_splits,
                    self.o_lat, self.dtype, self.lse, stream)

    def project_out(self, w_uv, stream=None):
        mla_out_uv(self.o_lat, w_uv, self.out, self.batch * self.q_len, self.n_heads, self.dtype, stream)

    @property
    def fused_post(self):
        """bf16 steps whose (query row, head) pairs fit in one wave of CTAs, one
        per SM (each stages a head's 128 KB W_UV), merge the splits and apply
        W_UV in one launch (mla_combine_out_uv); larger ones use combine and the
        tensor-core GEMM (8 rows x 128 heads fused: a 33 us longer step)."""
        if self.dtype != MLA_BF16:
            return False
        sms = self.torch.cuda.get_device_properties(self.device).multi_processor_count
        return self.batch * self.q_len * self.n_heads <= sms

    def finish(self, w_uv, stream=None):
        """After the attention: o_lat, lse and out (combine, then out_uv)."""
        if self.fused_post:
            mla_combine_out_uv(self.o_part, self.lse_part, self.batch * self.q_len, self.n_heads, self.num_splits,
                               w_uv, self.o_lat, self.out, self.lse, stream)
        else:
            self.combine(stream)
            self.project_out(w_uv, stream)

    @property
    def launches_per_step(self):
        return (4 if self.fused_post else 5) + (1 if self.q8 else 0)

    # -- the projections on either side of the path ---------------------------
    def append_from_hidden(self, h, w_kva, seq_ids, positions, stream=None):
        """The new tokens' cache rows straight from hidden states h (bf16
        [n_new, d_model]): kv_a = h W_kv,a^T, then the rows of mla_cache_append,
        in one launch (mla_kv_proj_append).  w_kva: bf16 [576, d_model]."""
        n_new, d_model = int(h.shape[0]), int(h.shape[1])
        need = mla_kv_proj_workspace_bytes(n_new)
        ws = getattr(self, "_kv_ws", None)
        if ws is None or ws.numel() < need:
            ws = self._kv_ws = self.torch.empty((max(need, 1),), dtype=self.torch.uint8, device=self.device)
        mla_kv_proj_append(h, w_kva, n_new, d_model, ws, seq_ids, positions, self.block_table, self.batch,
                           self.max_pages, PAGE, self.norm_gain, self.eps, self.rope_cos, self.rope_sin,
                           self.max_pos, self.cache, self.cache_scale, self.cache_dtype, self.num_pages, self.err,
                           stream)

    def project_model(self, w_o, u=None, stream=None):
        """u = W_O [out_1; ...; out_H] for every query row (mla_out_proj on the
        step's `out`); w_o: bf16 [d_model, H*128]; returns u, fp32 [rows, d_model]."""
        rows, d_model = self.batch * self.q_len, int(w_o.shape[0])
        if u is None:
            u = self.torch.empty((rows, d_model), dtype=self.torch.float32, device=self.device)
        mla_out_proj(self.out, w_o, u, rows, self.n_heads, d_model, stream)
        return u

    # -- the whole step ----------------------------------------------------
    def run(self, kv_a_new, seq_ids, positions, q_nope, q_pe, w_uk, w_uv, stream=None):
        """Append the step's new rows, then attend; returns `out` [B*T, H, 128]."""
        self.append(kv_a_new, seq_ids, positions, stream)
        self.absorb(q_nope, q_pe, w_uk, stream)
        self.attend(stream)
        self.finish(w_uv, stream)
        return self.out


    # -- the step as CUDA graphs ------------------------------------------------
    def capture(self, kv_a_new, seq_ids, positions, q_nope, q_pe, w_uk, w_uv, host_in=(), host_out=None):
        """Record the step's calls as CUDA graphs on this device: `pre` (append
        and absorb, as parallel branches), `attend` (the split-KV decode), `post`
        (combine and out_uv, or their fused form) and `whole` (all of them in
        one graph).  A replay launches the same kernels with the same
        arguments; the graphs read the given tensors and write `out` in place,
        so the caller refreshes the inputs' contents before each replay.

        host_in: (device tensor, pinned host tensor) pairs copied host->device
        at the start of `pre`; host_out: a pinned host tensor that `post` ends
        by copying `out` into.  Returns a StepGraphs."""
        torch = self.torch

        def copies_in():
            for dst, src in host_in:
                dst.copy_(src, non_blocking=True)

        # append and absorb_q are independent: in the graph they are two
        # branches (append on a forked stream), joined before the attention
        fork = torch.cuda.Stream(device=self.device)

        def pre():
            copies_in()
            main = torch.cuda.current_stream(self.device)
            fork.wait_stream(main)
            with torch.cuda.stream(fork):
                self.append(kv_a_new, seq_ids, positions)
            self.absorb(q_nope, q_pe, w_uk)
            main.wait_stream(fork)

        def post():
            self.finish(w_uv)
            if host_out is not None:
                host_out.copy_(self.out, non_blocking=True)

        parts = (pre, self.attend, post)
        # eager passes first (module loading, kernel attributes), on a side stream
        side = torch.cuda.Stream(device=self.device)
        side.wait_stream(torch.cuda.current_stream(self.device))
        with torch.cuda.stream(side):
            for _ in range(2):
                for fn in parts:
                    fn()
        torch.cuda.current_stream(self.device).wait_stream(side)
        torch.cuda.synchronize(self.device)
        graphs = []
        for fn in parts + (lambda: [f() for f in parts],):
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g, capture_error_mode="thread_local"):
                fn()
            graphs.append(g)
        return StepGraphs(*graphs)


class StepGraphs:
    """The graphs of one captured step: `pre`, `attend` and `post` (for timing
    the attention between them) and `whole`, the same launches as one graph,
    which `replay()` runs on the current stream."""

    def __init__(self, pre, attend, post, whole):
        self.pre, self.attend, self.post, self.whole = pre, attend, post, whole

    def replay(self):
        self.whole.replay()
