"""Python binding of libmla.so, the sm_100a absorbed-MLA decode library.

Argument marshalling only: every function forwards to the C entry point of
the same name in ``include/mla.h`` and raises ``MlaError`` on a non-OK
status.  Tensor arguments are torch tensors (their device pointers are
passed); PyTorch supplies device memory and streams, nothing else.  There is
no CPU fallback: if the shared library is missing, every call raises.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libmla.so")

MLA_OK, MLA_ERR_INVALID_ARG, MLA_ERR_UNSUPPORTED, MLA_ERR_CUDA, MLA_ERR_BAD_INDEX, MLA_ERR_TIMEOUT = range(6)
MLA_F32, MLA_BF16, MLA_E4M3 = 0, 1, 2
MLA_DEVERR_PAGE, MLA_DEVERR_POSITION, MLA_DEVERR_TIMEOUT = 0x1, 0x2, 0x4
D_C, D_R, D_ROW, D_NOPE, D_V, PAGE = 512, 64, 576, 128, 128, 64

# entry points with their ctypes signatures (p = pointer, i = int, f = float, d = double)
_SIGS = {
    "mla_status_string": ("s", "i"),
    "mla_last_error_message": ("s", ""),
    "mla_version": ("i", ""),
    "mla_rope_table": ("i", "dipp"),
    "mla_decode_workspace_bytes": ("z", "iiii"),
    "mla_cache_append": ("i", "piipppiiipfppippiipp"),
    "mla_absorb_q": ("i", "ppppiiip"),
    "mla_decode_fwd": ("i", "pippiipiipiiiiifpppp"),
    "mla_split_q_e4m3": ("i", "piippp"),
    "mla_decode_fwd_q8": ("i", "ppppipiipiiiiifpppp"),
    "mla_combine": ("i", "ppiiipipp"),
    "mla_combine_shards": ("i", "ppiiipipp"),
    "mla_out_uv": ("i", "pppiiip"),
    "mla_decode_static": ("i", "pippiipiipiiiiifpippp"),
    "mla_test_set_decode_wait": ("i", "Qi"),
    "mla_out_proj": ("i", "pppiiip"),
    "mla_kv_proj_workspace_bytes": ("z", "i"),
    "mla_kv_proj_append": ("i", "ppiippppiiipfppippiipp"),
    "mla_decompress_kv": ("i", "piiippipppp"),
    "mla_combine_out_uv": ("i", "ppiiippppp"),
    "mla_attend_naive": ("i", "pppippipiipiiifpppp"),
}
_CT = {"p": ctypes.c_void_p, "i": ctypes.c_int, "f": ctypes.c_float, "d": ctypes.c_double,
       "s": ctypes.c_char_p, "z": ctypes.c_size_t, "Q": ctypes.c_ulonglong}

_lib = None


class MlaError(RuntimeError):
    def __init__(self, fn, status, msg):
        super().__init__(f"{fn}: status {status} ({status_string(status)}): {msg}")
        self.status = status


def lib():
    """Load libmla.so (once).  Raises if it has not been built."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"libmla.so not built at {LIB_PATH}; run "
                               "`python -m latent_attention_decode_absorbed_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in _SIGS.items():
            f = getattr(L, name)
            f.restype = _CT[res]
            f.argtypes = [_CT[c] for c in args]
        _lib = L
    return _lib


def status_string(status: int) -> str:
    return lib().mla_status_string(int(status)).decode()


def _ptr(x) -> Optional[int]:
    if x is None:
        return None
    if isinstance(x, int):
        return x
    return x.data_ptr()


def _stream(stream) -> Optional[int]:
    if stream is None:
        import torch
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


def _check(fn, status):
    if status != MLA_OK:
        raise MlaError(fn, status, lib().mla_last_error_message().decode())


def dtype_code(t) -> int:
    import torch
    return {torch.float32: MLA_F32, torch.bfloat16: MLA_BF16, torch.uint8: MLA_E4M3,
            torch.float8_e4m3fn: MLA_E4M3}[t.dtype]


def pack_cache_rows(rows):
    """Logical cache rows [num_pages*64, 576] -> the page-blocked pool layout
    [num_pages, 9, 64, 64] (nine [64 rows x 64 columns] blocks per page).
    A pure layout transform (torch tensors, any dtype)."""
    n = rows.shape[0] // PAGE
    return rows.reshape(n, PAGE, D_ROW // 64, 64).permute(0, 2, 1, 3).contiguous()


def unpack_cache_rows(cache):
    """Page-blocked pool [num_pages, 9, 64, 64] -> logical rows [num_pages*64, 576]."""
    n = cache.shape[0]
    return cache.reshape(n, D_ROW // 64, PAGE, 64).permute(0, 2, 1, 3).reshape(n * PAGE, D_ROW)


def mla_version() -> int:
    return lib().mla_version()


def mla_decode_workspace_bytes(batch: int, q_len: int, n_heads: int, num_splits: int) -> int:
    """Bytes of the fp32 split partials (o_part + lse_part) mla_decode_fwd writes."""
    return int(lib().mla_decode_workspace_bytes(int(batch), int(q_len), int(n_heads), int(num_splits)))


def mla_rope_table(theta: float, max_pos: int, cos_out, sin_out):
    """Host tables [max_pos, 32] float32 (numpy arrays or CPU tensors)."""
    cp = cos_out.ctypes.data if hasattr(cos_out, "ctypes") else cos_out.data_ptr()
    sp = sin_out.ctypes.data if hasattr(sin_out, "ctypes") else sin_out.data_ptr()
    _check("mla_rope_table", lib().mla_rope_table(float(theta), int(max_pos), cp, sp))


def mla_cache_append(kv_a, kv_dtype, n_new, seq_ids, positions, block_table, batch, max_pages_per_seq,
                     page_size, norm_gain, eps, rope_cos, rope_sin, rope_max_pos, cache, cache_scale,
                     cache_dtype, num_pages, err_word=None, stream=None):
    _check("mla_cache_append", lib().mla_cache_append(
        _ptr(kv_a), int(kv_dtype), int(n_new), _ptr(seq_ids), _ptr(positions), _ptr(block_table),
        int(batch), int(max_pages_per_seq), int(page_size), _ptr(norm_gain), float(eps), _ptr(rope_cos),
        _ptr(rope_sin), int(rope_max_pos), _ptr(cache), _ptr(cache_scale), int(cache_dtype),
        int(num_pages), _ptr(err_word), _stream(stream)))


def mla_absorb_q(q_nope, q_pe, w_uk, q_abs, rows, n_heads, dtype, stream=None):
    _check("mla_absorb_q", lib().mla_absorb_q(_ptr(q_nope), _ptr(q_pe), _ptr(w_uk), _ptr(q_abs),
                                              int(rows), int(n_heads), int(dtype), _stream(stream)))


def mla_decode_fwd(q_abs, q_dtype, cache, cache_scale, cache_dtype, num_pages, block_table,
                   max_pages_per_seq, page_size, seq_lens, batch, q_len, n_heads, num_splits,
                   split_tokens, softmax_scale, o_part, lse_part, err_word=None, stream=None):
    _check("mla_decode_fwd", lib().mla_decode_fwd(
        _ptr(q_abs), int(q_dtype), _ptr(cache), _ptr(cache_scale), int(cache_dtype), int(num_pages),
        _ptr(block_table), int(max_pages_per_seq), int(page_size), _ptr(seq_lens), int(batch),
        int(q_len), int(n_heads), int(num_splits), int(split_tokens), float(softmax_scale),
        _ptr(o_part), _ptr(lse_part), _ptr(err_word), _stream(stream)))


def mla_split_q_e4m3(q_abs, rows, n_heads, q8, q_scale, stream=None):
    """bf16 q_abs [rows, H, 576] -> two-term e4m3 q8 [rows, 2, H, 576] (uint8) and q_scale [rows, H]."""
    _check("mla_split_q_e4m3", lib().mla_split_q_e4m3(_ptr(q_abs), int(rows), int(n_heads), _ptr(q8), _ptr(q_scale),
                                                      _stream(stream)))


def mla_decode_fwd_q8(q8, q_scale, cache, cache_scale, num_pages, block_table, max_pages_per_seq, page_size,
                      seq_lens, batch, q_len, n_heads, num_splits, split_tokens, softmax_scale, o_part, lse_part,
                      err_word=None, stream=None):
    """mla_decode_fwd over an e4m3 cache on 8-bit MMAs, from mla_split_q_e4m3's query form."""
    _check("mla_decode_fwd_q8", lib().mla_decode_fwd_q8(
        _ptr(q8), _ptr(q_scale), _ptr(cache), _ptr(cache_scale), int(num_pages), _ptr(block_table),
        int(max_pages_per_seq), int(page_size), _ptr(seq_lens), int(batch), int(q_len), int(n_heads),
        int(num_splits), int(split_tokens), float(softmax_scale), _ptr(o_part), _ptr(lse_part), _ptr(err_word),
        _stream(stream)))


def mla_combine(o_part, lse_part, rows, n_heads, num_splits, o_lat, o_dtype, lse_out=None, stream=None):
    _check("mla_combine", lib().mla_combine(_ptr(o_part), _ptr(lse_part), int(rows), int(n_heads),
                                            int(num_splits), _ptr(o_lat), int(o_dtype), _ptr(lse_out),
                                            _stream(stream)))


def mla_combine_shards(o_shard, lse_shard, num_shards, rows, n_heads, o_lat, o_dtype, lse_out=None,
                       stream=None):
    _check("mla_combine_shards", lib().mla_combine_shards(_ptr(o_shard), _ptr(lse_shard), int(num_shards),
                                                          int(rows), int(n_heads), _ptr(o_lat), int(o_dtype),
                                                          _ptr(lse_out), _stream(stream)))


def mla_out_uv(o_lat, w_uv, out, rows, n_heads, dtype, stream=None):
    _check("mla_out_uv", lib().mla_out_uv(_ptr(o_lat), _ptr(w_uv), _ptr(out), int(rows), int(n_heads),
                                          int(dtype), _stream(stream)))


def mla_decode_static(q_abs, q_dtype, cache, cache_scale, cache_dtype, num_pages, block_table,
                      max_pages_per_seq, page_size, seq_lens, batch, q_len, n_heads, num_splits,
                      split_tokens, softmax_scale, o_lat, o_dtype, lse_out=None, err_word=None, stream=None):
    """Attention + combine without caller workspace (library-held scratch);
    see the header for its size limit and sharing rules."""
    _check("mla_decode_static", lib().mla_decode_static(
        _ptr(q_abs), int(q_dtype), _ptr(cache), _ptr(cache_scale), int(cache_dtype), int(num_pages),
        _ptr(block_table), int(max_pages_per_seq), int(page_size), _ptr(seq_lens), int(batch),
        int(q_len), int(n_heads), int(num_splits), int(split_tokens), float(softmax_scale),
        _ptr(o_lat), int(o_dtype), _ptr(lse_out), _ptr(err_word), _stream(stream)))


MLA_STATIC_MAX_PARTIALS = 8192


def mla_out_proj(out, w_o, u, rows, n_heads, d_model, stream=None):
    """u[r] = W_O [out[r, 0]; ...; out[r, H-1]] (fp32 u, overwritten)."""
    _check("mla_out_proj", lib().mla_out_proj(_ptr(out), _ptr(w_o), _ptr(u), int(rows), int(n_heads), int(d_model),
                                              _stream(stream)))


def mla_combine_out_uv(o_part, lse_part, rows, n_heads, num_splits, w_uv, o_lat, out, lse_out=None, stream=None):
    """mla_combine then mla_out_uv in one launch (bf16, few rows); o_lat may be None."""
    _check("mla_combine_out_uv", lib().mla_combine_out_uv(_ptr(o_part), _ptr(lse_part), int(rows), int(n_heads),
                                                          int(num_splits), _ptr(w_uv), _ptr(o_lat), _ptr(out),
                                                          _ptr(lse_out), _stream(stream)))


def mla_decompress_kv(cache, cache_dtype, num_pages, page_size, w_uk, w_uv, n_heads, k_c, v_c, err_word=None,
                      stream=None):
    """Per-head keys and values of every cached row (the non-absorbed path's
    decompression): k_c, v_c bf16 [num_pages, 64, n_heads, 128]."""
    _check("mla_decompress_kv", lib().mla_decompress_kv(_ptr(cache), int(cache_dtype), int(num_pages), int(page_size),
                                                        _ptr(w_uk), _ptr(w_uv), int(n_heads), _ptr(k_c), _ptr(v_c),
                                                        _ptr(err_word), _stream(stream)))


def mla_attend_naive(q_nope, q_pe, cache, cache_dtype, k_c, v_c, num_pages, block_table, max_pages_per_seq,
                     page_size, seq_lens, batch, q_len, n_heads, softmax_scale, out, lse=None, err_word=None,
                     stream=None):
    """Standard attention per head over decompressed keys and values: out bf16
    [batch*q_len, n_heads, 128], lse fp32 [batch*q_len, n_heads] (optional)."""
    _check("mla_attend_naive", lib().mla_attend_naive(
        _ptr(q_nope), _ptr(q_pe), _ptr(cache), int(cache_dtype), _ptr(k_c), _ptr(v_c), int(num_pages),
        _ptr(block_table), int(max_pages_per_seq), int(page_size), _ptr(seq_lens), int(batch), int(q_len),
        int(n_heads), float(softmax_scale), _ptr(out), _ptr(lse), _ptr(err_word), _stream(stream)))


def mla_kv_proj_workspace_bytes(n_new) -> int:
    return int(lib().mla_kv_proj_workspace_bytes(int(n_new)))


def mla_kv_proj_append(h, w_kva, n_new, d_model, workspace, seq_ids, positions, block_table, batch,
                       max_pages_per_seq, page_size, norm_gain, eps, rope_cos, rope_sin, rope_max_pos, cache,
                       cache_scale, cache_dtype, num_pages, err_word=None, stream=None):
    """kv_a = W_kv,a h, then mla_cache_append's row writer, in one kernel."""
    _check("mla_kv_proj_append", lib().mla_kv_proj_append(
        _ptr(h), _ptr(w_kva), int(n_new), int(d_model), _ptr(workspace), _ptr(seq_ids), _ptr(positions),
        _ptr(block_table), int(batch), int(max_pages_per_seq), int(page_size), _ptr(norm_gain), float(eps),
        _ptr(rope_cos), _ptr(rope_sin), int(rope_max_pos), _ptr(cache), _ptr(cache_scale), int(cache_dtype),
        int(num_pages), _ptr(err_word), _stream(stream)))


def mla_test_set_decode_wait(limit_cycles=0, withhold_q_load=False):
    """Test hook (include/mla_test.h): bound of the decode kernel's barrier
    waits in SM cycles (0 = the default) and whether the first query load of
    every CTA pair is left out so that a wait runs out."""
    _check("mla_test_set_decode_wait", lib().mla_test_set_decode_wait(int(limit_cycles), int(bool(withhold_q_load))))

from .step import DecodeStep  # noqa: E402,F401
