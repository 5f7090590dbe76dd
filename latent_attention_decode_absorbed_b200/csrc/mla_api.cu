// C ABI of libmla.so: argument validation and kernel dispatch.
#include <math.h>
#include <stdarg.h>
#include <stdio.h>
#include <string.h>

#include "mla.h"
#include "mla_internal.h"

namespace mla {

static thread_local char g_msg[512] = "";

mla_status fail(mla_status s, const char* fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(g_msg, sizeof(g_msg), fmt, ap);
  va_end(ap);
  return s;
}

mla_status cuda_status(cudaError_t e, const char* what) {
  if (e == cudaSuccess) return MLA_OK;
  return fail(MLA_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
}

static bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

}  // namespace mla

using namespace mla;

#define MLA_REQUIRE(cond, code, ...) \
  do {                               \
    if (!(cond)) return fail(code, __VA_ARGS__); \
  } while (0)

extern "C" {

const char* mla_status_string(int status) {
  switch (status) {
    case MLA_OK: return "ok";
    case MLA_ERR_INVALID_ARG: return "invalid argument";
    case MLA_ERR_UNSUPPORTED: return "unsupported configuration";
    case MLA_ERR_CUDA: return "CUDA error";
    case MLA_ERR_BAD_INDEX: return "index out of range";
    case MLA_ERR_TIMEOUT: return "device wait timed out";
    default: return "unknown status";
  }
}

const char* mla_last_error_message(void) { return g_msg; }

int mla_version(void) { return 10000; }

size_t mla_decode_workspace_bytes(int batch, int q_len, int n_heads, int num_splits) {
  if (batch <= 0 || q_len <= 0 || n_heads <= 0 || num_splits <= 0) return 0;
  return (size_t)batch * q_len * n_heads * num_splits * (MLA_D_C + 1) * sizeof(float);
}

mla_status mla_rope_table(double theta, int max_pos, float* cos_out, float* sin_out) {
  MLA_REQUIRE(cos_out && sin_out, MLA_ERR_INVALID_ARG, "mla_rope_table: null output");
  MLA_REQUIRE(max_pos >= 1, MLA_ERR_INVALID_ARG, "mla_rope_table: max_pos must be >= 1");
  MLA_REQUIRE(theta > 1.0 && isfinite(theta), MLA_ERR_INVALID_ARG, "mla_rope_table: theta must be > 1");
  const int half = MLA_D_R / 2;
  for (int i = 0; i < half; ++i) {
    const double inv_freq = pow(theta, -2.0 * i / (double)MLA_D_R);
    for (int p = 0; p < max_pos; ++p) {
      const double ang = (double)p * inv_freq;
      cos_out[(size_t)p * half + i] = (float)cos(ang);
      sin_out[(size_t)p * half + i] = (float)sin(ang);
    }
  }
  return MLA_OK;
}

mla_status mla_cache_append(const void* kv_a, mla_dtype kv_dtype, int n_new, const int32_t* seq_ids,
                            const int32_t* positions, const int32_t* block_table, int batch,
                            int max_pages_per_seq, int page_size, const float* norm_gain, float eps,
                            const float* rope_cos, const float* rope_sin, int rope_max_pos, void* cache,
                            float* cache_scale, mla_dtype cache_dtype, int num_pages, int32_t* err_word,
                            cudaStream_t stream) {
  MLA_REQUIRE(n_new >= 0, MLA_ERR_INVALID_ARG, "mla_cache_append: n_new < 0");
  MLA_REQUIRE(kv_dtype == MLA_F32 || kv_dtype == MLA_BF16, MLA_ERR_UNSUPPORTED,
              "mla_cache_append: kv_dtype must be F32 or BF16");
  MLA_REQUIRE(cache_dtype == MLA_F32 || cache_dtype == MLA_BF16 || cache_dtype == MLA_E4M3,
              MLA_ERR_UNSUPPORTED, "mla_cache_append: bad cache_dtype");
  MLA_REQUIRE(page_size == MLA_PAGE, MLA_ERR_UNSUPPORTED, "mla_cache_append: page_size must be %d", MLA_PAGE);
  MLA_REQUIRE(batch >= 1 && max_pages_per_seq >= 1 && num_pages >= 1 && rope_max_pos >= 1,
              MLA_ERR_INVALID_ARG, "mla_cache_append: batch, max_pages_per_seq, num_pages, rope_max_pos must be >= 1");
  MLA_REQUIRE(eps >= 0.f && isfinite(eps), MLA_ERR_INVALID_ARG, "mla_cache_append: eps must be finite and >= 0");
  MLA_REQUIRE((long long)max_pages_per_seq * page_size < (1ll << 31), MLA_ERR_INVALID_ARG,
              "mla_cache_append: table capacity overflows int32 positions");
  if (n_new == 0) return MLA_OK;
  MLA_REQUIRE(kv_a && seq_ids && positions && block_table && rope_cos && rope_sin && cache,
              MLA_ERR_INVALID_ARG, "mla_cache_append: null pointer");
  MLA_REQUIRE(cache_dtype != MLA_E4M3 || cache_scale, MLA_ERR_INVALID_ARG,
              "mla_cache_append: E4M3 cache needs cache_scale");
  MLA_REQUIRE(aligned(kv_a, 16) && aligned(cache, 16) && aligned(norm_gain, 16), MLA_ERR_INVALID_ARG,
              "mla_cache_append: kv_a, cache and norm_gain must be 16-byte aligned");
  AppendArgs a{kv_a, kv_dtype, n_new, seq_ids, positions, block_table, batch, max_pages_per_seq,
               page_size, norm_gain, eps, rope_cos, rope_sin, rope_max_pos, cache, cache_scale,
               cache_dtype, num_pages, err_word};
  return cuda_status(launch_append(a, stream), "mla_cache_append launch");
}

static mla_status check_proj(const char* fn, const void* a, const void* b, const void* c, int rows,
                             int n_heads, mla_dtype dtype) {
  MLA_REQUIRE(rows >= 0, MLA_ERR_INVALID_ARG, "%s: rows < 0", fn);
  MLA_REQUIRE(n_heads >= 1 && n_heads <= MLA_MAX_HEADS, MLA_ERR_INVALID_ARG, "%s: n_heads must be in [1, %d]",
              fn, MLA_MAX_HEADS);
  MLA_REQUIRE(dtype == MLA_F32 || dtype == MLA_BF16, MLA_ERR_UNSUPPORTED, "%s: dtype must be F32 or BF16", fn);
  MLA_REQUIRE(rows <= 65535 * 8, MLA_ERR_UNSUPPORTED, "%s: rows above %d", fn, 65535 * 8);
  if (rows == 0) return MLA_OK;
  MLA_REQUIRE(a && b && c, MLA_ERR_INVALID_ARG, "%s: null pointer", fn);
  MLA_REQUIRE(aligned(a, 16) && aligned(b, 16) && aligned(c, 16), MLA_ERR_INVALID_ARG,
              "%s: pointers must be 16-byte aligned", fn);
  return MLA_OK;
}

mla_status mla_absorb_q(const void* q_nope, const void* q_pe, const void* w_uk, void* q_abs, int rows,
                        int n_heads, mla_dtype dtype, cudaStream_t stream) {
  mla_status s = check_proj("mla_absorb_q", q_nope, w_uk, q_abs, rows, n_heads, dtype);
  if (s != MLA_OK || rows == 0) return s;
  MLA_REQUIRE(q_pe, MLA_ERR_INVALID_ARG, "mla_absorb_q: null q_pe");
  return cuda_status(launch_absorb_q(q_nope, q_pe, w_uk, q_abs, rows, n_heads, dtype, stream),
                     "mla_absorb_q launch");
}

mla_status mla_out_uv(const void* o_lat, const void* w_uv, void* out, int rows, int n_heads, mla_dtype dtype,
                      cudaStream_t stream) {
  mla_status s = check_proj("mla_out_uv", o_lat, w_uv, out, rows, n_heads, dtype);
  if (s != MLA_OK || rows == 0) return s;
  return cuda_status(launch_out_uv(o_lat, w_uv, out, rows, n_heads, dtype, stream), "mla_out_uv launch");
}

mla_status mla_decode_fwd(const void* q_abs, mla_dtype q_dtype, const void* cache, const float* cache_scale,
                          mla_dtype cache_dtype, int num_pages, const int32_t* block_table,
                          int max_pages_per_seq, int page_size, const int32_t* seq_lens, int batch, int q_len,
                          int n_heads, int num_splits, int split_tokens, float softmax_scale, float* o_part,
                          float* lse_part, int32_t* err_word, cudaStream_t stream) {
  MLA_REQUIRE(page_size == MLA_PAGE, MLA_ERR_UNSUPPORTED, "mla_decode_fwd: page_size must be %d", MLA_PAGE);
  MLA_REQUIRE(batch >= 1 && q_len >= 1 && num_pages >= 1 && max_pages_per_seq >= 1, MLA_ERR_INVALID_ARG,
              "mla_decode_fwd: batch, q_len, num_pages, max_pages_per_seq must be >= 1");
  MLA_REQUIRE(n_heads >= 1 && n_heads <= MLA_MAX_HEADS, MLA_ERR_INVALID_ARG,
              "mla_decode_fwd: n_heads must be in [1, %d]", MLA_MAX_HEADS);
  MLA_REQUIRE(num_splits >= 1 && split_tokens >= page_size && split_tokens % page_size == 0,
              MLA_ERR_INVALID_ARG, "mla_decode_fwd: need num_splits >= 1 and split_tokens a positive multiple of page_size");
  MLA_REQUIRE((long long)num_splits * split_tokens >= (long long)max_pages_per_seq * page_size,
              MLA_ERR_INVALID_ARG, "mla_decode_fwd: num_splits * split_tokens must cover max_pages_per_seq * page_size");
  MLA_REQUIRE((long long)max_pages_per_seq * page_size < (1ll << 31), MLA_ERR_INVALID_ARG,
              "mla_decode_fwd: table capacity overflows int32 positions");
  MLA_REQUIRE(isfinite(softmax_scale) && softmax_scale > 0.f, MLA_ERR_INVALID_ARG,
              "mla_decode_fwd: softmax_scale must be finite and > 0");
  MLA_REQUIRE((q_dtype == MLA_F32 && cache_dtype == MLA_F32) ||
                  (q_dtype == MLA_BF16 && (cache_dtype == MLA_BF16 || cache_dtype == MLA_E4M3)),
              MLA_ERR_UNSUPPORTED, "mla_decode_fwd: supported (q, cache) dtypes are (F32, F32), (BF16, BF16), (BF16, E4M3)");
  MLA_REQUIRE(q_abs && cache && block_table && seq_lens && o_part && lse_part, MLA_ERR_INVALID_ARG,
              "mla_decode_fwd: null pointer");
  MLA_REQUIRE(cache_dtype != MLA_E4M3 || cache_scale, MLA_ERR_INVALID_ARG,
              "mla_decode_fwd: E4M3 cache needs cache_scale");
  MLA_REQUIRE(aligned(q_abs, 16) && aligned(cache, 128) && aligned(o_part, 16), MLA_ERR_INVALID_ARG,
              "mla_decode_fwd: q_abs and o_part must be 16-byte aligned, cache 128-byte aligned");
  MLA_REQUIRE((long long)batch * q_len <= 65535, MLA_ERR_UNSUPPORTED, "mla_decode_fwd: batch*q_len above 65535");
  DecodeArgs a{q_abs, q_dtype, cache, cache_scale, cache_dtype, num_pages, block_table, max_pages_per_seq,
               page_size, seq_lens, batch, q_len, n_heads, num_splits, split_tokens, softmax_scale,
               o_part, lse_part, err_word};
  if (decode_pair_supported(a))
    return cuda_status(launch_decode_pair(a, stream), "mla_decode_fwd launch (tcgen05, head-split pairs)");
  if (decode_tc_supported(a)) return cuda_status(launch_decode_tc(a, stream), "mla_decode_fwd launch (tcgen05)");
  return cuda_status(launch_decode_simt(a, stream), "mla_decode_fwd launch");
}

mla_status mla_split_q_e4m3(const void* q_abs, int rows, int n_heads, void* q8, float* q_scale,
                            cudaStream_t stream) {
  MLA_REQUIRE(rows >= 0, MLA_ERR_INVALID_ARG, "mla_split_q_e4m3: rows < 0");
  MLA_REQUIRE(n_heads >= 1 && n_heads <= MLA_MAX_HEADS, MLA_ERR_INVALID_ARG,
              "mla_split_q_e4m3: n_heads must be in [1, %d]", MLA_MAX_HEADS);
  MLA_REQUIRE((long long)rows * n_heads * 32 < (1ll << 31), MLA_ERR_UNSUPPORTED, "mla_split_q_e4m3: too many rows");
  if (rows == 0) return MLA_OK;
  MLA_REQUIRE(q_abs && q8 && q_scale, MLA_ERR_INVALID_ARG, "mla_split_q_e4m3: null pointer");
  MLA_REQUIRE(aligned(q_abs, 16) && aligned(q8, 16) && aligned(q_scale, 4), MLA_ERR_INVALID_ARG,
              "mla_split_q_e4m3: q_abs and q8 must be 16-byte aligned");
  return cuda_status(launch_split_q_e4m3(q_abs, rows, n_heads, q8, q_scale, stream), "mla_split_q_e4m3 launch");
}

mla_status mla_decode_fwd_q8(const void* q8, const float* q_scale, const void* cache, const float* cache_scale,
                             int num_pages, const int32_t* block_table, int max_pages_per_seq, int page_size,
                             const int32_t* seq_lens, int batch, int q_len, int n_heads, int num_splits,
                             int split_tokens, float softmax_scale, float* o_part, float* lse_part,
                             int32_t* err_word, cudaStream_t stream) {
  MLA_REQUIRE(page_size == MLA_PAGE, MLA_ERR_UNSUPPORTED, "mla_decode_fwd_q8: page_size must be %d", MLA_PAGE);
  MLA_REQUIRE(batch >= 1 && q_len >= 1 && num_pages >= 1 && max_pages_per_seq >= 1, MLA_ERR_INVALID_ARG,
              "mla_decode_fwd_q8: batch, q_len, num_pages, max_pages_per_seq must be >= 1");
  MLA_REQUIRE(n_heads > 64 && n_heads <= MLA_MAX_HEADS, MLA_ERR_UNSUPPORTED,
              "mla_decode_fwd_q8: n_heads must be in [65, %d]", MLA_MAX_HEADS);
  MLA_REQUIRE(num_splits >= 1 && split_tokens >= page_size && split_tokens % page_size == 0,
              MLA_ERR_INVALID_ARG, "mla_decode_fwd_q8: need num_splits >= 1 and split_tokens a positive multiple of page_size");
  MLA_REQUIRE((long long)num_splits * split_tokens >= (long long)max_pages_per_seq * page_size,
              MLA_ERR_INVALID_ARG, "mla_decode_fwd_q8: num_splits * split_tokens must cover max_pages_per_seq * page_size");
  MLA_REQUIRE((long long)max_pages_per_seq * page_size < (1ll << 31), MLA_ERR_INVALID_ARG,
              "mla_decode_fwd_q8: table capacity overflows int32 positions");
  MLA_REQUIRE(isfinite(softmax_scale) && softmax_scale > 0.f, MLA_ERR_INVALID_ARG,
              "mla_decode_fwd_q8: softmax_scale must be finite and > 0");
  MLA_REQUIRE(q8 && q_scale && cache && cache_scale && block_table && seq_lens && o_part && lse_part,
              MLA_ERR_INVALID_ARG, "mla_decode_fwd_q8: null pointer");
  MLA_REQUIRE(aligned(q8, 16) && aligned(cache, 128) && aligned(o_part, 16), MLA_ERR_INVALID_ARG,
              "mla_decode_fwd_q8: q8 and o_part must be 16-byte aligned, cache 128-byte aligned");
  MLA_REQUIRE((long long)batch * q_len <= 65535, MLA_ERR_UNSUPPORTED, "mla_decode_fwd_q8: batch*q_len above 65535");
  DecodeArgs a{q8, MLA_E4M3, cache, cache_scale, MLA_E4M3, num_pages, block_table, max_pages_per_seq,
               page_size, seq_lens, batch, q_len, n_heads, num_splits, split_tokens, softmax_scale,
               o_part, lse_part, err_word, q_scale};
  MLA_REQUIRE(decode_pair_supported(a), MLA_ERR_UNSUPPORTED, "mla_decode_fwd_q8: unsupported sizes");
  return cuda_status(launch_decode_pair(a, stream), "mla_decode_fwd_q8 launch (tcgen05 kind::f8f6f4, head-split pairs)");
}

mla_status mla_out_proj(const void* out, const void* w_o, float* u, int rows, int n_heads, int d_model,
                        cudaStream_t stream) {
  MLA_REQUIRE(rows >= 0, MLA_ERR_INVALID_ARG, "mla_out_proj: rows < 0");
  MLA_REQUIRE(n_heads >= 1 && n_heads <= MLA_MAX_HEADS, MLA_ERR_INVALID_ARG, "mla_out_proj: n_heads must be in [1, %d]",
              MLA_MAX_HEADS);
  MLA_REQUIRE(d_model >= 256 && d_model % 256 == 0 && d_model <= 65536, MLA_ERR_UNSUPPORTED,
              "mla_out_proj: d_model must be a multiple of 256 in [256, 65536]");
  MLA_REQUIRE(rows <= 65535 * 128, MLA_ERR_UNSUPPORTED, "mla_out_proj: rows above %d", 65535 * 128);
  if (rows == 0) return MLA_OK;
  MLA_REQUIRE(out && w_o && u, MLA_ERR_INVALID_ARG, "mla_out_proj: null pointer");
  MLA_REQUIRE(aligned(out, 16) && aligned(w_o, 16) && aligned(u, 16), MLA_ERR_INVALID_ARG,
              "mla_out_proj: pointers must be 16-byte aligned");
  return cuda_status(launch_out_proj(out, w_o, u, rows, n_heads, d_model, stream), "mla_out_proj launch");
}

mla_status mla_decompress_kv(const void* cache, mla_dtype cache_dtype, int num_pages, int page_size,
                             const void* w_uk, const void* w_uv, int n_heads, void* k_c, void* v_c, int32_t* err_word,
                             cudaStream_t stream) {
  MLA_REQUIRE(num_pages >= 0, MLA_ERR_INVALID_ARG, "mla_decompress_kv: num_pages < 0");
  MLA_REQUIRE(cache_dtype == MLA_BF16, MLA_ERR_UNSUPPORTED, "mla_decompress_kv: the cache must be bf16");
  MLA_REQUIRE(page_size == MLA_PAGE, MLA_ERR_UNSUPPORTED, "mla_decompress_kv: page_size must be %d", MLA_PAGE);
  MLA_REQUIRE(n_heads >= 1 && n_heads <= MLA_MAX_HEADS, MLA_ERR_INVALID_ARG,
              "mla_decompress_kv: n_heads must be in [1, %d]", MLA_MAX_HEADS);
  MLA_REQUIRE(num_pages <= 2 * 65535, MLA_ERR_UNSUPPORTED, "mla_decompress_kv: more than %d pages", 2 * 65535);
  if (num_pages == 0) return MLA_OK;
  MLA_REQUIRE(cache && w_uk && w_uv && k_c && v_c, MLA_ERR_INVALID_ARG, "mla_decompress_kv: null pointer");
  MLA_REQUIRE(aligned(cache, 128) && aligned(w_uk, 16) && aligned(w_uv, 16) && aligned(k_c, 16) && aligned(v_c, 16),
              MLA_ERR_INVALID_ARG, "mla_decompress_kv: misaligned pointer");
  return cuda_status(launch_decompress_kv(cache, num_pages, w_uk, w_uv, n_heads, k_c, v_c, err_word, stream),
                     "mla_decompress_kv launch");
}

mla_status mla_attend_naive(const void* q_nope, const void* q_pe, const void* cache, mla_dtype cache_dtype,
                            const void* k_c, const void* v_c, int num_pages, const int32_t* block_table,
                            int max_pages_per_seq, int page_size, const int32_t* seq_lens, int batch, int q_len,
                            int n_heads, float softmax_scale, void* out, float* lse, int32_t* err_word,
                            cudaStream_t stream) {
  MLA_REQUIRE(batch >= 0 && q_len >= 1 && num_pages >= 0 && max_pages_per_seq >= 1, MLA_ERR_INVALID_ARG,
              "mla_attend_naive: bad sizes");
  MLA_REQUIRE(cache_dtype == MLA_BF16, MLA_ERR_UNSUPPORTED, "mla_attend_naive: the cache must be bf16");
  MLA_REQUIRE(page_size == MLA_PAGE, MLA_ERR_UNSUPPORTED, "mla_attend_naive: page_size must be %d", MLA_PAGE);
  MLA_REQUIRE(n_heads >= 1 && n_heads <= MLA_MAX_HEADS, MLA_ERR_INVALID_ARG,
              "mla_attend_naive: n_heads must be in [1, %d]", MLA_MAX_HEADS);
  MLA_REQUIRE(softmax_scale > 0.f, MLA_ERR_INVALID_ARG, "mla_attend_naive: softmax_scale must be > 0");
  MLA_REQUIRE((long long)batch * q_len <= 0x7fffffff, MLA_ERR_UNSUPPORTED, "mla_attend_naive: too many rows");
  if (batch == 0) return MLA_OK;
  MLA_REQUIRE(q_nope && q_pe && cache && k_c && v_c && block_table && seq_lens && out, MLA_ERR_INVALID_ARG,
              "mla_attend_naive: null pointer");
  MLA_REQUIRE(aligned(q_nope, 16) && aligned(q_pe, 16) && aligned(cache, 128) && aligned(k_c, 16) &&
                  aligned(v_c, 16) && aligned(out, 16),
              MLA_ERR_INVALID_ARG, "mla_attend_naive: misaligned pointer");
  NaiveArgs a{q_nope, q_pe, cache, k_c, v_c, num_pages, block_table, max_pages_per_seq, seq_lens, batch, q_len,
              n_heads, softmax_scale, out, lse, err_word};
  return cuda_status(launch_attend_naive(a, stream), "mla_attend_naive launch");
}

size_t mla_kv_proj_workspace_bytes(int n_new) {
  if (n_new <= 0) return 0;
  return (size_t)n_new * MLA_D_ROW * sizeof(float) + (size_t)((n_new + 127) / 128) * sizeof(unsigned);
}

mla_status mla_kv_proj_append(const void* h, const void* w_kva, int n_new, int d_model, void* workspace,
                              const int32_t* seq_ids, const int32_t* positions, const int32_t* block_table,
                              int batch, int max_pages_per_seq, int page_size, const float* norm_gain, float eps,
                              const float* rope_cos, const float* rope_sin, int rope_max_pos, void* cache,
                              float* cache_scale, mla_dtype cache_dtype, int num_pages, int32_t* err_word,
                              cudaStream_t stream) {
  MLA_REQUIRE(n_new >= 0, MLA_ERR_INVALID_ARG, "mla_kv_proj_append: n_new < 0");
  MLA_REQUIRE(d_model >= 64 && d_model % 64 == 0 && d_model <= 65536, MLA_ERR_UNSUPPORTED,
              "mla_kv_proj_append: d_model must be a multiple of 64 in [64, 65536]");
  MLA_REQUIRE(cache_dtype == MLA_F32 || cache_dtype == MLA_BF16 || cache_dtype == MLA_E4M3, MLA_ERR_UNSUPPORTED,
              "mla_kv_proj_append: bad cache_dtype");
  MLA_REQUIRE(page_size == MLA_PAGE, MLA_ERR_UNSUPPORTED, "mla_kv_proj_append: page_size must be %d", MLA_PAGE);
  MLA_REQUIRE(batch >= 1 && max_pages_per_seq >= 1 && num_pages >= 1 && rope_max_pos >= 1, MLA_ERR_INVALID_ARG,
              "mla_kv_proj_append: batch, max_pages_per_seq, num_pages, rope_max_pos must be >= 1");
  MLA_REQUIRE(eps >= 0.f && isfinite(eps), MLA_ERR_INVALID_ARG, "mla_kv_proj_append: eps must be finite and >= 0");
  MLA_REQUIRE((long long)max_pages_per_seq * page_size < (1ll << 31), MLA_ERR_INVALID_ARG,
              "mla_kv_proj_append: table capacity overflows int32 positions");
  MLA_REQUIRE(n_new <= 65535 * 128, MLA_ERR_UNSUPPORTED, "mla_kv_proj_append: n_new above %d", 65535 * 128);
  if (n_new == 0) return MLA_OK;
  MLA_REQUIRE(h && w_kva && workspace && seq_ids && positions && block_table && rope_cos && rope_sin && cache,
              MLA_ERR_INVALID_ARG, "mla_kv_proj_append: null pointer");
  MLA_REQUIRE(cache_dtype != MLA_E4M3 || cache_scale, MLA_ERR_INVALID_ARG,
              "mla_kv_proj_append: E4M3 cache needs cache_scale");
  MLA_REQUIRE(aligned(h, 16) && aligned(w_kva, 16) && aligned(workspace, 16) && aligned(cache, 16) &&
                  aligned(norm_gain, 16),
              MLA_ERR_INVALID_ARG, "mla_kv_proj_append: h, w_kva, workspace, cache and norm_gain must be 16-byte aligned");
  AppendArgs a{nullptr, MLA_F32, n_new, seq_ids, positions, block_table, batch, max_pages_per_seq, page_size,
               norm_gain, eps, rope_cos, rope_sin, rope_max_pos, cache, cache_scale, cache_dtype, num_pages, err_word};
  return cuda_status(launch_kv_proj_append(h, w_kva, d_model, static_cast<float*>(workspace), a, stream),
                     "mla_kv_proj_append launch");
}

mla_status mla_combine(const float* o_part, const float* lse_part, int rows, int n_heads, int num_splits,
                       void* o_lat, mla_dtype o_dtype, float* lse_out, cudaStream_t stream) {
  MLA_REQUIRE(rows >= 0 && n_heads >= 1 && n_heads <= MLA_MAX_HEADS && num_splits >= 1, MLA_ERR_INVALID_ARG,
              "mla_combine: need rows >= 0, n_heads in [1, %d], num_splits >= 1", MLA_MAX_HEADS);
  MLA_REQUIRE(o_dtype == MLA_F32 || o_dtype == MLA_BF16, MLA_ERR_UNSUPPORTED, "mla_combine: o_dtype must be F32 or BF16");
  MLA_REQUIRE(num_splits <= 8192, MLA_ERR_UNSUPPORTED, "mla_combine: num_splits above 8192");
  if (rows == 0) return MLA_OK;
  MLA_REQUIRE(o_part && lse_part && o_lat, MLA_ERR_INVALID_ARG, "mla_combine: null pointer");
  MLA_REQUIRE(aligned(o_part, 16) && aligned(o_lat, 16), MLA_ERR_INVALID_ARG,
              "mla_combine: o_part and o_lat must be 16-byte aligned");
  return cuda_status(launch_combine(o_part, lse_part, rows, n_heads, num_splits, false, o_lat, o_dtype, lse_out,
                                    stream),
                     "mla_combine launch");
}

mla_status mla_combine_out_uv(const float* o_part, const float* lse_part, int rows, int n_heads, int num_splits,
                              const void* w_uv, void* o_lat, void* out, float* lse_out, cudaStream_t stream) {
  MLA_REQUIRE(rows >= 0 && n_heads >= 1 && n_heads <= MLA_MAX_HEADS && num_splits >= 1, MLA_ERR_INVALID_ARG,
              "mla_combine_out_uv: need rows >= 0, n_heads in [1, %d], num_splits >= 1", MLA_MAX_HEADS);
  MLA_REQUIRE(num_splits <= 8192, MLA_ERR_UNSUPPORTED, "mla_combine_out_uv: num_splits above 8192");
  if (rows == 0) return MLA_OK;
  MLA_REQUIRE(o_part && lse_part && w_uv && out, MLA_ERR_INVALID_ARG, "mla_combine_out_uv: null pointer");
  MLA_REQUIRE(aligned(o_part, 16) && aligned(w_uv, 16) && aligned(out, 16) && (!o_lat || aligned(o_lat, 16)),
              MLA_ERR_INVALID_ARG, "mla_combine_out_uv: pointers must be 16-byte aligned");
  return cuda_status(launch_combine_out_uv(o_part, lse_part, rows, n_heads, num_splits, w_uv, o_lat, out, lse_out,
                                           stream),
                     "mla_combine_out_uv launch");
}

mla_status mla_combine_shards(const float* o_shard, const float* lse_shard, int num_shards, int rows,
                              int n_heads, void* o_lat, mla_dtype o_dtype, float* lse_out, cudaStream_t stream) {
  MLA_REQUIRE(rows >= 0 && n_heads >= 1 && n_heads <= MLA_MAX_HEADS && num_shards >= 1, MLA_ERR_INVALID_ARG,
              "mla_combine_shards: need rows >= 0, n_heads in [1, %d], num_shards >= 1", MLA_MAX_HEADS);
  MLA_REQUIRE(o_dtype == MLA_F32 || o_dtype == MLA_BF16, MLA_ERR_UNSUPPORTED,
              "mla_combine_shards: o_dtype must be F32 or BF16");
  MLA_REQUIRE(num_shards <= 8192, MLA_ERR_UNSUPPORTED, "mla_combine_shards: num_shards above 8192");
  if (rows == 0) return MLA_OK;
  MLA_REQUIRE(o_shard && lse_shard && o_lat, MLA_ERR_INVALID_ARG, "mla_combine_shards: null pointer");
  MLA_REQUIRE(aligned(o_shard, 16) && aligned(o_lat, 16), MLA_ERR_INVALID_ARG,
              "mla_combine_shards: o_shard and o_lat must be 16-byte aligned");
  return cuda_status(launch_combine(o_shard, lse_shard, rows, n_heads, num_shards, true, o_lat, o_dtype, lse_out,
                                    stream),
                     "mla_combine_shards launch");
}

}  // extern "C"
