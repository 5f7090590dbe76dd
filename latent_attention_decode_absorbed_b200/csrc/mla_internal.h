// Internal declarations shared by the library's translation units.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include "mla.h"

namespace mla {

// Records a message for mla_last_error_message() on this thread and returns s.
mla_status fail(mla_status s, const char* fmt, ...);
// Turns a CUDA error from a launch into MLA_ERR_CUDA with its text.
mla_status cuda_status(cudaError_t e, const char* what);

struct AppendArgs {
  const void* kv_a; int kv_dtype; int n_new;
  const int32_t* seq_ids; const int32_t* positions;
  const int32_t* block_table; int batch; int max_pages; int page_size;
  const float* gain; float eps;
  const float* rope_cos; const float* rope_sin; int rope_max_pos;
  void* cache; float* cache_scale; int cache_dtype; int num_pages;
  int32_t* err;
};
cudaError_t launch_append(const AppendArgs& a, cudaStream_t st);

cudaError_t launch_absorb_q(const void* q_nope, const void* q_pe, const void* w_uk, void* q_abs,
                            int rows, int n_heads, int dtype, cudaStream_t st);
cudaError_t launch_out_uv(const void* o_lat, const void* w_uv, void* out, int rows, int n_heads,
                          int dtype, cudaStream_t st);
// tensor-core versions (bf16): one tcgen05 GEMM per head
cudaError_t launch_absorb_q_tc(const void* q_nope, const void* q_pe, const void* w_uk, void* q_abs, int rows,
                               int n_heads, cudaStream_t st);
cudaError_t launch_out_uv_tc(const void* o_lat, const void* w_uv, void* out, int rows, int n_heads, cudaStream_t st);

struct DecodeArgs {
  const void* q_abs; int q_dtype;
  const void* cache; const float* cache_scale; int cache_dtype; int num_pages;
  const int32_t* block_table; int max_pages; int page_size;
  const int32_t* seq_lens; int batch; int q_len; int n_heads;
  int num_splits; int split_tokens; float softmax_scale;
  float* o_part; float* lse_part; int32_t* err;
};
cudaError_t launch_decode_simt(const DecodeArgs& a, cudaStream_t st);
// tcgen05 path: bf16 queries over a bf16 or e4m3 cache
bool decode_tc_supported(const DecodeArgs& a);
cudaError_t launch_decode_tc(const DecodeArgs& a, cudaStream_t st);

// shard_major: parts laid out [num_parts, rows, n_heads, 512] (per-GPU results
// of a row-sharded sequence) instead of [rows, n_heads, num_parts, 512]
cudaError_t launch_combine(const float* o_part, const float* lse_part, int rows, int n_heads,
                           int num_parts, bool shard_major, void* o_lat, int o_dtype, float* lse_out,
                           cudaStream_t st);

}  // namespace mla
