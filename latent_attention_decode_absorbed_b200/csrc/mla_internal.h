// Internal declarations shared by the library's translation units.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <atomic>

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

// the two-term e4m3 form of bf16 absorbed queries (see mla_split_q_e4m3)
cudaError_t launch_split_q_e4m3(const void* q_abs, int rows, int n_heads, void* q8, float* q_scale, cudaStream_t st);
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
  const float* q_scale;   // q_dtype E4M3: the two-term query's scale per (row, head)
};
cudaError_t launch_decode_simt(const DecodeArgs& a, cudaStream_t st);
// tcgen05 path for 65..128 heads (heads split across a CTA pair): bf16 queries over
// a bf16 or e4m3 cache, or the two-term e4m3 query over an e4m3 cache (8-bit MMAs)
bool decode_pair_supported(const DecodeArgs& a);
cudaError_t launch_decode_pair(const DecodeArgs& a, cudaStream_t st);
// tcgen05 path: bf16 queries over a bf16 or e4m3 cache
bool decode_tc_supported(const DecodeArgs& a);
cudaError_t launch_decode_tc(const DecodeArgs& a, cudaStream_t st);

// split-K tcgen05 GEMMs of the projections around the attention core
cudaError_t launch_out_proj(const void* out_heads, const void* w_o, float* u, int rows, int n_heads, int d_model,
                            cudaStream_t st);
cudaError_t launch_kv_proj_append(const void* h, const void* w_kva, int d_model, float* workspace,
                                  const AppendArgs& a, cudaStream_t st);

// the non-absorbed comparison path: per-head keys and values decompressed
// from the latents, then standard attention per head
cudaError_t launch_decompress_kv(const void* cache, int num_pages, const void* w_uk, const void* w_uv, int n_heads,
                                 void* k_c, void* v_c, int32_t* err, cudaStream_t st);
struct NaiveArgs {
  const void* q_nope; const void* q_pe; const void* cache; const void* k_c; const void* v_c; int num_pages;
  const int32_t* block_table; int max_pages; const int32_t* seq_lens; int batch; int q_len; int n_heads;
  float softmax_scale; void* out; float* lse; int32_t* err;
};
cudaError_t launch_attend_naive(const NaiveArgs& a, cudaStream_t st);

// the merge and the value up-projection in one launch (bf16, few query rows)
cudaError_t launch_combine_out_uv(const float* o_part, const float* lse_part, int rows, int n_heads, int num_splits,
                                  const void* w_uv, void* o_lat, void* out, float* lse_out, cudaStream_t st);

// shard_major: parts laid out [num_parts, rows, n_heads, 512] (per-GPU results
// of a row-sharded sequence) instead of [rows, n_heads, num_parts, 512]
cudaError_t launch_combine(const float* o_part, const float* lse_part, int rows, int n_heads,
                           int num_parts, bool shard_major, void* o_lat, int o_dtype, float* lse_out,
                           cudaStream_t st);

// Launches `kernel` with programmatic dependent launch allowed: it may start
// (its set-up, up to griddep_wait()) while the previous kernel on the stream
// is still running.  Used for the kernels of the decode step, which all call
// griddep_wait() before touching global memory.
template <typename... KArgs, typename... Args>
cudaError_t launch_dependent(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st,
                             Args... args) {
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, static_cast<KArgs>(args)...);
}

// Bound (SM cycles, about 2 s at 2 GHz) of every barrier wait in the
// tensor-core decode kernels, and the test hook that withholds one query load
// (both set through mla_test_set_decode_wait, read at launch).
inline std::atomic<unsigned long long> g_wait_limit{4000000000ull};
inline std::atomic<int> g_withhold_q{0};

// cuTensorMapEncodeTiled through the runtime's driver entry point (no -lcuda).
typedef CUresult (*TensorMapEncodeFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                      const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                      CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);
inline TensorMapEncodeFn tensor_map_encoder() {
  static TensorMapEncodeFn fn = [] {
    void* f = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      return reinterpret_cast<TensorMapEncodeFn>(f);
    return static_cast<TensorMapEncodeFn>(nullptr);
  }();
  return fn;
}

// CTA pairs that fit on the current device at one pair per two SMs.
inline long long sm_pair_count() {
  int dev = 0, sms = 0;
  if (cudaGetDevice(&dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || sms < 2)
    return 1;
  return sms / 2;
}

}  // namespace mla
