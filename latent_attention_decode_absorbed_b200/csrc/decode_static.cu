// mla_decode_static: attention + combine with library-held scratch.
//
// For callers that cannot allocate device memory themselves.  The split
// partials live in a file-scope device array of fixed size; host code never
// uses the array's name as a device address but looks the address up once
// per device with cudaGetSymbolAddress, with that device current.
#include <mutex>

#include "mla.h"
#include "mla_internal.h"

namespace mla {
namespace {

constexpr size_t kPartials = MLA_STATIC_MAX_PARTIALS;
// o_part [kPartials, 512] followed by lse_part [kPartials]
static __device__ __align__(256) float g_partials[kPartials * MLA_D_C + kPartials];

constexpr int kMaxDevices = 64;
std::mutex g_mu;
float* g_addr[kMaxDevices] = {};

// Device address of g_partials on the current device (looked up on first use).
mla_status scratch_address(float** out) {
  int dev = -1;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_status(e, "mla_decode_static: cudaGetDevice");
  if (dev < 0 || dev >= kMaxDevices)
    return fail(MLA_ERR_UNSUPPORTED, "mla_decode_static: device ordinal %d above %d", dev, kMaxDevices - 1);
  std::lock_guard<std::mutex> lock(g_mu);
  if (g_addr[dev] == nullptr) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_partials);
    if (e != cudaSuccess) return cuda_status(e, "mla_decode_static: cudaGetSymbolAddress");
    g_addr[dev] = static_cast<float*>(p);
  }
  *out = g_addr[dev];
  return MLA_OK;
}

}  // namespace
}  // namespace mla

using namespace mla;

extern "C" mla_status mla_decode_static(const void* q_abs, mla_dtype q_dtype, const void* cache,
                                        const float* cache_scale, mla_dtype cache_dtype, int num_pages,
                                        const int32_t* block_table, int max_pages_per_seq, int page_size,
                                        const int32_t* seq_lens, int batch, int q_len, int n_heads,
                                        int num_splits, int split_tokens, float softmax_scale, void* o_lat,
                                        mla_dtype o_dtype, float* lse_out, int32_t* err_word,
                                        cudaStream_t stream) {
  if (batch < 1 || q_len < 1 || n_heads < 1 || num_splits < 1)
    return fail(MLA_ERR_INVALID_ARG, "mla_decode_static: batch, q_len, n_heads, num_splits must be >= 1");
  const unsigned long long partials =
      (unsigned long long)batch * q_len * n_heads * (unsigned long long)num_splits;
  if (partials > kPartials)
    return fail(MLA_ERR_INVALID_ARG,
                "mla_decode_static: batch*q_len*n_heads*num_splits = %llu exceeds the static scratch "
                "capacity of %d partial rows (%.1f MB); use mla_decode_fwd + mla_combine with a "
                "caller-provided workspace",
                partials, MLA_STATIC_MAX_PARTIALS, sizeof(float) * (double)kPartials * (MLA_D_C + 1) / 1e6);
  if (o_lat == nullptr) return fail(MLA_ERR_INVALID_ARG, "mla_decode_static: null o_lat");
  if (o_dtype != MLA_F32 && o_dtype != MLA_BF16)
    return fail(MLA_ERR_UNSUPPORTED, "mla_decode_static: o_dtype must be F32 or BF16");
  float* scratch = nullptr;
  mla_status s = scratch_address(&scratch);
  if (s != MLA_OK) return s;
  float* o_part = scratch;
  float* lse_part = scratch + kPartials * MLA_D_C;
  s = mla_decode_fwd(q_abs, q_dtype, cache, cache_scale, cache_dtype, num_pages, block_table, max_pages_per_seq,
                     page_size, seq_lens, batch, q_len, n_heads, num_splits, split_tokens, softmax_scale, o_part,
                     lse_part, err_word, stream);
  if (s != MLA_OK) return s;
  return mla_combine(o_part, lse_part, batch * q_len, n_heads, num_splits, o_lat, o_dtype, lse_out, stream);
}
