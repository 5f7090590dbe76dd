// mla_decode_static: attention + combine with library-held scratch.
//
// For callers that cannot allocate device memory themselves.  The split
// partials live in a file-scope device array of fixed size; host code never
// uses the array's name as a device address but looks the address up once
// per device (and again if that device's context was replaced, e.g. after
// cudaDeviceReset) with cudaGetSymbolAddress, with that device current.
#include <cuda.h>

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
// The looked-up address is only valid in the context it was looked up in:
// after cudaDeviceReset the device gets a new primary context and the array a
// new address.  Each entry therefore remembers the context's unique id.
struct ScratchEntry {
  unsigned long long ctx_id;
  float* addr;
};
ScratchEntry g_addr[kMaxDevices] = {};

typedef CUresult (*CtxGetCurrentFn)(CUcontext*);
typedef CUresult (*CtxGetIdFn)(CUcontext, unsigned long long*);

// Unique id of the calling thread's current context (0 if it cannot be read).
unsigned long long current_ctx_id() {
  static CtxGetCurrentFn get_cur = nullptr;
  static CtxGetIdFn get_id = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* f = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &f, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_cur = reinterpret_cast<CtxGetCurrentFn>(f);
    f = nullptr;
    if (cudaGetDriverEntryPoint("cuCtxGetId", &f, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_id = reinterpret_cast<CtxGetIdFn>(f);
  });
  CUcontext ctx = nullptr;
  unsigned long long id = 0;
  if (get_cur && get_id && get_cur(&ctx) == CUDA_SUCCESS && ctx && get_id(ctx, &id) == CUDA_SUCCESS) return id;
  return 0;
}

// Device address of g_partials on the current device: looked up once per
// device and context (cudaGetSymbolAddress allocates nothing).
mla_status scratch_address(float** out) {
  int dev = -1;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_status(e, "mla_decode_static: cudaGetDevice");
  if (dev < 0 || dev >= kMaxDevices)
    return fail(MLA_ERR_UNSUPPORTED, "mla_decode_static: device ordinal %d above %d", dev, kMaxDevices - 1);
  std::lock_guard<std::mutex> lock(g_mu);
  unsigned long long id = current_ctx_id();   // 0 while no context is current yet
  if (id == 0 || g_addr[dev].addr == nullptr || g_addr[dev].ctx_id != id) {
    // set-up for this device and context (binds the context if none is current)
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_partials);
    if (e != cudaSuccess) return cuda_status(e, "mla_decode_static: cudaGetSymbolAddress");
    g_addr[dev].addr = static_cast<float*>(p);
    g_addr[dev].ctx_id = current_ctx_id();
  }
  *out = g_addr[dev].addr;
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
