// Per-head projections on either side of latent attention.
//
//   absorb_q:  q_abs[r,h,0:512] = W_UK[h]^T q_nope[r,h]  and q_abs[r,h,512:] = q_pe[r,h]
//   out_uv:    out[r,h,:]       = W_UV[h]   o_lat[r,h]
//
// "DeepSeek-V2: MLA Explained", "Optimization Note": W_UK merges into the
// query and W_UV is applied after the softmax sum.  Each is a batched per-head
// product with a short row count (B*T) against a 128x512 weight per head: the
// weight read (16.8 MB bf16 at 128 heads) dominates, so a CTA streams one
// head's weight once for up to kRB rows held in shared memory.
#include "mla_device.cuh"
#include "mla_internal.h"

namespace mla {
namespace {

constexpr int kRB = 8;  // query rows per CTA

template <typename T>
__global__ void __launch_bounds__(256) absorb_q_kernel(const T* __restrict__ q_nope, const T* __restrict__ q_pe,
                                                       const T* __restrict__ w_uk, T* __restrict__ q_abs,
                                                       int rows, int H) {
  const int h = blockIdx.x;
  const int r0 = blockIdx.y * kRB;
  const int nr = min(kRB, rows - r0);
  __shared__ float qs[kRB][MLA_D_NOPE];
  for (int i = threadIdx.x; i < kRB * MLA_D_NOPE; i += blockDim.x) {
    int rr = i / MLA_D_NOPE, k = i % MLA_D_NOPE;
    qs[rr][k] = rr < nr ? to_f32(q_nope[((size_t)(r0 + rr) * H + h) * MLA_D_NOPE + k]) : 0.f;
  }
  __syncthreads();
  const int c = 2 * threadIdx.x;  // two latent columns per thread
  float acc[kRB][2];
#pragma unroll
  for (int rr = 0; rr < kRB; ++rr) acc[rr][0] = acc[rr][1] = 0.f;
  const T* w = w_uk + (size_t)h * MLA_D_NOPE * MLA_D_C + c;
#pragma unroll 4
  for (int k = 0; k < MLA_D_NOPE; ++k) {
    float w0 = to_f32(w[(size_t)k * MLA_D_C]);
    float w1 = to_f32(w[(size_t)k * MLA_D_C + 1]);
#pragma unroll
    for (int rr = 0; rr < kRB; ++rr) {
      acc[rr][0] = fmaf(qs[rr][k], w0, acc[rr][0]);
      acc[rr][1] = fmaf(qs[rr][k], w1, acc[rr][1]);
    }
  }
#pragma unroll
  for (int rr = 0; rr < kRB; ++rr) {
    if (rr < nr) {
      T* dst = q_abs + ((size_t)(r0 + rr) * H + h) * MLA_D_ROW;
      dst[c] = from_f32<T>(acc[rr][0]);
      dst[c + 1] = from_f32<T>(acc[rr][1]);
      if (threadIdx.x < MLA_D_R)
        dst[MLA_D_C + threadIdx.x] = q_pe[((size_t)(r0 + rr) * H + h) * MLA_D_R + threadIdx.x];
    }
  }
}

template <typename T>
__global__ void __launch_bounds__(256) out_uv_kernel(const T* __restrict__ o_lat, const T* __restrict__ w_uv,
                                                     T* __restrict__ out, int rows, int H) {
  const int h = blockIdx.x;
  const int r0 = blockIdx.y * kRB;
  const int nr = min(kRB, rows - r0);
  __shared__ float os[kRB][MLA_D_C];
  for (int i = threadIdx.x; i < kRB * MLA_D_C; i += blockDim.x) {
    int rr = i / MLA_D_C, c = i % MLA_D_C;
    os[rr][c] = rr < nr ? to_f32(o_lat[((size_t)(r0 + rr) * H + h) * MLA_D_C + c]) : 0.f;
  }
  __syncthreads();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  for (int i = warp; i < MLA_D_V; i += 8) {
    float w[16];
    load16(w_uv + ((size_t)h * MLA_D_V + i) * MLA_D_C + 16 * lane, w);
    float acc[kRB];
#pragma unroll
    for (int rr = 0; rr < kRB; ++rr) {
      float s = 0.f;
#pragma unroll
      for (int k = 0; k < 16; ++k) s = fmaf(w[k], os[rr][16 * lane + k], s);
      acc[rr] = warp_sum(s);
    }
    if (lane < nr) {
      float v = acc[0];
#pragma unroll
      for (int rr = 1; rr < kRB; ++rr) if (lane == rr) v = acc[rr];
      out[((size_t)(r0 + lane) * H + h) * MLA_D_V + i] = from_f32<T>(v);
    }
  }
}

}  // namespace

cudaError_t launch_absorb_q(const void* q_nope, const void* q_pe, const void* w_uk, void* q_abs,
                            int rows, int n_heads, int dtype, cudaStream_t st) {
  dim3 grid(n_heads, (rows + kRB - 1) / kRB);
  if (dtype == MLA_F32)
    absorb_q_kernel<float><<<grid, 256, 0, st>>>((const float*)q_nope, (const float*)q_pe,
                                                  (const float*)w_uk, (float*)q_abs, rows, n_heads);
  else
    absorb_q_kernel<__nv_bfloat16><<<grid, 256, 0, st>>>(
        (const __nv_bfloat16*)q_nope, (const __nv_bfloat16*)q_pe, (const __nv_bfloat16*)w_uk,
        (__nv_bfloat16*)q_abs, rows, n_heads);
  return cudaGetLastError();
}

cudaError_t launch_out_uv(const void* o_lat, const void* w_uv, void* out, int rows, int n_heads,
                          int dtype, cudaStream_t st) {
  dim3 grid(n_heads, (rows + kRB - 1) / kRB);
  if (dtype == MLA_F32)
    out_uv_kernel<float><<<grid, 256, 0, st>>>((const float*)o_lat, (const float*)w_uv, (float*)out,
                                                rows, n_heads);
  else
    out_uv_kernel<__nv_bfloat16><<<grid, 256, 0, st>>>((const __nv_bfloat16*)o_lat,
                                                        (const __nv_bfloat16*)w_uv,
                                                        (__nv_bfloat16*)out, rows, n_heads);
  return cudaGetLastError();
}

}  // namespace mla
