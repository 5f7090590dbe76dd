// Log-sum-exp merge of split-KV partials.
//
// The softmax sum of "DeepSeek-V2: MLA Explained", "MLA Full Formulas" part 3
// splits exactly over disjoint row ranges: with each split's normalised
// output o_s and log-normaliser lse_s, the full output is the lse-weighted
// mean of the o_s.  One CTA per (query row, head); 128 threads x 4 channels.
#include <math.h>

#include "mla_device.cuh"
#include "mla_internal.h"

namespace mla {
namespace {

template <typename OT>
__global__ void __launch_bounds__(128) combine_kernel(const float* __restrict__ o_part,
                                                      const float* __restrict__ lse_part, int S,
                                                      OT* __restrict__ o_lat, float* __restrict__ lse_out) {
  extern __shared__ float w[];               // [S] weights
  __shared__ float red[4];
  const size_t rh = blockIdx.x;
  const float* lp = lse_part + rh * S;
  // max over splits
  float mx = -INFINITY;
  for (int s = threadIdx.x; s < S; s += blockDim.x) mx = fmaxf(mx, lp[s]);
  mx = warp_max(mx);
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = mx;
  __syncthreads();
  mx = fmaxf(fmaxf(red[0], red[1]), fmaxf(red[2], red[3]));
  __syncthreads();
  float sum = 0.f;
  for (int s = threadIdx.x; s < S; s += blockDim.x) {
    const float v = lp[s];
    const float ws = (mx == -INFINITY || v == -INFINITY) ? 0.f : expf(v - mx);
    w[s] = ws;
    sum += ws;
  }
  sum = warp_sum(sum);
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = sum;
  __syncthreads();
  sum = red[0] + red[1] + red[2] + red[3];
  const float inv = sum > 0.f ? 1.0f / sum : 0.f;
  const float4* op = reinterpret_cast<const float4*>(o_part + rh * (size_t)S * MLA_D_C) + threadIdx.x;
  float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
  for (int s = 0; s < S; ++s) {
    const float ws = w[s];
    if (ws == 0.f) continue;
    const float4 v = op[(size_t)s * (MLA_D_C / 4)];
    acc.x = fmaf(ws, v.x, acc.x); acc.y = fmaf(ws, v.y, acc.y);
    acc.z = fmaf(ws, v.z, acc.z); acc.w = fmaf(ws, v.w, acc.w);
  }
  OT* dst = o_lat + rh * MLA_D_C + 4 * threadIdx.x;
  dst[0] = from_f32<OT>(acc.x * inv); dst[1] = from_f32<OT>(acc.y * inv);
  dst[2] = from_f32<OT>(acc.z * inv); dst[3] = from_f32<OT>(acc.w * inv);
  if (lse_out && threadIdx.x == 0) lse_out[rh] = sum > 0.f ? mx + logf(sum) : -INFINITY;
}

}  // namespace

cudaError_t launch_combine(const float* o_part, const float* lse_part, int rows, int n_heads,
                           int num_splits, void* o_lat, int o_dtype, float* lse_out,
                           cudaStream_t st) {
  const size_t n = (size_t)rows * n_heads;
  if (n == 0) return cudaSuccess;
  const size_t smem = (size_t)num_splits * sizeof(float);
  if (o_dtype == MLA_F32)
    combine_kernel<float><<<(unsigned)n, 128, smem, st>>>(o_part, lse_part, num_splits, (float*)o_lat, lse_out);
  else
    combine_kernel<__nv_bfloat16><<<(unsigned)n, 128, smem, st>>>(o_part, lse_part, num_splits,
                                                                  (__nv_bfloat16*)o_lat, lse_out);
  return cudaGetLastError();
}

}  // namespace mla
