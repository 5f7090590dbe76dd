// Log-sum-exp merge of split-KV partials.
//
// The softmax sum of "DeepSeek-V2: MLA Explained", "MLA Full Formulas" part 3
// splits exactly over disjoint row ranges: with each split's normalised
// output o_s and log-normaliser lse_s, the full output is the lse-weighted
// mean of the o_s.  One CTA per (query row, head); 128 threads x 4 channels.
// The same merge serves two layouts of the parts: the splits of one decode
// launch ([rows, heads, splits, 512]) and the per-GPU results of a sequence
// whose rows are sharded across GPUs ([shards, rows, heads, 512]).
#include <math.h>

#include "mla_device.cuh"
#include "mla_internal.h"

namespace mla {
namespace {

// Strides (in floats) between the parts of one (row, head) and between
// consecutive (row, head) pairs, for o (multiples of 4) and for lse.
struct PartStrides {
  size_t o_part, o_rh, l_part, l_rh;
};

template <typename OT>
__global__ void __launch_bounds__(128) combine_kernel(const float* __restrict__ o_part,
                                                      const float* __restrict__ lse_part, int S, PartStrides st,
                                                      OT* __restrict__ o_lat, float* __restrict__ lse_out) {
  extern __shared__ float w[];               // [S] weights
  __shared__ float red[4];
  griddep_wait();
  griddep_launch_dependents();
  const size_t rh = blockIdx.x;
  const float* lp = lse_part + rh * st.l_rh;
  // max over splits
  float mx = -INFINITY;
  for (int s = threadIdx.x; s < S; s += blockDim.x) mx = fmaxf(mx, lp[s * st.l_part]);
  mx = warp_max(mx);
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = mx;
  __syncthreads();
  mx = fmaxf(fmaxf(red[0], red[1]), fmaxf(red[2], red[3]));
  __syncthreads();
  float sum = 0.f;
  for (int s = threadIdx.x; s < S; s += blockDim.x) {
    const float v = lp[s * st.l_part];
    const float ws = (mx == -INFINITY || v == -INFINITY) ? 0.f : expf(v - mx);
    w[s] = ws;
    sum += ws;
  }
  sum = warp_sum(sum);
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = sum;
  __syncthreads();
  sum = red[0] + red[1] + red[2] + red[3];
  const float inv = sum > 0.f ? 1.0f / sum : 0.f;
  const float4* op = reinterpret_cast<const float4*>(o_part + rh * st.o_rh) + threadIdx.x;
  const size_t ps = st.o_part / 4;
  float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
  // eight parts per batch: their loads are issued together, so a batch costs
  // one memory latency (parts of weight 0 are not read: their o may be unset)
  for (int s0 = 0; s0 < S; s0 += 8) {
    float ws[8];
    float4 v[8];
#pragma unroll
    for (int k = 0; k < 8; ++k) {
      ws[k] = s0 + k < S ? w[s0 + k] : 0.f;
      v[k] = ws[k] != 0.f ? op[(size_t)(s0 + k) * ps] : make_float4(0.f, 0.f, 0.f, 0.f);
    }
#pragma unroll
    for (int k = 0; k < 8; ++k) {
      acc.x = fmaf(ws[k], v[k].x, acc.x); acc.y = fmaf(ws[k], v[k].y, acc.y);
      acc.z = fmaf(ws[k], v[k].z, acc.z); acc.w = fmaf(ws[k], v[k].w, acc.w);
    }
  }
  OT* dst = o_lat + rh * MLA_D_C + 4 * threadIdx.x;
  dst[0] = from_f32<OT>(acc.x * inv); dst[1] = from_f32<OT>(acc.y * inv);
  dst[2] = from_f32<OT>(acc.z * inv); dst[3] = from_f32<OT>(acc.w * inv);
  if (lse_out && threadIdx.x == 0) lse_out[rh] = sum > 0.f ? mx + logf(sum) : -INFINITY;
}

}  // namespace

cudaError_t launch_combine(const float* o_part, const float* lse_part, int rows, int n_heads,
                           int num_parts, bool shard_major, void* o_lat, int o_dtype, float* lse_out,
                           cudaStream_t st) {
  const size_t n = (size_t)rows * n_heads;
  if (n == 0) return cudaSuccess;
  const size_t smem = (size_t)num_parts * sizeof(float);
  // splits of one launch: [rows, heads, parts, 512]; shards: [parts, rows, heads, 512]
  const PartStrides ps = shard_major ? PartStrides{n * MLA_D_C, MLA_D_C, n, 1}
                                     : PartStrides{MLA_D_C, (size_t)num_parts * MLA_D_C, 1, (size_t)num_parts};
  if (o_dtype == MLA_F32)
    return launch_dependent(combine_kernel<float>, dim3((unsigned)n), dim3(128), smem, st, o_part, lse_part,
                            num_parts, ps, (float*)o_lat, lse_out);
  return launch_dependent(combine_kernel<__nv_bfloat16>, dim3((unsigned)n), dim3(128), smem, st, o_part, lse_part,
                          num_parts, ps, (__nv_bfloat16*)o_lat, lse_out);
}

}  // namespace mla
