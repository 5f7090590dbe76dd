// The two-term e4m3 form of absorbed queries, the query operand of the 8-bit
// tensor-core decode over an e4m3 cache.
//
// An e4m3 cache ("DeepSeek'in MLA'si latent attention ile KV cache'i %93
// sikistiriyor", cache section; OCP FP8 E4M3) lets both GEMMs of the decode
// run on 8-bit MMAs, whose two operands are both 8-bit.  One e4m3 rounding of
// the query (relative 2^-4) would move the scores too far, so the query is
// carried as two e4m3 terms on one fp32 scale per (row, head):
//   a = max|q|, inv = 448 / a, y = q * inv, hi = e4m3(y), lo = e4m3(y - hi),
//   scale = a / 448
// with every step in fp32 round-to-nearest-even; q ~ scale * (hi + lo) to
// about 2^-8 relative.  One warp per (row, head) vector of 576 values: lane l
// holds values 2 (l + 32 k) and 2 (l + 32 k) + 1, k = 0..8, so every load and
// store of the warp is contiguous.  Memory-bound: 1152 bytes in, 1156 out.
#include "mla_device.cuh"
#include "mla_internal.h"

namespace mla {
namespace {

__global__ void __launch_bounds__(256) split_q_kernel(const __nv_bfloat16* __restrict__ q_abs, int n_vec,
                                                      int n_heads, uint8_t* __restrict__ q8,
                                                      float* __restrict__ q_scale) {
  griddep_wait();
  griddep_launch_dependents();
  const int vec = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (vec >= n_vec) return;
  const int row = vec / n_heads, h = vec - row * n_heads;
  const uint32_t* src = reinterpret_cast<const uint32_t*>(q_abs + (size_t)vec * MLA_D_ROW);
  float2 x[9];
  float amax = 0.f;
#pragma unroll
  for (int k = 0; k < 9; ++k) {
    const uint32_t w = __ldg(src + lane + 32 * k);
    x[k] = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&w));
    amax = fmaxf(amax, fmaxf(fabsf(x[k].x), fabsf(x[k].y)));
  }
  amax = warp_max(amax);
  const float inv = amax > 0.f ? __fdiv_rn(448.f, amax) : 0.f;
  uint16_t* hi = reinterpret_cast<uint16_t*>(q8 + ((size_t)(2 * row) * n_heads + h) * MLA_D_ROW);
  uint16_t* lo = reinterpret_cast<uint16_t*>(q8 + ((size_t)(2 * row + 1) * n_heads + h) * MLA_D_ROW);
#pragma unroll
  for (int k = 0; k < 9; ++k) {
    uint32_t h2, l2;
    split_e4m3x2(__fmul_rn(x[k].x, inv), __fmul_rn(x[k].y, inv), h2, l2);
    hi[lane + 32 * k] = (uint16_t)h2;
    lo[lane + 32 * k] = (uint16_t)l2;
  }
  if (lane == 0) q_scale[vec] = __fdiv_rn(amax, 448.f);
}

}  // namespace

cudaError_t launch_split_q_e4m3(const void* q_abs, int rows, int n_heads, void* q8, float* q_scale,
                                cudaStream_t st) {
  const int n_vec = rows * n_heads;
  if (n_vec == 0) return cudaSuccess;
  return launch_dependent(split_q_kernel, dim3((unsigned)((n_vec + 7) / 8)), dim3(256), 0, st,
                          static_cast<const __nv_bfloat16*>(q_abs), n_vec, n_heads, static_cast<uint8_t*>(q8),
                          q_scale);
}

}  // namespace mla
