// Split-KV latent attention on the CUDA cores, exact fp32 arithmetic.
//
// Serves the fp32 cache (small head counts).  "DeepSeek-V2: MLA Explained",
// "MLA Full Formulas" part 3 in absorbed form: per (query row, head, split)
// z_j = scale * q_abs . row_j over the split's visible rows, an online softmax
// and a softmax-weighted sum of the 512 latent channels of the rows.
//
// CTA = (split, group of 16 heads, query row); one warp per head.  Rows are
// staged 32 at a time in shared memory as fp32; lane l owns channels l+32k.
#include <math.h>

#include "mla_device.cuh"
#include "mla_internal.h"

namespace mla {
namespace {

constexpr int kRows = 32;
constexpr int kHeadsPerCta = 16;

template <typename QT, int CK>
__global__ void __launch_bounds__(512) decode_simt_kernel(DecodeArgs a) {
  extern __shared__ float tile[];            // [kRows][576]
  __shared__ long long slot_of[kRows];
  __shared__ float scale_of[kRows];
  const int s = blockIdx.x;
  const int r = blockIdx.z;
  const int b = r / a.q_len, t = r % a.q_len;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int h = blockIdx.y * kHeadsPerCta + warp;
  const bool active = h < a.n_heads;
  const int L = a.seq_lens[b];
  const int n_vis = L - a.q_len + t + 1;
  const int lo = s * a.split_tokens;
  const int hi = min((s + 1) * a.split_tokens, n_vis);

  float q[18];
  {
    const QT* qp = reinterpret_cast<const QT*>(a.q_abs) + ((size_t)r * a.n_heads + (active ? h : 0)) * MLA_D_ROW;
#pragma unroll
    for (int k = 0; k < 18; ++k) q[k] = to_f32(qp[lane + 32 * k]);
  }
  float m = -INFINITY, l = 0.f;
  float o[16];
#pragma unroll
  for (int k = 0; k < 16; ++k) o[k] = 0.f;

  for (int j0 = lo; j0 < hi; j0 += kRows) {
    const int n = min(kRows, hi - j0);
    __syncthreads();
    if (threadIdx.x < kRows) {
      long long sl = -1;
      float sc = 1.f;
      if (threadIdx.x < n) {
        const int j = j0 + threadIdx.x;
        const int pidx = j / a.page_size;
        const int page = pidx < a.max_pages ? a.block_table[(size_t)b * a.max_pages + pidx] : -1;
        if (page >= 0 && page < a.num_pages) {
          sl = (long long)page * a.page_size + j % a.page_size;
          if (CK == MLA_E4M3) sc = a.cache_scale[sl];
        } else {
          flag_error(a.err, MLA_DEVERR_PAGE);
        }
      }
      slot_of[threadIdx.x] = sl;
      scale_of[threadIdx.x] = sc;
    }
    __syncthreads();
    for (int i = threadIdx.x; i < n * MLA_D_ROW; i += blockDim.x) {
      const int jj = i / MLA_D_ROW, d = i % MLA_D_ROW;
      const long long sl = slot_of[jj];
      float v = 0.f;
      if (sl >= 0) {
        const size_t ci = cache_index((size_t)sl, d);
        if (CK == MLA_F32) v = reinterpret_cast<const float*>(a.cache)[ci];
        else if (CK == MLA_BF16) v = to_f32(reinterpret_cast<const __nv_bfloat16*>(a.cache)[ci]);
        else v = e4m3_to_f32(reinterpret_cast<const uint8_t*>(a.cache)[ci]) * scale_of[jj];
      }
      tile[jj * MLA_D_ROW + d] = v;
    }
    __syncthreads();
    if (!active) continue;
    float sc = -INFINITY;                    // lane jj ends up with row jj's score
    for (int jj = 0; jj < n; ++jj) {
      float part = 0.f;
#pragma unroll
      for (int k = 0; k < 18; ++k) part = fmaf(q[k], tile[jj * MLA_D_ROW + lane + 32 * k], part);
      part = warp_sum(part);
      if (lane == jj) sc = (slot_of[jj] >= 0) ? part * a.softmax_scale : -INFINITY;
    }
    const float mt = warp_max(sc);
    const float mn = fmaxf(m, mt);
    if (mn == -INFINITY) continue;          // every row of the tile was skipped
    const float alpha = expf(m - mn);
    const float p = (lane < n) ? expf(sc - mn) : 0.f;
    l = l * alpha + warp_sum(p);
#pragma unroll
    for (int k = 0; k < 16; ++k) o[k] *= alpha;
    for (int jj = 0; jj < n; ++jj) {
      const float pj = __shfl_sync(0xffffffffu, p, jj);
#pragma unroll
      for (int k = 0; k < 16; ++k) o[k] = fmaf(pj, tile[jj * MLA_D_ROW + lane + 32 * k], o[k]);
    }
    m = mn;
  }
  if (!active) return;
  const size_t base = ((size_t)r * a.n_heads + h) * a.num_splits + s;
  const float inv = l > 0.f ? 1.0f / l : 0.f;
#pragma unroll
  for (int k = 0; k < 16; ++k) a.o_part[base * MLA_D_C + lane + 32 * k] = o[k] * inv;
  if (lane == 0) a.lse_part[base] = l > 0.f ? m + logf(l) : -INFINITY;
}

template <typename QT, int CK>
cudaError_t launch_t(const DecodeArgs& a, cudaStream_t st) {
  const size_t smem = (size_t)kRows * MLA_D_ROW * sizeof(float);
  cudaError_t e = cudaFuncSetAttribute(decode_simt_kernel<QT, CK>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  dim3 grid(a.num_splits, (a.n_heads + kHeadsPerCta - 1) / kHeadsPerCta, a.batch * a.q_len);
  decode_simt_kernel<QT, CK><<<grid, 512, smem, st>>>(a);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_decode_simt(const DecodeArgs& a, cudaStream_t st) {
  if (a.q_dtype == MLA_F32) {
    if (a.cache_dtype == MLA_F32) return launch_t<float, MLA_F32>(a, st);
    if (a.cache_dtype == MLA_BF16) return launch_t<float, MLA_BF16>(a, st);
    return launch_t<float, MLA_E4M3>(a, st);
  }
  if (a.cache_dtype == MLA_F32) return launch_t<__nv_bfloat16, MLA_F32>(a, st);
  if (a.cache_dtype == MLA_BF16) return launch_t<__nv_bfloat16, MLA_BF16>(a, st);
  return launch_t<__nv_bfloat16, MLA_E4M3>(a, st);
}

}  // namespace mla
