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
#include "sm100.cuh"

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

// combine_out_uv (bf16): the merge above for one (query row, head), then the
// value up-projection out[r,h,:] = W_UV[h] o_lat[r,h,:] ("MLA Full Formulas"
// part 2, applied after the attention sum per "Optimization Note") in the same
// CTA, for steps with few query rows.  The head's W_UV (128 KB) is copied into
// shared memory by one bulk copy started at entry (no earlier kernel writes
// the weights), so its load overlaps the merge.  o_lat is rounded to bf16
// exactly as mla_combine stores it (and stored too); warp w then computes
// outputs 32 w .. 32 w + 31, lane l taking 16-byte pieces l and l + 32 of
// each weight row, a butterfly sum per output.
constexpr uint32_t kWuvBytes = MLA_D_V * MLA_D_C * 2;

__global__ void __launch_bounds__(128) combine_out_uv_kernel(const float* __restrict__ o_part,
                                                             const float* __restrict__ lse_part, int S,
                                                             const __nv_bfloat16* __restrict__ w_uv, int H,
                                                             __nv_bfloat16* __restrict__ o_lat,
                                                             __nv_bfloat16* __restrict__ out,
                                                             float* __restrict__ lse_out) {
  extern __shared__ __align__(1024) uint8_t dyn[];   // W_UV[h] (128 KB), then [S] weights
  __shared__ float red[4];
  __shared__ __align__(16) __nv_bfloat16 ol[MLA_D_C];
  __shared__ __align__(8) uint64_t wbar;
  __shared__ int abort_w;
  const __nv_bfloat16* ws_w = reinterpret_cast<const __nv_bfloat16*>(dyn);
  float* w = reinterpret_cast<float*>(dyn + kWuvBytes);
  const size_t rh = blockIdx.x;
  const int h = (int)(rh % (size_t)H);
  const uint32_t bar = sm100::smem_u32(&wbar);
  if (threadIdx.x == 0) {
    sm100::mbar_init(bar, 1);
    abort_w = 0;
    sm100::fence_mbar_init();
    sm100::mbar_arrive_expect_tx(bar, kWuvBytes);
    sm100::bulk_load(sm100::smem_u32(dyn), w_uv + (size_t)h * MLA_D_V * MLA_D_C, kWuvBytes, bar);
  }
  griddep_wait();
  griddep_launch_dependents();
  const float* lp = lse_part + rh * S;
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
  for (int s0 = 0; s0 < S; s0 += 8) {
    float wk[8];
    float4 v[8];
#pragma unroll
    for (int k = 0; k < 8; ++k) {
      wk[k] = s0 + k < S ? w[s0 + k] : 0.f;
      v[k] = wk[k] != 0.f ? op[(size_t)(s0 + k) * (MLA_D_C / 4)] : make_float4(0.f, 0.f, 0.f, 0.f);
    }
#pragma unroll
    for (int k = 0; k < 8; ++k) {
      acc.x = fmaf(wk[k], v[k].x, acc.x); acc.y = fmaf(wk[k], v[k].y, acc.y);
      acc.z = fmaf(wk[k], v[k].z, acc.z); acc.w = fmaf(wk[k], v[k].w, acc.w);
    }
  }
  const __nv_bfloat162 a2 = __floats2bfloat162_rn(acc.x * inv, acc.y * inv);
  const __nv_bfloat162 b2 = __floats2bfloat162_rn(acc.z * inv, acc.w * inv);
  *reinterpret_cast<__nv_bfloat162*>(ol + 4 * threadIdx.x) = a2;
  *reinterpret_cast<__nv_bfloat162*>(ol + 4 * threadIdx.x + 2) = b2;
  if (o_lat) {
    __nv_bfloat162* dst = reinterpret_cast<__nv_bfloat162*>(o_lat + rh * MLA_D_C + 4 * threadIdx.x);
    dst[0] = a2;
    dst[1] = b2;
  }
  if (lse_out && threadIdx.x == 0) lse_out[rh] = sum > 0.f ? mx + logf(sum) : -INFINITY;
  __syncthreads();
  // ---- out = W_UV[h] o_lat: lane l holds o_lat elements 8l..8l+7 and 256+8l..256+8l+7
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const bool wok = sm100::mbar_wait<false>(bar, 0, &abort_w);
  if (!wok) {
    // the weight copy did not complete within the bound: NaN rather than a
    // wrong output, after giving the copy time to land in this CTA's memory
    out[rh * MLA_D_V + 32 * warp + lane] = __float2bfloat16_rn(NAN);
    const uint64_t t0 = sm100::globaltimer();
    while (sm100::globaltimer() - t0 < 2000000ull) {
    }
    return;
  }
  float x[16];
  {
    const uint4 u0 = *reinterpret_cast<const uint4*>(ol + 8 * lane);
    const uint4 u1 = *reinterpret_cast<const uint4*>(ol + 256 + 8 * lane);
    const __nv_bfloat162* p0 = reinterpret_cast<const __nv_bfloat162*>(&u0);
    const __nv_bfloat162* p1 = reinterpret_cast<const __nv_bfloat162*>(&u1);
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const float2 f0 = __bfloat1622float2(p0[e]), f1 = __bfloat1622float2(p1[e]);
      x[2 * e] = f0.x; x[2 * e + 1] = f0.y; x[8 + 2 * e] = f1.x; x[8 + 2 * e + 1] = f1.y;
    }
  }
  const __nv_bfloat16* wrow = ws_w + (size_t)(32 * warp) * MLA_D_C;
  float res = 0.f;                           // lane l ends with output 32 warp + l
#pragma unroll 4
  for (int n = 0; n < 32; ++n) {
    const uint4 wa = *reinterpret_cast<const uint4*>(wrow + (size_t)n * MLA_D_C + 8 * lane);
    const uint4 wb = *reinterpret_cast<const uint4*>(wrow + (size_t)n * MLA_D_C + 256 + 8 * lane);
    const __nv_bfloat162* pa = reinterpret_cast<const __nv_bfloat162*>(&wa);
    const __nv_bfloat162* pb = reinterpret_cast<const __nv_bfloat162*>(&wb);
    float d = 0.f;
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const float2 fa = __bfloat1622float2(pa[e]), fb = __bfloat1622float2(pb[e]);
      d = fmaf(fa.x, x[2 * e], d); d = fmaf(fa.y, x[2 * e + 1], d);
      d = fmaf(fb.x, x[8 + 2 * e], d); d = fmaf(fb.y, x[8 + 2 * e + 1], d);
    }
    d = warp_sum(d);
    if (lane == n) res = d;
  }
  out[rh * MLA_D_V + 32 * warp + lane] = __float2bfloat16_rn(res);
}

}  // namespace

cudaError_t launch_combine_out_uv(const float* o_part, const float* lse_part, int rows, int n_heads, int num_splits,
                                  const void* w_uv, void* o_lat, void* out, float* lse_out, cudaStream_t st) {
  const size_t n = (size_t)rows * n_heads;
  if (n == 0) return cudaSuccess;
  const size_t smem = kWuvBytes + (size_t)num_splits * sizeof(float);
  cudaError_t e = cudaFuncSetAttribute(combine_out_uv_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  return launch_dependent(combine_out_uv_kernel, dim3((unsigned)n), dim3(128), smem, st,
                          o_part, lse_part, num_splits, static_cast<const __nv_bfloat16*>(w_uv), n_heads,
                          static_cast<__nv_bfloat16*>(o_lat), static_cast<__nv_bfloat16*>(out), lse_out);
}

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
