// Per-head projections on either side of latent attention.
//
//   absorb_q:  q_abs[r,h,0:512] = W_UK[h]^T q_nope[r,h]  and q_abs[r,h,512:] = q_pe[r,h]
//   out_uv:    out[r,h,:]       = W_UV[h]   o_lat[r,h]
//
// "DeepSeek-V2: MLA Explained", "Optimization Note": W_UK merges into the
// query and W_UV is applied after the softmax sum.  Each is a batched per-head
// product with a short row count (B*T) against a 128x512 weight per head: the
// weight read (16.8 MB bf16 at 128 heads) dominates, so CTAs split each head's
// weight into slices, keep all of a slice's 16-byte loads in flight, and reuse
// each weight element for up to kRB rows held in shared memory.
#include "mla_device.cuh"
#include "mla_internal.h"

namespace mla {
namespace {

constexpr int kRB = 8;        // query rows per CTA
// bf16 projections run on the tensor cores (project_tc.cu); the CUDA-core
// kernels below serve fp32
constexpr bool kUseTensorCores = true;
constexpr int kThr = 128;     // threads per CTA

// 16-byte vector of T, widened to float
template <typename T> struct Vec;
template <> struct Vec<float> {
  static constexpr int N = 4;
  __device__ static void load(const float* p, float* v) {
    const float4 x = *reinterpret_cast<const float4*>(p);
    v[0] = x.x; v[1] = x.y; v[2] = x.z; v[3] = x.w;
  }
};
template <> struct Vec<__nv_bfloat16> {
  static constexpr int N = 8;
  __device__ static void load(const __nv_bfloat16* p, float* v) {
    const uint4 x = *reinterpret_cast<const uint4*>(p);
    const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&x);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const float2 f = __bfloat1622float2(h[i]);
      v[2 * i] = f.x; v[2 * i + 1] = f.y;
    }
  }
};

// absorb_q: CTA (head h, rows r0..r0+7, columns 128*z..128*z+127).  Thread t
// owns VEC adjacent columns and a slice of the 128 contraction rows k, so each
// thread has its whole slice of W_UK in flight as 16-byte loads; the k-slices
// are summed through shared memory.
template <typename T>
__global__ void __launch_bounds__(kThr) absorb_q_kernel(const T* __restrict__ q_nope, const T* __restrict__ q_pe,
                                                        const T* __restrict__ w_uk, T* __restrict__ q_abs,
                                                        int rows, int H) {
  constexpr int V = Vec<T>::N;
  constexpr int NCG = 128 / V;            // column groups per CTA
  constexpr int NKG = kThr / NCG;         // k slices
  constexpr int KPG = MLA_D_NOPE / NKG;   // k per slice
  const int h = blockIdx.x, r0 = blockIdx.y * kRB, z = blockIdx.z;
  const int nr = min(kRB, rows - r0);
  __shared__ float qs[kRB][MLA_D_NOPE];
  __shared__ float part[NKG][kRB][128];
  // stage the rows' q_nope (16-byte loads, all issued before use)
  {
    constexpr int PER_ROW = MLA_D_NOPE / V;                  // vectors per row
    constexpr int NV = (kRB * PER_ROW + kThr - 1) / kThr;
    float v[NV][V];
#pragma unroll
    for (int j = 0; j < NV; ++j) {
      const int i = threadIdx.x + j * kThr, rr = i / PER_ROW, cv = i % PER_ROW;
      if (i < kRB * PER_ROW && rr < nr) Vec<T>::load(q_nope + ((size_t)(r0 + rr) * H + h) * MLA_D_NOPE + V * cv, v[j]);
      else
#pragma unroll
        for (int e = 0; e < V; ++e) v[j][e] = 0.f;
    }
#pragma unroll
    for (int j = 0; j < NV; ++j) {
      const int i = threadIdx.x + j * kThr, rr = i / PER_ROW, cv = i % PER_ROW;
      if (i < kRB * PER_ROW)
#pragma unroll
        for (int e = 0; e < V; ++e) qs[rr][V * cv + e] = v[j][e];
    }
  }
  __syncthreads();
  const int cg = threadIdx.x % NCG, kg = threadIdx.x / NCG;
  const int c0 = 128 * z + V * cg;
  float acc[kRB][V];
#pragma unroll
  for (int rr = 0; rr < kRB; ++rr)
#pragma unroll
    for (int e = 0; e < V; ++e) acc[rr][e] = 0.f;
  const T* w = w_uk + ((size_t)h * MLA_D_NOPE + kg * KPG) * MLA_D_C + c0;
#pragma unroll
  for (int kb = 0; kb < KPG; kb += 8) {
    uint4 raw[8];
#pragma unroll
    for (int j = 0; j < 8; ++j) raw[j] = __ldg(reinterpret_cast<const uint4*>(w + (size_t)(kb + j) * MLA_D_C));
    float wv[8][V];
#pragma unroll
    for (int j = 0; j < 8; ++j) Vec<T>::load(reinterpret_cast<const T*>(&raw[j]), wv[j]);
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const int k = kg * KPG + kb + j;
#pragma unroll
      for (int rr = 0; rr < kRB; ++rr) {
        const float qv = qs[rr][k];
#pragma unroll
        for (int e = 0; e < V; ++e) acc[rr][e] = fmaf(qv, wv[j][e], acc[rr][e]);
      }
    }
  }
#pragma unroll
  for (int rr = 0; rr < kRB; ++rr)
#pragma unroll
    for (int e = 0; e < V; ++e) part[kg][rr][V * cg + e] = acc[rr][e];
  __syncthreads();
  for (int i = threadIdx.x; i < kRB * 128; i += kThr) {
    const int rr = i / 128, cl = i % 128;
    if (rr >= nr) continue;
    float v = 0.f;
#pragma unroll
    for (int g = 0; g < NKG; ++g) v += part[g][rr][cl];
    q_abs[((size_t)(r0 + rr) * H + h) * MLA_D_ROW + 128 * z + cl] = from_f32<T>(v);
  }
  if (z == 0 && threadIdx.x < MLA_D_R)
    for (int rr = 0; rr < nr; ++rr)
      q_abs[((size_t)(r0 + rr) * H + h) * MLA_D_ROW + MLA_D_C + threadIdx.x] =
          q_pe[((size_t)(r0 + rr) * H + h) * MLA_D_R + threadIdx.x];
}

// out_uv: CTA (head h, rows r0..r0+7, outputs 32*z..32*z+31).  Four adjacent
// threads share an output n and split its 512 contraction columns in quarters
// (16-byte loads, all in flight); two xor-shuffles sum the quarters.
template <typename T>
__global__ void __launch_bounds__(kThr) out_uv_kernel(const T* __restrict__ o_lat, const T* __restrict__ w_uv,
                                                      T* __restrict__ out, int rows, int H) {
  constexpr int V = Vec<T>::N;
  constexpr int KQ = MLA_D_C / 4;          // columns per quarter
  const int h = blockIdx.x, r0 = blockIdx.y * kRB, z = blockIdx.z;
  const int nr = min(kRB, rows - r0);
  __shared__ float os[kRB][4][KQ + 1];     // +1: the four quarters fall in different banks
  // stage the rows' o_lat (16-byte loads, all issued before use)
  {
    constexpr int PER_ROW = MLA_D_C / V;
    constexpr int NV = (kRB * PER_ROW + kThr - 1) / kThr;
    float v[NV][V];
#pragma unroll
    for (int j = 0; j < NV; ++j) {
      const int i = threadIdx.x + j * kThr, rr = i / PER_ROW, cv = i % PER_ROW;
      if (i < kRB * PER_ROW && rr < nr) Vec<T>::load(o_lat + ((size_t)(r0 + rr) * H + h) * MLA_D_C + V * cv, v[j]);
      else
#pragma unroll
        for (int e = 0; e < V; ++e) v[j][e] = 0.f;
    }
#pragma unroll
    for (int j = 0; j < NV; ++j) {
      const int i = threadIdx.x + j * kThr, rr = i / PER_ROW, cv = i % PER_ROW;
      if (i < kRB * PER_ROW)
#pragma unroll
        for (int e = 0; e < V; ++e) {
          const int c = V * cv + e;
          os[rr][c / KQ][c % KQ] = v[j][e];
        }
    }
  }
  __syncthreads();
  const int lane = threadIdx.x & 31;
  const int n = 32 * z + threadIdx.x / 4, q = threadIdx.x % 4;
  const T* w = w_uv + ((size_t)h * MLA_D_V + n) * MLA_D_C + KQ * q;
  float acc[kRB];
#pragma unroll
  for (int rr = 0; rr < kRB; ++rr) acc[rr] = 0.f;
  // all of this thread's weight slice (KQ * sizeof(T) bytes) is requested before any use
  constexpr int NL = KQ / V;
  uint4 raw[NL];
#pragma unroll
  for (int j = 0; j < NL; ++j) raw[j] = __ldg(reinterpret_cast<const uint4*>(w + (size_t)j * V));
#pragma unroll
  for (int j = 0; j < NL; ++j) {
    float wv[V];
    Vec<T>::load(reinterpret_cast<const T*>(&raw[j]), wv);
#pragma unroll
    for (int e = 0; e < V; ++e)
#pragma unroll
      for (int rr = 0; rr < kRB; ++rr) acc[rr] = fmaf(wv[e], os[rr][q][j * V + e], acc[rr]);
  }
#pragma unroll
  for (int rr = 0; rr < kRB; ++rr) {
    acc[rr] += __shfl_xor_sync(0xffffffffu, acc[rr], 1);
    acc[rr] += __shfl_xor_sync(0xffffffffu, acc[rr], 2);
  }
  (void)lane;
#pragma unroll
  for (int rr = 0; rr < kRB; ++rr)
    if ((rr & 3) == q && rr < nr) out[((size_t)(r0 + rr) * H + h) * MLA_D_V + n] = from_f32<T>(acc[rr]);
}

}  // namespace

cudaError_t launch_absorb_q(const void* q_nope, const void* q_pe, const void* w_uk, void* q_abs,
                            int rows, int n_heads, int dtype, cudaStream_t st) {
  if (rows == 0) return cudaSuccess;
  if (dtype == MLA_BF16 && kUseTensorCores) return launch_absorb_q_tc(q_nope, q_pe, w_uk, q_abs, rows, n_heads, st);
  dim3 grid(n_heads, (rows + kRB - 1) / kRB, MLA_D_C / 128);
  if (dtype == MLA_F32)
    absorb_q_kernel<float><<<grid, kThr, 0, st>>>((const float*)q_nope, (const float*)q_pe,
                                                  (const float*)w_uk, (float*)q_abs, rows, n_heads);
  else
    absorb_q_kernel<__nv_bfloat16><<<grid, kThr, 0, st>>>(
        (const __nv_bfloat16*)q_nope, (const __nv_bfloat16*)q_pe, (const __nv_bfloat16*)w_uk,
        (__nv_bfloat16*)q_abs, rows, n_heads);
  return cudaGetLastError();
}

cudaError_t launch_out_uv(const void* o_lat, const void* w_uv, void* out, int rows, int n_heads,
                          int dtype, cudaStream_t st) {
  if (rows == 0) return cudaSuccess;
  if (dtype == MLA_BF16 && kUseTensorCores) return launch_out_uv_tc(o_lat, w_uv, out, rows, n_heads, st);
  dim3 grid(n_heads, (rows + kRB - 1) / kRB, MLA_D_V / 32);
  if (dtype == MLA_F32)
    out_uv_kernel<float><<<grid, kThr, 0, st>>>((const float*)o_lat, (const float*)w_uv, (float*)out,
                                                rows, n_heads);
  else
    out_uv_kernel<__nv_bfloat16><<<grid, kThr, 0, st>>>((const __nv_bfloat16*)o_lat,
                                                        (const __nv_bfloat16*)w_uv,
                                                        (__nv_bfloat16*)out, rows, n_heads);
  return cudaGetLastError();
}

}  // namespace mla
