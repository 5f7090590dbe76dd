// Small device helpers shared by the kernels: element loads/stores per dtype,
// warp reductions and the device error word.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp8.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "mla.h"

namespace mla {

// Programmatic dependent launch.  griddep_wait: wait until the kernel before
// this one on the stream has completed and its memory is visible (returns at
// once when this launch did not allow an early start).  Everything before it
// may overlap the previous kernel, so it touches no global memory.
// griddep_launch_dependents: the next kernel may begin its own set-up.
__device__ __forceinline__ void griddep_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void griddep_launch_dependents() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}

// Page-blocked cache layout: a 64-row page is stored as nine blocks of
// [64 rows x 64 columns], block c holding columns 64c..64c+63, so every
// block is contiguous in memory.  Element index of (slot = page*64 + row, d).
__device__ __forceinline__ size_t cache_index(size_t slot, int d) {
  const size_t page = slot >> 6;
  const int row = static_cast<int>(slot & 63);
  return ((page * (MLA_D_ROW / 64) + (d >> 6)) * 64 + row) * 64 + (d & 63);
}

__device__ __forceinline__ void flag_error(int32_t* err, int32_t bits) {
  if (err) atomicOr(err, bits);
}

// dtype tags for templates
struct F32 { using T = float; static constexpr int kBytes = 4; };
struct BF16 { using T = __nv_bfloat16; static constexpr int kBytes = 2; };

__device__ __forceinline__ float to_f32(float v) { return v; }
__device__ __forceinline__ float to_f32(__nv_bfloat16 v) { return __bfloat162float(v); }

template <typename T> __device__ __forceinline__ T from_f32(float v);
template <> __device__ __forceinline__ float from_f32<float>(float v) { return v; }
template <> __device__ __forceinline__ __nv_bfloat16 from_f32<__nv_bfloat16>(float v) {
  return __float2bfloat16_rn(v);
}

// e4m3 code -> float (exact)
__device__ __forceinline__ float e4m3_to_f32(uint8_t c) {
  __half_raw h = __nv_cvt_fp8_to_halfraw(static_cast<__nv_fp8_storage_t>(c), __NV_E4M3);
  return __half2float(__half(h));
}

// Load 16 consecutive elements (16-byte aligned) as floats.
__device__ __forceinline__ void load16(const float* p, float* v) {
  const float4* q = reinterpret_cast<const float4*>(p);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    float4 x = q[i];
    v[4 * i] = x.x; v[4 * i + 1] = x.y; v[4 * i + 2] = x.z; v[4 * i + 3] = x.w;
  }
}
__device__ __forceinline__ void load16(const __nv_bfloat16* p, float* v) {
  const uint4* q = reinterpret_cast<const uint4*>(p);
#pragma unroll
  for (int i = 0; i < 2; ++i) {
    uint4 x = q[i];
    const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&x);
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      float2 f = __bfloat1622float2(h[k]);
      v[8 * i + 2 * k] = f.x; v[8 * i + 2 * k + 1] = f.y;
    }
  }
}

// Two-term e4m3 form of (x0, x1): hi = e4m3(x), lo = e4m3(x - hi) (the
// difference is exact in fp32), both round-to-nearest-even and saturating;
// each pair packed with x0's code in the low byte.
__device__ __forceinline__ void split_e4m3x2(float x0, float x1, uint32_t& hi, uint32_t& lo) {
  const __nv_fp8x2_storage_t h = __nv_cvt_float2_to_fp8x2(make_float2(x0, x1), __NV_SATFINITE, __NV_E4M3);
  const float2 b = __half22float2(__half2(__nv_cvt_fp8x2_to_halfraw2(h, __NV_E4M3)));
  const __nv_fp8x2_storage_t l =
      __nv_cvt_float2_to_fp8x2(make_float2(x0 - b.x, x1 - b.y), __NV_SATFINITE, __NV_E4M3);
  hi = h;
  lo = l;
}

}  // namespace mla
