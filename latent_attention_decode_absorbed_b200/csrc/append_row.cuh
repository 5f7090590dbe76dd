// The cache-row writer shared by the append kernel and the fused projection
// kernel: one warp writes one token's 576-number cache row into the
// page-blocked pool ("KV Compression - DeepSeek-V3", "How it works": split
// [512, 64], RMSNorm on the latent, RoPE on the rope part).  The sum of
// squares uses a fixed xor-shuffle tree, the RoPE rotation separate
// fp32 roundings (no fused multiply-add), so the stored bits do not depend
// on which kernel calls it.
#pragma once

#include "mla_device.cuh"
#include "mla_internal.h"

namespace mla {

// c[16]: this lane's latent channels [16 lane, 16 lane + 16) as read;
// x0, x1: its rope pair (channels 512 + 2 lane, + 1).  s, p: the token's
// sequence and position.  CK: MLA_F32, MLA_BF16, MLA_E4M3.
template <int CK>
__device__ __forceinline__ void append_row(const AppendArgs& a, int s, int p, float* c, float x0, float x1,
                                           int lane) {
  if (s < 0 || s >= a.batch || p < 0 || p >= a.max_pages * a.page_size || p >= a.rope_max_pos) {
    if (lane == 0) flag_error(a.err, MLA_DEVERR_POSITION);
    return;
  }
  const int page = a.block_table[(size_t)s * a.max_pages + p / a.page_size];
  if (page < 0 || page >= a.num_pages) {
    if (lane == 0) flag_error(a.err, MLA_DEVERR_PAGE);
    return;
  }
  const size_t slot = (size_t)page * a.page_size + (p % a.page_size);
  float ss = 0.f;
#pragma unroll
  for (int i = 0; i < 16; ++i) ss = fmaf(c[i], c[i], ss);
  ss = warp_sum(ss);
  const float rms = sqrtf(ss * (1.0f / MLA_D_C) + a.eps);
  const float inv = 1.0f / rms;
#pragma unroll
  for (int i = 0; i < 16; ++i) {
    float g = a.gain ? a.gain[16 * lane + i] : 1.0f;
    c[i] = (c[i] * inv) * g;
  }
  const float cs = a.rope_cos[(size_t)p * (MLA_D_R / 2) + lane];
  const float sn = a.rope_sin[(size_t)p * (MLA_D_R / 2) + lane];
  const float r0 = __fsub_rn(__fmul_rn(x0, cs), __fmul_rn(x1, sn));
  const float r1 = __fadd_rn(__fmul_rn(x0, sn), __fmul_rn(x1, cs));
  if constexpr (CK == MLA_E4M3) {
    float am = fmaxf(fabsf(r0), fabsf(r1));
#pragma unroll
    for (int i = 0; i < 16; ++i) am = fmaxf(am, fabsf(c[i]));
    am = warp_max(am);
    const float q = am > 0.f ? 448.0f / am : 0.f;
    uint8_t* dst = reinterpret_cast<uint8_t*>(a.cache);
    uint32_t w[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      uint16_t lo = __nv_cvt_float2_to_fp8x2(make_float2(c[4 * i] * q, c[4 * i + 1] * q), __NV_SATFINITE, __NV_E4M3);
      uint16_t hi = __nv_cvt_float2_to_fp8x2(make_float2(c[4 * i + 2] * q, c[4 * i + 3] * q), __NV_SATFINITE, __NV_E4M3);
      w[i] = (uint32_t)lo | ((uint32_t)hi << 16);
    }
    *reinterpret_cast<uint4*>(dst + cache_index(slot, 16 * lane)) = make_uint4(w[0], w[1], w[2], w[3]);
    uint16_t rk = __nv_cvt_float2_to_fp8x2(make_float2(r0 * q, r1 * q), __NV_SATFINITE, __NV_E4M3);
    *reinterpret_cast<uint16_t*>(dst + cache_index(slot, MLA_D_C + 2 * lane)) = rk;
    if (lane == 0) a.cache_scale[slot] = am * (1.0f / 448.0f);
  } else if constexpr (CK == MLA_BF16) {
    __nv_bfloat16* dst = reinterpret_cast<__nv_bfloat16*>(a.cache);
    uint32_t w[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      __nv_bfloat162 h = __floats2bfloat162_rn(c[2 * i], c[2 * i + 1]);
      w[i] = *reinterpret_cast<uint32_t*>(&h);
    }
    uint4* d4 = reinterpret_cast<uint4*>(dst + cache_index(slot, 16 * lane));
    d4[0] = make_uint4(w[0], w[1], w[2], w[3]);
    d4[1] = make_uint4(w[4], w[5], w[6], w[7]);
    __nv_bfloat162 rk = __floats2bfloat162_rn(r0, r1);
    *reinterpret_cast<__nv_bfloat162*>(dst + cache_index(slot, MLA_D_C + 2 * lane)) = rk;
  } else {
    float* dst = reinterpret_cast<float*>(a.cache);
    float4* d4 = reinterpret_cast<float4*>(dst + cache_index(slot, 16 * lane));
#pragma unroll
    for (int i = 0; i < 4; ++i) d4[i] = make_float4(c[4 * i], c[4 * i + 1], c[4 * i + 2], c[4 * i + 3]);
    *reinterpret_cast<float2*>(dst + cache_index(slot, MLA_D_C + 2 * lane)) = make_float2(r0, r1);
  }
}

}  // namespace mla
