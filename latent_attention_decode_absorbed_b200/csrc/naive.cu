// The non-absorbed ("level 2") decode path, kept to be measured against the
// absorbed one: per-head keys and values are decompressed from the cached
// latents at every step, then attention runs per head in the standard form.
//
// "HuggingFace version does NOT use efficient MLA caching" lists the ways MLA
// inference can be run; level 2 caches the latent but projects it back up to
// per-head K and V before attending.  "DeepSeek-V2: MLA Explained", "MLA Full
// Formulas" parts 2 and 3:
//   k^C_{j,i} = W^UK_i c_j,  v^C_{j,i} = W^UV_i c_j,  k_{j,i} = [k^C_{j,i}; k^R_j]
//   o_{t,i}   = sum_j softmax_j(q_{t,i} . k_{j,i} / sqrt(128 + 64)) v^C_{j,i}
// with q_{t,i} = [q^C_{t,i}; q^R_{t,i}] (not absorbed).  Per cached row and
// 128 heads that is 64 KB of bf16 keys and values written and read again,
// against the 1152-byte row the absorbed path reads.
//
// decompress_kernel: one tcgen05 GEMM tile per (page pair, head, K or V):
//   D[128 rows x 128] = C[128 rows x 512] . W[h][128 x 512]^T
// A = the two pages' latent blocks (the cache's own 128-byte swizzled boxes),
// B = the head's weight rows, both K-major, a four-stage TMA ring over the
// eight 64-wide K steps; the accumulator is read back by rows and stored bf16.
//
// attend_naive_kernel: CUDA cores, one CTA per (query row, head); sixteen
// warps take interleaved chunks of eight visible rows (lane l holds elements
// 4l..4l+3 of the 128-wide key and value, 2l..2l+1 of the rope key), keep a
// running max and sum, and merge through shared memory at the end.
#include <math.h>

#include "mla_device.cuh"
#include "mla_internal.h"
#include "sm100.cuh"

namespace mla {
namespace {

using namespace sm100;

constexpr int kDThreads = 128;
constexpr int kDStages = 4;
constexpr int kDBox = 8192;                       // [64 rows x 64] bf16
constexpr int kDStage = 4 * kDBox;                // A: two page blocks, B: [128 x 64]
constexpr int kDMisc = kDStages * kDStage;
constexpr int kDSmem = kDMisc + 256 + 1024;
constexpr int kDK = MLA_D_C / 64;                 // eight K steps

__device__ __forceinline__ void mma1_w(uint32_t d, uint64_t a, uint64_t b, uint32_t idesc, uint32_t acc) {
  asm volatile(
      "{\n\t.reg .pred p, e;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "elect.sync _|e, 0xffffffff;\n\t"
      "@e tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d),
      "l"(a), "l"(b), "r"(idesc), "r"(acc)
      : "memory");
}
__device__ __forceinline__ void commit1_w(uint32_t bar) {
  asm volatile(
      "{\n\t.reg .pred e;\n\t"
      "elect.sync _|e, 0xffffffff;\n\t"
      "@e tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];\n\t}" ::"r"(bar)
      : "memory");
}

__device__ __forceinline__ void tmem_alloc1(uint32_t dst_smem, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(dst_smem), "r"(ncols)
               : "memory");
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc1(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}

struct DecompParams {
  int num_pages, H;
  __nv_bfloat16* k_c;             // [num_pages, 64, H, 128]
  __nv_bfloat16* v_c;
  unsigned long long wait_limit;
  int32_t* err;
};

__global__ void __launch_bounds__(kDThreads, 1)
    decompress_kernel(const __grid_constant__ CUtensorMap tm_cache, const __grid_constant__ CUtensorMap tm_wk,
                      const __grid_constant__ CUtensorMap tm_wv, const DecompParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t s_base = smem_u32(smem);
  uint8_t* misc = smem + kDMisc;
  const uint32_t s_misc = s_base + kDMisc;
  auto bar = [&](int i) -> uint32_t { return s_misc + 8 * i; };   // full[4], empty[4], done
  volatile int* abort_flag = reinterpret_cast<volatile int*>(misc + 80);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint64_t lim = p.wait_limit;
  const int pg0 = 2 * blockIdx.x;
  const int pg1 = min(pg0 + 1, p.num_pages - 1);  // an odd pool's last tile loads page pg0 twice
  const int h = blockIdx.y;
  const bool vals = blockIdx.z != 0;

  if (threadIdx.x == 0) {
    for (int i = 0; i < kDStages; ++i) {
      mbar_init(bar(i), 1);
      mbar_init(bar(kDStages + i), 1);
    }
    mbar_init(bar(2 * kDStages), 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0) tmem_alloc1(s_misc + 72, 128);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *reinterpret_cast<volatile uint32_t*>(misc + 72);

  if (warp == 0) {
    // ---- TMA producer: latent block c of both pages, and the weight's K step c
    if (lane == 0) {
      const CUtensorMap* tw = vals ? &tm_wv : &tm_wk;
      tma_prefetch_desc(&tm_cache);
      tma_prefetch_desc(tw);
      for (int c = 0; c < kDK; ++c) {
        const int s = c % kDStages;
        if (c >= kDStages && !mbar_wait<false>(bar(kDStages + s), ((c / kDStages) - 1) & 1, abort_flag, lim)) break;
        mbar_arrive_expect_tx(bar(s), kDStage);
        const uint32_t dst = s_base + s * kDStage;
        tma_load_2d(dst, &tm_cache, 0, (pg0 * 9 + c) * 64, bar(s));
        tma_load_2d(dst + kDBox, &tm_cache, 0, (pg1 * 9 + c) * 64, bar(s));
        tma_load_2d(dst + 2 * kDBox, tw, 64 * c, 128 * h, bar(s));
      }
    }
  } else if (warp == 1) {
    // ---- MMA issuer: M = 128 rows, N = 128 outputs, K = 16 per MMA
    constexpr uint32_t id = idesc_f16(128, 128, false, false);
    for (int c = 0; c < kDK; ++c) {
      const int s = c % kDStages;
      if (!__all_sync(0xffffffffu, mbar_wait<false>(bar(s), (c / kDStages) & 1, abort_flag, lim))) break;
      tc_fence_after();
      const uint32_t a0 = s_base + s * kDStage;
      const uint64_t ad = smem_desc_sw128(a0, 16, 1024), bd = smem_desc_sw128(a0 + 2 * kDBox, 16, 1024);
#pragma unroll
      for (int ks = 0; ks < 4; ++ks) mma1_w(tmem, ad + 2 * ks, bd + 2 * ks, id, (c | ks) != 0);
      commit1_w(bar(kDStages + s));
    }
    commit1_w(bar(2 * kDStages));
  }
  // ---- epilogue (all four warps): thread = tile row, 128 outputs stored bf16
  const bool ok = __all_sync(0xffffffffu, mbar_wait<false>(bar(2 * kDStages), 0, abort_flag, lim) && !*abort_flag);
  tc_fence_after();
  const int m = 32 * warp + lane;
  const int page = pg0 + (m >> 6);
  if (ok) {
    __nv_bfloat16* dst = (vals ? p.v_c : p.k_c) + (((size_t)page * 64 + (m & 63)) * p.H + h) * MLA_D_NOPE;
    const uint32_t taddr = tmem + (static_cast<uint32_t>(32 * warp) << 16);
#pragma unroll 1
    for (int c4 = 0; c4 < 4; ++c4) {
      float v[32];
      tmem_ld<32>(taddr + 32 * c4, v);
      tmem_wait_ld();
      if (page < p.num_pages) {
        uint4* d4 = reinterpret_cast<uint4*>(dst + 32 * c4);
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          uint32_t w[4];
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const __nv_bfloat162 x = __floats2bfloat162_rn(v[8 * q + 2 * e], v[8 * q + 2 * e + 1]);
            w[e] = *reinterpret_cast<const uint32_t*>(&x);
          }
          d4[q] = make_uint4(w[0], w[1], w[2], w[3]);
        }
      }
    }
  } else if (threadIdx.x == 0) {
    flag_error(p.err, MLA_DEVERR_TIMEOUT);
  }
  if (*abort_flag) {
    // let copies and MMAs already in flight land before the memory is released
    const uint64_t t0 = globaltimer();
    while (globaltimer() - t0 < 2000000ull) {
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc1(tmem, 128);
  }
}

// ------------------------------------------------------------------ attention
constexpr int kAWarps = 16;
constexpr int kAChunk = 8;                         // rows per warp step

struct NaiveParams {
  const __nv_bfloat16* q_nope;   // [rows, H, 128]
  const __nv_bfloat16* q_pe;     // [rows, H, 64]
  const __nv_bfloat16* cache;    // [num_pages, 9, 64, 64]: the rope keys (block 8)
  const __nv_bfloat16* k_c;      // [num_pages, 64, H, 128]
  const __nv_bfloat16* v_c;
  int num_pages;
  const int32_t* block_table;
  int max_pages;
  const int32_t* seq_lens;
  int q_len, H;
  float scale_log2;              // softmax_scale * log2(e)
  __nv_bfloat16* out;            // [rows, H, 128]
  float* lse;                    // [rows, H] or null
  int32_t* err;
};

__device__ __forceinline__ void bf16x4(uint2 u, float* f) {
  const float2 a = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&u.x));
  const float2 b = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&u.y));
  f[0] = a.x; f[1] = a.y; f[2] = b.x; f[3] = b.y;
}

__global__ void __launch_bounds__(32 * kAWarps) attend_naive_kernel(const NaiveParams p) {
  __shared__ float s_m[kAWarps], s_l[kAWarps];
  __shared__ float s_o[kAWarps][MLA_D_V];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int r = blockIdx.x, h = blockIdx.y;
  const int b = r / p.q_len, t = r % p.q_len;
  const int n_vis = p.seq_lens[b] - p.q_len + t + 1;
  float qn[4], qp[2];
  bf16x4(*reinterpret_cast<const uint2*>(p.q_nope + ((size_t)r * p.H + h) * MLA_D_NOPE + 4 * lane), qn);
  {
    const float2 x = __bfloat1622float2(
        *reinterpret_cast<const __nv_bfloat162*>(p.q_pe + ((size_t)r * p.H + h) * MLA_D_R + 2 * lane));
    qp[0] = x.x; qp[1] = x.y;
  }
  float m = -INFINITY, l = 0.f, o[4] = {0.f, 0.f, 0.f, 0.f};
  for (int j0 = kAChunk * warp; j0 < n_vis; j0 += kAChunk * kAWarps) {
    // the chunk's rows share one page (j0 is a multiple of 8)
    const int pidx = j0 >> 6;
    int pg = pidx < p.max_pages ? p.block_table[(size_t)b * p.max_pages + pidx] : -1;
    const bool pok = pg >= 0 && pg < p.num_pages;
    if (!pok) {
      if (lane == 0) flag_error(p.err, MLA_DEVERR_PAGE);
      pg = 0;
    }
    uint2 kc[kAChunk], vc[kAChunk];
    uint32_t kr[kAChunk];
#pragma unroll
    for (int k = 0; k < kAChunk; ++k) {
      const int row = (j0 + k) & 63;
      const size_t kv = (((size_t)pg * 64 + row) * p.H + h) * MLA_D_NOPE + 4 * lane;
      kc[k] = *reinterpret_cast<const uint2*>(p.k_c + kv);
      vc[k] = *reinterpret_cast<const uint2*>(p.v_c + kv);
      kr[k] = *reinterpret_cast<const uint32_t*>(p.cache + ((size_t)pg * 9 + 8) * 4096 + row * 64 + 2 * lane);
    }
    float s[kAChunk];
#pragma unroll
    for (int k = 0; k < kAChunk; ++k) {
      float f[4];
      bf16x4(kc[k], f);
      const float2 e = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&kr[k]));
      s[k] = qn[0] * f[0] + qn[1] * f[1] + qn[2] * f[2] + qn[3] * f[3] + qp[0] * e.x + qp[1] * e.y;
    }
#pragma unroll
    for (int k = 0; k < kAChunk; ++k) s[k] = warp_sum(s[k]);
    float mc = -INFINITY;
#pragma unroll
    for (int k = 0; k < kAChunk; ++k) {
      s[k] = (pok && j0 + k < n_vis) ? s[k] * p.scale_log2 : -INFINITY;
      mc = fmaxf(mc, s[k]);
    }
    const float m_new = fmaxf(m, mc);
    if (m_new == -INFINITY) continue;
    const float alpha = exp2f(m - m_new);        // 0 while nothing was kept (m = -inf)
    l *= alpha;
#pragma unroll
    for (int e = 0; e < 4; ++e) o[e] *= alpha;
#pragma unroll
    for (int k = 0; k < kAChunk; ++k) {
      const float pk = exp2f(s[k] - m_new);
      float f[4];
      bf16x4(vc[k], f);
      l += pk;
#pragma unroll
      for (int e = 0; e < 4; ++e) o[e] = fmaf(pk, f[e], o[e]);
    }
    m = m_new;
  }
  if (lane == 0) {
    s_m[warp] = m;
    s_l[warp] = l;
  }
#pragma unroll
  for (int e = 0; e < 4; ++e) s_o[warp][4 * lane + e] = o[e];
  __syncthreads();
  if (threadIdx.x < MLA_D_V) {
    float mm = -INFINITY;
#pragma unroll
    for (int w = 0; w < kAWarps; ++w) mm = fmaxf(mm, s_m[w]);
    float lt = 0.f, acc = 0.f;
    if (mm != -INFINITY) {
#pragma unroll
      for (int w = 0; w < kAWarps; ++w) {
        const float f = exp2f(s_m[w] - mm);      // 0 for a warp that kept nothing
        lt += f * s_l[w];
        acc += f * s_o[w][threadIdx.x];
      }
    }
    const float v = lt > 0.f ? acc / lt : 0.f;
    p.out[((size_t)r * p.H + h) * MLA_D_V + threadIdx.x] = __float2bfloat16_rn(v);
    if (p.lse && threadIdx.x == 0)
      p.lse[(size_t)r * p.H + h] = lt > 0.f ? (mm + log2f(lt)) * 0.69314718055994531f : -INFINITY;
  }
}

}  // namespace

cudaError_t launch_decompress_kv(const void* cache, int num_pages, const void* w_uk, const void* w_uv, int n_heads,
                                 void* k_c, void* v_c, int32_t* err, cudaStream_t st) {
  if (num_pages == 0) return cudaSuccess;
  TensorMapEncodeFn enc = tensor_map_encoder();
  if (!enc) return cudaErrorNotSupported;
  CUtensorMap tc, tk, tv;
  {
    // the page-blocked pool as 2-D [num_pages * 9 * 64 lines x 64 columns]: boxes of one block
    cuuint64_t dims[2] = {64, (cuuint64_t)num_pages * 9 * 64};
    cuuint64_t strides[1] = {128};
    cuuint32_t box[2] = {64, 64};
    cuuint32_t es[2] = {1, 1};
    if (enc(&tc, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(cache), dims, strides, box, es,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return cudaErrorInvalidValue;
  }
  for (int k = 0; k < 2; ++k) {
    // W [H * 128 rows x 512]: boxes of 64 columns x one head's 128 rows
    cuuint64_t dims[2] = {MLA_D_C, (cuuint64_t)n_heads * 128};
    cuuint64_t strides[1] = {MLA_D_C * 2};
    cuuint32_t box[2] = {64, 128};
    cuuint32_t es[2] = {1, 1};
    if (enc(k == 0 ? &tk : &tv, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(k == 0 ? w_uk : w_uv), dims,
            strides, box, es, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return cudaErrorInvalidValue;
  }
  cudaError_t e = cudaFuncSetAttribute(decompress_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kDSmem);
  if (e != cudaSuccess) return e;
  DecompParams p{num_pages, n_heads, static_cast<__nv_bfloat16*>(k_c), static_cast<__nv_bfloat16*>(v_c),
                 g_wait_limit.load(), err};
  decompress_kernel<<<dim3((unsigned)((num_pages + 1) / 2), (unsigned)n_heads, 2), kDThreads, kDSmem, st>>>(tc, tk,
                                                                                                          tv, p);
  return cudaGetLastError();
}

cudaError_t launch_attend_naive(const NaiveArgs& a, cudaStream_t st) {
  const int rows = a.batch * a.q_len;
  if (rows == 0) return cudaSuccess;
  NaiveParams p{static_cast<const __nv_bfloat16*>(a.q_nope), static_cast<const __nv_bfloat16*>(a.q_pe),
                static_cast<const __nv_bfloat16*>(a.cache), static_cast<const __nv_bfloat16*>(a.k_c),
                static_cast<const __nv_bfloat16*>(a.v_c), a.num_pages, a.block_table, a.max_pages, a.seq_lens,
                a.q_len, a.n_heads, a.softmax_scale * 1.4426950408889634f, static_cast<__nv_bfloat16*>(a.out),
                a.lse, a.err};
  attend_naive_kernel<<<dim3((unsigned)rows, (unsigned)a.n_heads), 32 * kAWarps, 0, st>>>(p);
  return cudaGetLastError();
}

}  // namespace mla
