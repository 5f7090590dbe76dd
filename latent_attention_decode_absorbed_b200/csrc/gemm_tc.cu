// Split-K GEMM on the tcgen05 tensor cores for the projections on either
// side of the attention core, with bf16 operands and fp32 accumulation:
//
//   C[M x N] += A[M x K] . B[N x K]^T            (A, B row-major, K contiguous)
//
//   mla_out_proj        u = [o_1; ...; o_H] . W_O^T   ("DeepSeek-V2: MLA Explained",
//                       "MLA Full Formulas" part 3: concatenate all heads and project)
//   mla_kv_proj_append  kv_a = h . W_kv,a^T, then the cache rows of kv_a
//                       ("KV Compression - DeepSeek-V3", "How it works", Eq. (1):
//                       the 576-wide joint down-projection feeding the cache)
//
// Decode-time M (tokens) is small and the weights are large, so the GEMMs
// are bound by streaming the weight once: a CTA computes one [128 x BN] tile
// over one K range (the grid splits K until it covers the SMs), streams its
// A and B slices through a four-stage TMA ring, accumulates in TMEM, and adds
// its fp32 tile into C with vector reductions.  For the wkv_a projection the
// last CTA to finish an M tile then writes that tile's cache rows from the
// reduced fp32 rows with the same row writer as mla_cache_append (RMSNorm,
// RoPE, cast or e4m3 quantisation, page scatter), so one kernel goes from the
// hidden states to the cache.
#include "append_row.cuh"
#include "mla_device.cuh"
#include "mla_internal.h"
#include "sm100.cuh"

namespace mla {
namespace {

using namespace sm100;

constexpr int kGThreads = 128;
constexpr int kGStages = 4;
constexpr int kBM = 128;
constexpr int kBK = 64;                  // one 128-byte line of bf16 per row per stage

__device__ __forceinline__ void mma1_f16_w(uint32_t d, uint64_t a, uint64_t b, uint32_t idesc, uint32_t acc) {
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
// c[0..3] += v (fp32, one 16-byte vector reduction in L2)
__device__ __forceinline__ void red_add_v4(float* c, float a, float b, float d, float e) {
  asm volatile("red.global.add.v4.f32 [%0], {%1, %2, %3, %4};" ::"l"(c), "f"(a), "f"(b), "f"(d), "f"(e) : "memory");
}

struct GemmParams {
  int M, N, K, kchunk;        // K range of one CTA: [blockIdx.z * kchunk, + kchunk)
  float* C;                   // [M, N] fp32, row stride N
  unsigned* tile_done;        // APPEND: one counter per M tile (zero at launch)
  int ctas_per_mtile;         // APPEND: gridDim.x * gridDim.z
  int cache_dtype;            // APPEND: MLA_F32 / MLA_BF16 / MLA_E4M3
  unsigned long long wait_limit;
  int32_t* err;
};

template <int BN>
struct GemmLayout {
  static constexpr int kABytes = kBM * 128;            // [128 rows x 64] bf16
  static constexpr int kBBytes = BN * 128;             // [BN rows x 64] bf16
  static constexpr int kStage = kABytes + kBBytes;
  static constexpr int kMisc = kGStages * kStage;       // barriers, TMEM slot, flags
  static constexpr int kSmem = kMisc + 256 + 1024;
  static constexpr uint32_t kTmemCols = 256;
  static_assert(kSmem <= 227 * 1024, "shared memory budget");
};

template <int BN, bool APPEND>
__global__ void __launch_bounds__(kGThreads, 1)
    gemm_splitk_kernel(const __grid_constant__ CUtensorMap tm_a, const __grid_constant__ CUtensorMap tm_b,
                       const GemmParams p, const AppendArgs app) {
  using LY = GemmLayout<BN>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t s_base = smem_u32(smem);
  uint8_t* misc = smem + LY::kMisc;
  const uint32_t s_misc = s_base + LY::kMisc;
  auto bar = [&](int i) -> uint32_t { return s_misc + 8 * i; };   // full[4], empty[4], done
  volatile int* abort_flag = reinterpret_cast<volatile int*>(misc + 80);
  volatile int* last_flag = reinterpret_cast<volatile int*>(misc + 84);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint64_t lim = p.wait_limit;
  const int n0 = blockIdx.x * BN, m0 = blockIdx.y * kBM, k0 = blockIdx.z * p.kchunk;
  const int nk = p.kchunk / kBK;

  if (threadIdx.x == 0) {
    for (int i = 0; i < kGStages; ++i) {
      mbar_init(bar(i), 1);
      mbar_init(bar(kGStages + i), 1);
    }
    mbar_init(bar(2 * kGStages), 1);
    *abort_flag = 0;
    *last_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0) tmem_alloc1(s_misc + 72, LY::kTmemCols);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *reinterpret_cast<volatile uint32_t*>(misc + 72);

  if (warp == 0) {
    // ---- TMA producer: A [128 rows x 64] and B [BN rows x 64] per stage
    if (lane == 0) {
      tma_prefetch_desc(&tm_a);
      tma_prefetch_desc(&tm_b);
      for (int k = 0; k < nk; ++k) {
        const int s = k % kGStages;
        if (k >= kGStages && !mbar_wait<false>(bar(kGStages + s), ((k / kGStages) - 1) & 1, abort_flag, lim)) break;
        mbar_arrive_expect_tx(bar(s), LY::kStage);
        const uint32_t dst = s_base + s * LY::kStage;
        tma_load_2d(dst, &tm_a, k0 + k * kBK, m0, bar(s));
        tma_load_2d(dst + LY::kABytes, &tm_b, k0 + k * kBK, n0, bar(s));
      }
    }
  } else if (warp == 1) {
    // ---- MMA issuer (whole warp, one elected lane): M = 128, N = BN, K = 16
    constexpr uint32_t id = idesc_f16(kBM, BN, false, false);
    for (int k = 0; k < nk; ++k) {
      const int s = k % kGStages;
      if (!__all_sync(0xffffffffu, mbar_wait<false>(bar(s), (k / kGStages) & 1, abort_flag, lim))) break;
      tc_fence_after();
      const uint32_t a0 = s_base + s * LY::kStage;
      const uint64_t ad = smem_desc_sw128(a0, 16, 1024), bd = smem_desc_sw128(a0 + LY::kABytes, 16, 1024);
#pragma unroll
      for (int ks = 0; ks < 4; ++ks) mma1_f16_w(tmem, ad + 2 * ks, bd + 2 * ks, id, (k | ks) != 0);
      commit1_w(bar(kGStages + s));
    }
    commit1_w(bar(2 * kGStages));
  }
  // ---- epilogue (all four warps): thread = row, add the fp32 tile into C
  const bool ok = __all_sync(0xffffffffu, mbar_wait<false>(bar(2 * kGStages), 0, abort_flag, lim) && !*abort_flag);
  tc_fence_after();
  if (ok) {
    const int row = m0 + 32 * warp + lane;
    const uint32_t taddr = tmem + (static_cast<uint32_t>(32 * warp) << 16);
#pragma unroll 1
    for (int c = 0; c < BN; c += 32) {
      float v[32];
      tmem_ld<32>(taddr + c, v);
      tmem_wait_ld();
      if (row < p.M) {
        float* dst = p.C + (size_t)row * p.N + n0 + c;
#pragma unroll
        for (int j = 0; j < 8; ++j) red_add_v4(dst + 4 * j, v[4 * j], v[4 * j + 1], v[4 * j + 2], v[4 * j + 3]);
      }
    }
  } else if (threadIdx.x == 0) {
    flag_error(p.err, MLA_DEVERR_TIMEOUT);
  }
  if constexpr (APPEND) {
    // the last CTA of this M tile writes its tokens' cache rows from the
    // fully reduced fp32 kv_a rows
    __threadfence();
    __syncthreads();
    if (threadIdx.x == 0) {
      const unsigned prev = atomicAdd(p.tile_done + blockIdx.y, 1u);
      *last_flag = (prev == (unsigned)(p.ctas_per_mtile - 1)) ? 1 : 0;
    }
    __syncthreads();
    if (*last_flag && ok) {
      __threadfence();
      const int m_end = min(m0 + kBM, p.M);
      for (int tok = m0 + warp; tok < m_end; tok += kGThreads / 32) {
        const float* rowp = p.C + (size_t)tok * MLA_D_ROW;
        float c[16];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const float4 x = __ldcg(reinterpret_cast<const float4*>(rowp + 16 * lane) + i);
          c[4 * i] = x.x; c[4 * i + 1] = x.y; c[4 * i + 2] = x.z; c[4 * i + 3] = x.w;
        }
        const float2 r = __ldcg(reinterpret_cast<const float2*>(rowp + MLA_D_C + 2 * lane));
        const int sq = app.seq_ids[tok], pos = app.positions[tok];
        if (p.cache_dtype == MLA_E4M3) append_row<MLA_E4M3>(app, sq, pos, c, r.x, r.y, lane);
        else if (p.cache_dtype == MLA_BF16) append_row<MLA_BF16>(app, sq, pos, c, r.x, r.y, lane);
        else append_row<MLA_F32>(app, sq, pos, c, r.x, r.y, lane);
      }
    }
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
    tmem_dealloc1(tmem, LY::kTmemCols);
  }
}

// Largest divisor of n that is at most cap (n >= 1).
int largest_divisor_at_most(int n, int cap) {
  for (int d = cap < n ? cap : n; d > 1; --d)
    if (n % d == 0) return d;
  return 1;
}

template <int BN, bool APPEND>
cudaError_t launch_gemm(const void* A, const void* B, int M, int N, int K, float* C, unsigned* tile_done,
                        int cache_dtype, const AppendArgs& app, int32_t* err, cudaStream_t st) {
  using LY = GemmLayout<BN>;
  TensorMapEncodeFn enc = tensor_map_encoder();
  if (!enc) return cudaErrorNotSupported;
  CUtensorMap ta, tb;
  {
    cuuint64_t dims[2] = {(cuuint64_t)K, (cuuint64_t)M};
    cuuint64_t strides[1] = {(cuuint64_t)K * 2};
    cuuint32_t box[2] = {kBK, kBM};
    cuuint32_t es[2] = {1, 1};
    if (enc(&ta, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(A), dims, strides, box, es,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return cudaErrorInvalidValue;
  }
  {
    cuuint64_t dims[2] = {(cuuint64_t)K, (cuuint64_t)N};
    cuuint64_t strides[1] = {(cuuint64_t)K * 2};
    cuuint32_t box[2] = {kBK, (cuuint32_t)BN};
    cuuint32_t es[2] = {1, 1};
    if (enc(&tb, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(B), dims, strides, box, es,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return cudaErrorInvalidValue;
  }
  const int mtiles = (M + kBM - 1) / kBM, ntiles = N / BN;
  // split K until the grid covers the SMs (each split a whole number of 64-wide steps)
  int sms = 148, dev = 0;
  if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const int want = (sms + mtiles * ntiles - 1) / (mtiles * ntiles);
  const int ks = largest_divisor_at_most(K / kBK, want < 1 ? 1 : want);
  GemmParams p{M, N, K, K / ks, C, tile_done, ntiles * ks, cache_dtype, g_wait_limit.load(), err};
  cudaError_t e = cudaFuncSetAttribute(gemm_splitk_kernel<BN, APPEND>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       LY::kSmem);
  if (e != cudaSuccess) return e;
  gemm_splitk_kernel<BN, APPEND><<<dim3(ntiles, mtiles, ks), kGThreads, LY::kSmem, st>>>(ta, tb, p, app);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_out_proj(const void* out_heads, const void* w_o, float* u, int rows, int n_heads, int d_model,
                            cudaStream_t st) {
  cudaError_t e = cudaMemsetAsync(u, 0, (size_t)rows * d_model * sizeof(float), st);
  if (e != cudaSuccess) return e;
  AppendArgs none{};
  return launch_gemm<256, false>(out_heads, w_o, rows, d_model, n_heads * MLA_D_V, u, nullptr, 0, none, nullptr, st);
}

cudaError_t launch_kv_proj_append(const void* h, const void* w_kva, int d_model, float* workspace,
                                  const AppendArgs& a, cudaStream_t st) {
  const size_t kv_bytes = (size_t)a.n_new * MLA_D_ROW * sizeof(float);
  const int mtiles = (a.n_new + kBM - 1) / kBM;
  cudaError_t e = cudaMemsetAsync(workspace, 0, kv_bytes + (size_t)mtiles * sizeof(unsigned), st);
  if (e != cudaSuccess) return e;
  unsigned* counters = reinterpret_cast<unsigned*>(reinterpret_cast<uint8_t*>(workspace) + kv_bytes);
  return launch_gemm<192, true>(h, w_kva, a.n_new, MLA_D_ROW, d_model, workspace, counters, a.cache_dtype, a,
                                a.err, st);
}

}  // namespace mla
