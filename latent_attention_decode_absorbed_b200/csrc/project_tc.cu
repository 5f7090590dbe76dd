// Per-head projections on the tcgen05 tensor cores (bf16 operands, fp32
// accumulation in TMEM).
//
//   absorb_q:  q_abs[r,h,0:512] = q_nope[r,h,:] . W_UK[h]   (K = 128, N = 512)
//              q_abs[r,h,512:]  = q_pe[r,h,:]
//   out_uv:    out[r,h,:]       = o_lat[r,h,:] . W_UV[h]^T  (K = 512, N = 128)
//
// "DeepSeek-V2: MLA Explained", "Optimization Note": W_UK is merged into the
// query and W_UV is applied after the attention-weighted sum of latents.  For
// each head this is a small GEMM with the query rows as M: one CTA per
// (head, 128-row tile, N half) loads the rows (TMA; rows past the end are
// zero-filled) and its half of the head's weight (TMA, 128-byte swizzle) in
// one go, one thread issues the MMAs (M = 128, cta_group::1), and the four
// warps read the accumulator back by rows (thread = row) and store bf16.
// With few rows the kernel streams each weight once (16.8 MB per projection
// at 128 heads); with many rows it is a dense GEMM on the tensor pipe.
#include "mla_device.cuh"
#include "mla_internal.h"
#include "sm100.cuh"

namespace mla {
namespace {

using namespace sm100;

constexpr int kPThreads = 128;

// one-CTA MMA (cta_group::1) and its commit
__device__ __forceinline__ void mma_f16_cta(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                            bool accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"((uint32_t)accumulate)
      : "memory");
}
__device__ __forceinline__ void mma_commit_cta(uint32_t bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar) : "memory");
}
__device__ __forceinline__ void tmem_alloc_cta(uint32_t dst_smem, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(dst_smem), "r"(ncols)
               : "memory");
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc_cta(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}

// KIND 0: absorb_q (A = q_nope rows, K = 128; B = W_UK[h] N-major, N half = 256)
// KIND 1: out_uv   (A = o_lat rows,  K = 512; B = W_UV[h] K-major, N half = 64)
template <int KIND>
struct Proj {
  static constexpr int K = KIND == 0 ? MLA_D_NOPE : MLA_D_C;
  static constexpr int NH = KIND == 0 ? MLA_D_C / 2 : MLA_D_V / 2;   // N per CTA
  static constexpr int KC = K / 64;                                  // 64-wide K chunks
  static constexpr int kABytes = KC * 128 * 128;                     // [128 rows x K] bf16
  static constexpr int kBBytes = K * NH * 2;
  // out_uv streams its eight K chunks (A [128 rows x 64] + B [64 N x 64]) through
  // a four-stage ring: 96 KB instead of 192 KB, so two CTAs fit on an SM and the
  // 256 CTAs of a 128-head step run in one wave; absorb_q (K = 128) loads at once
  static constexpr int kStages = KIND == 0 ? 1 : 4;
  static constexpr int kStageA = 128 * 128, kStageB = NH * 128, kStage = kStageA + kStageB;
  static constexpr int kOperands = KIND == 0 ? kABytes + kBBytes : kStages * kStage;
  static constexpr int kSmem = kOperands + 1024 + 128;
  static constexpr uint32_t kTmemCols = NH < 32 ? 32 : NH;
};

template <int KIND>
__global__ void __launch_bounds__(kPThreads, 1)
    proj_tc_kernel(const __grid_constant__ CUtensorMap tm_a, const __grid_constant__ CUtensorMap tm_b,
                   const __nv_bfloat16* __restrict__ q_pe, __nv_bfloat16* __restrict__ out, int rows, int H,
                   int32_t* err) {
  using P = Proj<KIND>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t s_a = smem_u32(smem), s_b = s_a + P::kABytes;
  uint8_t* misc = smem + P::kOperands;
  // barriers: full[kStages], empty[kStages], done; then the TMEM slot and the abort flag
  const uint32_t bar_full = smem_u32(misc), bar_empty = bar_full + 8 * P::kStages,
                 bar_done = bar_full + 16 * P::kStages, tslot = bar_done + 8;
  volatile int* abort_flag = reinterpret_cast<volatile int*>(misc + 16 * P::kStages + 12);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int h = blockIdx.x, m0 = blockIdx.y * 128, nh = blockIdx.z;

  if (threadIdx.x == 0) {
    for (int i = 0; i < P::kStages; ++i) {
      mbar_init(bar_full + 8 * i, 1);
      mbar_init(bar_empty + 8 * i, 1);
    }
    mbar_init(bar_done, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0) tmem_alloc_cta(tslot, P::kTmemCols);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *reinterpret_cast<volatile uint32_t*>(misc + 16 * P::kStages + 8);
  griddep_wait();
  griddep_launch_dependents();

  bool ok = true;
  if (threadIdx.x == 0 && KIND == 0) {
    mbar_arrive_expect_tx(bar_full, P::kABytes + P::kBBytes);
    for (int c = 0; c < P::KC; ++c)   // rows m0.., K chunk c: [128 rows x 64] (rows past the end read as 0)
      tma_load_3d(s_a + c * 128 * 128, &tm_a, 64 * c, h, m0, bar_full);
    // W_UK[h] as [128 K rows x 64 N] boxes, N-major: 4 blocks of 64 N
    for (int nb = 0; nb < P::NH / 64; ++nb)
      tma_load_3d(s_b + nb * (P::K * 128), &tm_b, P::NH * nh + 64 * nb, 0, h, bar_full);
    ok = mbar_wait<false>(bar_full, 0, abort_flag);
    if (ok) {
      tc_fence_after();
      constexpr uint32_t idesc = idesc_f16(128, P::NH, false, true);
      for (int c = 0; c < P::KC; ++c) {
#pragma unroll
        for (int ks = 0; ks < 4; ++ks) {
          const uint64_t ad = smem_desc_sw128(s_a + c * 128 * 128 + ks * 32, 16, 1024);
          // N-major: 8 K rows per 1 KB atom, 64-N blocks kK*128 bytes apart
          const uint64_t bd = smem_desc_sw128(s_b + (4 * c + ks) * 2048, P::K * 128, 1024);
          mma_f16_cta(tmem, ad, bd, idesc, (c | ks) != 0);
        }
      }
      mma_commit_cta(bar_done);
    } else {
      *abort_flag = 1;
    }
  } else if (threadIdx.x == 0) {
    // out_uv: stage c holds rows m0.. of K chunk c ([128 x 64], rows past the end read as 0)
    // and W_UV[h] rows (N) nh*64.. of K chunk c ([64 x 64], K-major)
    auto load = [&](int c) {
      const int slot = c % P::kStages;
      const uint32_t dst = s_a + slot * P::kStage;
      mbar_arrive_expect_tx(bar_full + 8 * slot, P::kStage);
      tma_load_3d(dst, &tm_a, 64 * c, h, m0, bar_full + 8 * slot);
      tma_load_3d(dst + P::kStageA, &tm_b, 64 * c, P::NH * nh, h, bar_full + 8 * slot);
    };
    for (int c = 0; c < P::kStages && c < P::KC; ++c) load(c);
    constexpr uint32_t idesc = idesc_f16(128, P::NH, false, false);
    for (int c = 0; c < P::KC && ok; ++c) {
      const int slot = c % P::kStages;
      const uint32_t ph = (c / P::kStages) & 1u;
      ok = mbar_wait<false>(bar_full + 8 * slot, ph, abort_flag);
      if (!ok) break;
      tc_fence_after();
      const uint32_t a0 = s_a + slot * P::kStage;
#pragma unroll
      for (int ks = 0; ks < 4; ++ks)
        mma_f16_cta(tmem, smem_desc_sw128(a0 + ks * 32, 16, 1024),
                    smem_desc_sw128(a0 + P::kStageA + ks * 32, 16, 1024), idesc, (c | ks) != 0);
      mma_commit_cta(bar_empty + 8 * slot);
      if (c + P::kStages < P::KC) {
        // the slot is reused once these MMAs have read it
        ok = mbar_wait<false>(bar_empty + 8 * slot, ph, abort_flag);
        if (ok) load(c + P::kStages);
      }
    }
    if (ok) mma_commit_cta(bar_done);
    else *abort_flag = 1;
  }
  __syncthreads();
  if (!*abort_flag) ok = __all_sync(0xffffffffu, mbar_wait<false>(bar_done, 0, abort_flag));
  else ok = false;
  if (ok) {
    tc_fence_after();
    const int row = m0 + 32 * warp + lane;
    const uint32_t taddr = tmem + (static_cast<uint32_t>(32 * warp) << 16);
#pragma unroll 1
    for (int n0 = 0; n0 < P::NH; n0 += 32) {
      float v[32];
      tmem_ld<32>(taddr + n0, v);
      tmem_wait_ld();
      if (row < rows) {
        __nv_bfloat16* dst = out + ((size_t)row * H + h) * (KIND == 0 ? MLA_D_ROW : MLA_D_V) + P::NH * nh + n0;
#pragma unroll
        for (int j = 0; j < 32; j += 8) {
          uint32_t w[4];
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const __nv_bfloat162 b2 = __floats2bfloat162_rn(v[j + 2 * e], v[j + 2 * e + 1]);
            w[e] = *reinterpret_cast<const uint32_t*>(&b2);
          }
          *reinterpret_cast<uint4*>(dst + j) = make_uint4(w[0], w[1], w[2], w[3]);
        }
      }
    }
    if (KIND == 0 && nh == 0 && row < rows) {   // q_pe passes through
      const uint4* src = reinterpret_cast<const uint4*>(q_pe + ((size_t)row * H + h) * MLA_D_R);
      uint4* dst = reinterpret_cast<uint4*>(out + ((size_t)row * H + h) * MLA_D_ROW + MLA_D_C);
#pragma unroll
      for (int j = 0; j < MLA_D_R / 8; ++j) dst[j] = src[j];
    }
  }
  if (threadIdx.x == 0 && *abort_flag) flag_error(err, MLA_DEVERR_TIMEOUT);
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc_cta(tmem, P::kTmemCols);
  }
}

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);
EncodeTiledFn encode_fn_p() {
  static EncodeTiledFn fn = nullptr;
  static bool tried = false;
  if (!tried) {
    tried = true;
    void* f = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(f);
  }
  return fn;
}

// 3-D bf16 tensor map, 128-byte swizzle
bool map3(EncodeTiledFn enc, CUtensorMap* m, const void* base, cuuint64_t d0, cuuint64_t d1, cuuint64_t d2,
          cuuint32_t b0, cuuint32_t b1, cuuint32_t b2) {
  cuuint64_t dims[3] = {d0, d1, d2};
  cuuint64_t strides[2] = {d0 * 2, d0 * d1 * 2};
  cuuint32_t box[3] = {b0, b1, b2};
  cuuint32_t es[3] = {1, 1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, es,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int KIND>
cudaError_t launch_kind(const CUtensorMap& ta, const CUtensorMap& tb, const void* q_pe, void* out, int rows, int H,
                        int32_t* err, cudaStream_t st) {
  using P = Proj<KIND>;
  cudaError_t e = cudaFuncSetAttribute(proj_tc_kernel<KIND>, cudaFuncAttributeMaxDynamicSharedMemorySize, P::kSmem);
  if (e != cudaSuccess) return e;
  dim3 grid(H, (rows + 127) / 128, 2);
  return launch_dependent(proj_tc_kernel<KIND>, grid, dim3(kPThreads), P::kSmem, st, ta, tb,
                          static_cast<const __nv_bfloat16*>(q_pe), static_cast<__nv_bfloat16*>(out), rows, H, err);
}

}  // namespace

cudaError_t launch_absorb_q_tc(const void* q_nope, const void* q_pe, const void* w_uk, void* q_abs, int rows,
                               int n_heads, cudaStream_t st) {
  if (rows == 0) return cudaSuccess;
  EncodeTiledFn enc = encode_fn_p();
  if (!enc) return cudaErrorNotSupported;
  CUtensorMap ta, tb;
  // q_nope [rows, H, 128]: boxes [128 rows x 64]; W_UK [H, 128, 512]: boxes [128 K x 64 N]
  if (!map3(enc, &ta, q_nope, MLA_D_NOPE, n_heads, rows, 64, 1, 128) ||
      !map3(enc, &tb, w_uk, MLA_D_C, MLA_D_NOPE, n_heads, 64, 128, 1))
    return cudaErrorInvalidValue;
  return launch_kind<0>(ta, tb, q_pe, q_abs, rows, n_heads, nullptr, st);
}

cudaError_t launch_out_uv_tc(const void* o_lat, const void* w_uv, void* out, int rows, int n_heads, cudaStream_t st) {
  if (rows == 0) return cudaSuccess;
  EncodeTiledFn enc = encode_fn_p();
  if (!enc) return cudaErrorNotSupported;
  CUtensorMap ta, tb;
  // o_lat [rows, H, 512]: boxes [128 rows x 64]; W_UV [H, 128, 512]: boxes [64 N x 64 K]
  if (!map3(enc, &ta, o_lat, MLA_D_C, n_heads, rows, 64, 1, 128) ||
      !map3(enc, &tb, w_uv, MLA_D_C, MLA_D_V, n_heads, 64, 64, 1))
    return cudaErrorInvalidValue;
  return launch_kind<1>(ta, tb, nullptr, out, rows, n_heads, nullptr, st);
}

}  // namespace mla
