// Paged cache append: one warp writes one token's 576-number cache row (into
// the page-blocked layout: nine contiguous [64 rows x 64 columns] blocks per page).
//
// "KV Compression - DeepSeek-V3", "How it works": the 576-wide wkv_a output is
// split [512, 64]; the latent goes through RMSNorm and the rope part through
// RoPE; the absorb path stores the normalised latent and the rotated key.
// The kernel is memory-bound (2.3 KB in, 1.2 KB out per bf16 token); a warp
// moves a row with 16-byte accesses and reduces sum(c^2) with a fixed
// xor-shuffle tree.
#include "append_row.cuh"

namespace mla {
namespace {

template <typename IN, int CK>  // CK: MLA_F32, MLA_BF16, MLA_E4M3
__global__ void __launch_bounds__(256) append_kernel(AppendArgs a) {
  griddep_wait();
  griddep_launch_dependents();
  const int warp = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (warp >= a.n_new) return;
  const IN* row = reinterpret_cast<const IN*>(a.kv_a) + (size_t)warp * MLA_D_ROW;
  // latent: lane owns channels [16*lane, 16*lane + 16); rope key: pair `lane`
  float c[16];
  load16(row + 16 * lane, c);
  const float x0 = to_f32(row[MLA_D_C + 2 * lane]);
  const float x1 = to_f32(row[MLA_D_C + 2 * lane + 1]);
  append_row<CK>(a, a.seq_ids[warp], a.positions[warp], c, x0, x1, lane);
}

template <typename IN>
cudaError_t launch_in(const AppendArgs& a, cudaStream_t st) {
  dim3 block(256);
  dim3 grid((a.n_new + 7) / 8);
  switch (a.cache_dtype) {
    case MLA_F32: return launch_dependent(append_kernel<IN, MLA_F32>, grid, block, 0, st, a);
    case MLA_BF16: return launch_dependent(append_kernel<IN, MLA_BF16>, grid, block, 0, st, a);
    default: return launch_dependent(append_kernel<IN, MLA_E4M3>, grid, block, 0, st, a);
  }
}

}  // namespace

cudaError_t launch_append(const AppendArgs& a, cudaStream_t st) {
  if (a.n_new == 0) return cudaSuccess;
  if (a.kv_dtype == MLA_F32) return launch_in<float>(a, st);
  return launch_in<__nv_bfloat16>(a, st);
}

}  // namespace mla
