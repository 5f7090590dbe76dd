// Split-KV latent attention on the tcgen05 tensor cores (fp32 accumulation):
// CTA pairs, each working through (query row, split) units.
//
// What it computes ("DeepSeek-V2: MLA Explained", "MLA Full Formulas" part 3
// with the absorption of "Optimization Note"): for each head h of query row
// r and each cached row j of the split that the query sees,
//   z_j = scale * (q_abs[r,h,0:512] . c_j + q_abs[r,h,512:576] . k_j)
// then the split's normalised softmax-weighted mean of the latents c_j and
// its log-normaliser.
//
// How.  All heads share the cached rows, so the two contractions are dense
// GEMMs per tile of 256 rows, computed transposed so that neither the
// [heads x 576] query nor the [heads x 512] fp32 accumulator has to fit one
// SM:
//   S^T[256 rows x H]  = K[256 x 576] . Q[H x 576]^T        (cta_group::2, M=256)
//   O^T[512 dims x H] += V^T[512 x 256] . P^T[H x 256]^T    (two M=256 MMAs)
// CTA r of the pair holds rows [128r, 128r+128) of each tile for S^T, half of
// the heads of Q and of P^T (the split B operand), and dims
// {[128r,128r+128), [256+128r, 256+128r+128)} of O^T in its TMEM.  TMEM per
// CTA: two S^T buffers (2 x 128 columns) + O^T (2 x 128 columns) = 512.
//
// Cache rows stream through a ring of 32 KB shared-memory stages filled by
// TMA (128-byte swizzle) in the order the MMA consumes them.  A stage costs a
// fixed handshake (barrier wait, expected-bytes post, commit) whatever its
// size, and 16 KB stages cannot keep up with HBM, so a stage carries two
// column chunks of the score operand (four 8 KB boxes: [128 rows x 64
// columns] K-major per chunk, one box per page, issued by four lanes) or one
// page of the value operand (two 16 KB boxes: [64 rows x this CTA's 128 dims]
// read MN-major, one per dims block); the value loads of the peer's rows hit
// L2 (score loads are evict-last, value loads evict-first).  The pool is
// page-blocked, so every box is a contiguous read.  With an e4m3 cache the
// producer loads raw codes into a staging ring and converter warps widen them
// to f16 (value rows times their scale) into the same operand layout.
// Warp roles per CTA: 0 TMA producer and TMEM allocator, 1 MMA issuer
// (leader CTA only), [e4m3: 2-5 converters], then 16 softmax warps in four
// warpgroups, a quarter of the heads each (thread = cached row).
//
// Softmax per tile: each warp takes the per-head max of its 32 rows with a
// shuffle butterfly, the 4 warps of a warpgroup combine through shared memory, the
// pair exchanges its maxima through distributed shared memory, and the
// running max only moves when the tile max exceeds it by more than 2^8 (the
// accumulator is rescaled in TMEM then).  P = 2^(u - m) is written as bf16
// (f16 for e4m3) straight into the P^T operand of the CTA that owns those
// heads, in a ring of 64-row chunks.  The MMA issuer keeps the score GEMM two
// tiles ahead of the value GEMM, so the softmax of one tile overlaps the
// tensor work of the next ones.  Pairs are persistent (one per SM pair) and
// claim units dynamically, so one unit's loads and score GEMMs overlap the
// previous unit's epilogue.
#include <math.h>

#include <atomic>
#include <mutex>

#include "mla_device.cuh"
#include "mla_internal.h"
#include "sm100.cuh"

namespace mla {
namespace {

using namespace sm100;

constexpr int kSoftGroups = 4;           // softmax warpgroups, each a quarter of the heads
// 18 warps (bf16 cache) or 22 (e4m3 cache: four converter warps): see the role map above
template <bool F8>
constexpr int kThreadsT = 32 * ((F8 ? 6 : 2) + 4 * kSoftGroups);
constexpr int kWarpConv0 = 2, kConvWarps = 4;  // e4m3 converters
constexpr int kBox8 = 4096;                    // one e4m3 block: 64 rows x 64 bytes
constexpr int kStage8 = 4 * kBox8;             // e4m3 staging of one stage (at most four blocks)
constexpr int kSlotBytes = 32768;         // one ring stage
constexpr int kBoxBytes = 8192;           // 64 rows x 128 bytes
constexpr int kChunkBytes = 16384;        // one column chunk of 128 rows (both pages)
constexpr int kSStages = 5;               // score stages per tile: chunks {0,1} {2,3} {4,5} {6,7} {8}
constexpr bool kL2Hints = true;           // L2 residency policies on the cache loads

constexpr int kTile = 256;                // cached rows per pair tile
constexpr int kChunks = 9;                // 576 / 64 column chunks
constexpr float kRescaleLog2 = 8.0f;      // lazy rescale threshold (log2 units)
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kColS0 = 0, kColS1 = 128, kColO = 256;
constexpr int kWarpProd = 0, kWarpMma = 1;
constexpr int kQN = 8;                         // unit queue depth
template <bool F8>
constexpr int kWarpSoft0T = F8 ? 6 : 2;

struct TcParams {
  int n_heads, q_len, batch;
  const int32_t* block_table;
  int max_pages, num_pages;
  const int32_t* seq_lens;
  int num_splits, split_tokens;
  float scale_log2;            // softmax_scale * log2(e)
  const float* cache_scale;    // e4m3 cache: per-row dequantisation scale [num_pages * 64]
  unsigned* claim;             // unit counter of this launch (0 at launch; reset by the last pair)
  unsigned* done;              // pairs finished
  float* o_part;
  float* lse_part;
  int32_t* err;
  unsigned long long wait_limit;   // SM cycles a barrier wait may take before the launch aborts
  int withhold_q;                  // test hook: the leader leaves its first unit's query load out
};

template <int NH, bool F8>
struct Layout {
  static constexpr int HPW = NH / 2;                      // heads per CTA (its half of Q and P^T)
  static constexpr int HPG = NH / kSoftGroups;            // heads per softmax warpgroup
  static constexpr int kQChunk = HPW * 128;               // one 64-column chunk of this CTA's Q rows
  static constexpr int kPChunk = HPW * 128;               // 64 rows of P^T for this CTA's heads
  static constexpr int kPSlots = 6;                       // ring of P^T chunks (1.5 tiles)
  // misc area (bytes from kMisc)
  static constexpr int kBars = 0;                          // 64 barriers max
  static constexpr int kTmemSlot = 64 * 8;
  static constexpr int kAbort = kTmemSlot + 4;
  static constexpr int kChanged = kTmemSlot + 16;          // int [kSoftGroups]: running max moved
  static constexpr int kMused = kTmemSlot + 32;            // float [2][NH]
  static constexpr int kRed = kMused + 2 * NH * 4;          // float [kSoftGroups][4 warps][HPG]
  static constexpr int kOwnMax = kRed + kSoftGroups * 4 * HPG * 4;  // float [NH]
  static constexpr int kXMax = kOwnMax + NH * 4;            // float [2][NH]   written by the peer
  static constexpr int kLOwn = kXMax + 2 * NH * 4;          // float [NH]
  static constexpr int kLX = kLOwn + NH * 4;                // float [NH]      written by the peer
  static constexpr int kUnitQ = kLX + NH * 4;              // int [kQN]: units claimed for the pair
  static constexpr int kMiscBytes = kUnitQ + 4 * 8;
  // ring of operand stages: as many as fit next to Q, P^T and the misc area (at most 6)
  static constexpr int kFixed = kChunks * kQChunk + kPSlots * kPChunk + kMiscBytes + 1024;
  // (e4m3 cache: each stage also has a staging slot for the raw codes)
  static constexpr int kPerSlot = kSlotBytes + (F8 ? kStage8 : 0);
  static constexpr int kFit = (227 * 1024 - kFixed) / kPerSlot;
  static constexpr int kSlots = kFit > 6 ? 6 : kFit;
  static constexpr int kRing = 0;
  static constexpr int kStaging = kRing + kSlots * kSlotBytes;
  static constexpr int kQ = kStaging + (F8 ? kSlots * kStage8 : 0);
  static constexpr int kP = kQ + kChunks * kQChunk;
  static constexpr int kMisc = kP + kPSlots * kPChunk;
  static constexpr int kSmem = kMisc + kMiscBytes + 1024;  // + alignment slack
  static_assert(kSmem <= 227 * 1024 && kSlots >= 2, "shared memory budget");
};

// barrier indices in the misc area
template <int NS>
struct Bars {
  static constexpr int full = 0;                     // [NS] leader: TMA bytes of both CTAs
  static constexpr int empty = NS;                   // [NS] both: MMA done with the slot
  static constexpr int base = 2 * NS;
  static constexpr int s_full = base;                // [2]   both: S^T buffer ready
  static constexpr int s_free = base + 2;            // [2]   leader: both CTAs loaded the S^T buffer
  static constexpr int p_full = base + 4;            //       leader: both CTAs wrote P^T
  static constexpr int o_done = base + 5;            //       both: O^T MMAs of the tile done
  static constexpr int mx_full = base + 6;           // [2]   both: the peer's tile maxima arrived
  static constexpr int q_full = base + 8;            //       leader: Q of both CTAs loaded
  static constexpr int l_full = base + 9;            //       both: the peer's row sums arrived
  static constexpr int p_free = base + 10;           // [6]   both: O^T MMAs done with a P^T chunk slot
  static constexpr int q_free = base + 16;           //       both: the unit's score MMAs done (Q reusable)
  static constexpr int epi_done = base + 17;         //       leader: both CTAs read O^T out (TMEM reusable)
  // e4m3 cache only
  static constexpr int q_ready = base + 18;          //       leader: both CTAs converted Q to f16
  static constexpr int sfull8 = base + 19;           // [NS]  local: TMA bytes of a staging slot
  static constexpr int sempty8 = base + 19 + NS;     // [NS]  local: converters done with the staging slot
  static constexpr int uq_full = base + 19 + 2 * NS;   // [8]   both: unit queue slot written
  static constexpr int uq_empty = base + 27 + 2 * NS;  // [8]   leader: every consumer read the slot
  static constexpr int end = base + 35 + 2 * NS;
};

// Sum over the 32 lanes of a warp of each of C per-lane values, returned
// transposed: lane l gets the sum of index l % C.  log2(32) shuffle stages;
// the split stages halve the values each lane carries, so C = 32 costs 31
// shuffles instead of the 160 of C independent reductions.  v is clobbered.
template <int C>
__device__ __forceinline__ float transpose_reduce(float* v, int lane) {
#pragma unroll
  for (int off = 16; off >= C; off >>= 1) {
#pragma unroll
    for (int j = 0; j < C; ++j) v[j] += __shfl_xor_sync(0xffffffffu, v[j], off);
  }
#pragma unroll
  for (int off = C / 2; off >= 1; off >>= 1) {
    const bool up = (lane & off) != 0;
#pragma unroll
    for (int j = 0; j < off; ++j) {
      const float keep = up ? v[j + off] : v[j];
      const float send = up ? v[j] : v[j + off];
      v[j] = keep + __shfl_xor_sync(0xffffffffu, send, off);
    }
  }
  return v[0];
}

// Max over the 32 lanes of each of C per-lane values, returned transposed
// like transpose_reduce (lane l gets the max of index l % C); v is clobbered.
template <int C>
__device__ __forceinline__ float transpose_max(float* v, int lane) {
#pragma unroll
  for (int off = 16; off >= C; off >>= 1) {
#pragma unroll
    for (int j = 0; j < C; ++j) v[j] = fmaxf(v[j], __shfl_xor_sync(0xffffffffu, v[j], off));
  }
#pragma unroll
  for (int off = C / 2; off >= 1; off >>= 1) {
    const bool up = (lane & off) != 0;
#pragma unroll
    for (int j = 0; j < off; ++j) {
      const float keep = up ? v[j + off] : v[j];
      const float send = up ? v[j] : v[j + off];
      v[j] = fmaxf(keep, __shfl_xor_sync(0xffffffffu, send, off));
    }
  }
  return v[0];
}

// Store to the peer CTA's shared memory and signal 4 bytes of completed
// transaction on the peer's mbarrier (no release fence on the sender side).
__device__ __forceinline__ void st_async_f32(uint32_t cluster_addr, float v, uint32_t cluster_bar) {
  asm volatile("st.async.shared::cluster.mbarrier::complete_tx::bytes.b32 [%0], %1, [%2];" ::"r"(cluster_addr),
               "r"(__float_as_uint(v)), "r"(cluster_bar)
               : "memory");
}

__device__ __forceinline__ void st_cluster_b32(uint32_t addr, uint32_t v) {
  asm volatile("st.shared::cluster.b32 [%0], %1;" ::"r"(addr), "r"(v) : "memory");
}

// page id of a cached row of sequence b (0 for rows outside the table or the
// pool: those rows are masked by the softmax, and page 0 is readable memory)
__device__ __forceinline__ int page_of(const TcParams& p, int b, int row, bool* ok) {
  const int pidx = row >> 6;
  int pg = -1;
  if (pidx < p.max_pages) pg = p.block_table[(size_t)b * p.max_pages + pidx];
  *ok = pg >= 0 && pg < p.num_pages;
  return *ok ? pg : 0;
}

// The ring of operand slots shared by the pair: the leader's `full` barrier
// counts the bytes both CTAs load; `empty` is arrived by the MMA commit in
// both CTAs.  `kc` counts slots handed out, in the order the MMA uses them.
struct Ring {
  uint32_t base;      // shared address of slot 0
  uint32_t full0;     // barrier of slot 0 (this CTA's address)
  uint32_t empty0;
  int slots;
  uint32_t kc = 0;
};

template <int NH, bool F8>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kThreadsT<F8>, 1)
    decode_tc_kernel(const __grid_constant__ CUtensorMap tm_cache, const __grid_constant__ CUtensorMap tm_cache2,
                     const __grid_constant__ CUtensorMap tm_q, const TcParams p) {
  using LY = Layout<NH, F8>;
  constexpr int HPW = LY::HPW;
  constexpr int kThreads = kThreadsT<F8>;
  constexpr int kWarpSoft0 = kWarpSoft0T<F8>;
  // readers of each unit-queue entry: the peer's producer, the MMA issuer,
  // the converters and the softmax warps of both CTAs
  constexpr int kQConsumers = 2 + 2 * 4 * kSoftGroups + (F8 ? 2 * kConvWarps : 0);
  using B = Bars<LY::kSlots>;
  static_assert(B::end <= 64, "barrier area");

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t s_base = smem_u32(smem);
  const uint32_t s_q = s_base + LY::kQ, s_p = s_base + LY::kP;
  uint8_t* misc = smem + LY::kMisc;
  const uint32_t s_misc = s_base + LY::kMisc;
  auto bar = [&](int i) -> uint32_t { return s_misc + LY::kBars + 8 * i; };
  volatile int* abort_flag = reinterpret_cast<volatile int*>(misc + LY::kAbort);
  float* m_used = reinterpret_cast<float*>(misc + LY::kMused);
  float* red = reinterpret_cast<float*>(misc + LY::kRed);
  float* own_max = reinterpret_cast<float*>(misc + LY::kOwnMax);
  float* x_max = reinterpret_cast<float*>(misc + LY::kXMax);
  float* l_own = reinterpret_cast<float*>(misc + LY::kLOwn);
  float* l_x = reinterpret_cast<float*>(misc + LY::kLX);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint64_t lim = p.wait_limit;
  const uint32_t rank = cluster_rank();
  const uint32_t peer = rank ^ 1u;
  const bool leader = rank == 0;

  // ---- units: (query row r, split s); a persistent pair claims units one at a
  // time (see claim/next_unit); every role walks the pair's same sequence, so
  // barrier phases are counted globally (ring stages, tiles, units)
  const int S = p.num_splits;
  const int n_units = p.batch * p.q_len * S;
  const int pair = blockIdx.x >> 1, n_pairs = gridDim.x >> 1;
  struct UnitInfo { int r, s, b, lo, hi, n_tiles; };
  auto unit_at = [&](int u) -> UnitInfo {
    UnitInfo x;
    x.r = u / S;
    x.s = u % S;
    x.b = x.r / p.q_len;
    const int t = x.r % p.q_len;
    const int n_vis = p.seq_lens[x.b] - p.q_len + t + 1;
    x.lo = x.s * p.split_tokens;
    x.hi = min(x.lo + p.split_tokens, n_vis);
    const int n_tok = x.hi - x.lo;
    x.n_tiles = n_tok > 0 ? (n_tok + kTile - 1) / kTile : 0;
    return x;
  };

  // ---- set-up: barriers, TMEM, cluster sync
  if (threadIdx.x == 0) {
    for (int i = 0; i < LY::kSlots; ++i) {
      // bf16: one expect-tx arrival (the leader's producer) plus both CTAs' bytes;
      // e4m3: one arrival per converter warp of both CTAs
      mbar_init(bar(B::full + i), F8 ? 2 * kConvWarps : 1);
      mbar_init(bar(B::empty + i), 1);
      if constexpr (F8) {
        mbar_init(bar(B::sfull8 + i), 1);
        mbar_init(bar(B::sempty8 + i), kConvWarps);
      }
    }
    if constexpr (F8) mbar_init(bar(B::q_ready), 2 * kConvWarps);
    for (int i = 0; i < 2; ++i) {
      mbar_init(bar(B::s_full + i), 1);
      mbar_init(bar(B::s_free + i), 2 * 4 * kSoftGroups);
      mbar_init(bar(B::mx_full + i), kSoftGroups);   // local expect-tx arrivals + the peer's st.async bytes
    }
    mbar_init(bar(B::p_full), 2 * 4 * kSoftGroups);
    mbar_init(bar(B::o_done), 1);
    mbar_init(bar(B::q_full), 1);
    mbar_init(bar(B::q_free), 1);
    mbar_init(bar(B::epi_done), 2 * 4 * kSoftGroups);
    mbar_init(bar(B::l_full), kSoftGroups);
    for (int i = 0; i < LY::kPSlots; ++i) mbar_init(bar(B::p_free + i), 1);
    for (int i = 0; i < kQN; ++i) {
      mbar_init(bar(B::uq_full + i), 1);
      mbar_init(bar(B::uq_empty + i), kQConsumers);
    }
    *abort_flag = 0;
    fence_mbar_init();
  }
  for (int i = threadIdx.x; i < 2 * NH; i += kThreads) m_used[i] = -INFINITY;
  if (warp == kWarpProd) tmem_alloc_pair(s_misc + LY::kTmemSlot, kTmemCols);
  tc_fence_before();
  cluster_sync();
  tc_fence_after();
  const uint32_t tmem = *reinterpret_cast<volatile uint32_t*>(misc + LY::kTmemSlot);

  Ring ring{s_base + LY::kRing, bar(B::full), bar(B::empty), LY::kSlots};

  // ---- the pair's unit sequence: the leader's producer claims units from the
  // launch's counter (dynamic balance) and posts them, in order, to a queue in
  // both CTAs; every role reads every entry (-1: no units left)
  int* unit_q = reinterpret_cast<int*>(misc + LY::kUnitQ);
  auto claim = [&](uint32_t k) -> int {      // leader producer, lane 0
    const uint32_t slot = k % kQN;
    if (k >= kQN && !mbar_wait(bar(B::uq_empty + slot), ((k / kQN) - 1) & 1, abort_flag, lim)) return -2;
    const unsigned cu = atomicAdd(p.claim, 1u);
    const int uu = cu < (unsigned)n_units ? (int)cu : -1;
    *reinterpret_cast<volatile int*>(unit_q + slot) = uu;
    st_cluster_b32(mapa(smem_u32(unit_q + slot), peer), (uint32_t)uu);
    mbar_arrive_cluster(bar(B::uq_full + slot));
    mbar_arrive_cluster(mapa(bar(B::uq_full + slot), peer));
    return uu;
  };
  auto next_unit = [&](uint32_t k, bool whole_warp) -> int {
    const uint32_t slot = k % kQN;
    if (!mbar_wait(bar(B::uq_full + slot), (k / kQN) & 1, abort_flag, lim)) return -2;
    const int uu = *reinterpret_cast<volatile int*>(unit_q + slot);
    if (whole_warp) __syncwarp();
    if (lane == 0) mbar_arrive_cluster(mapa(bar(B::uq_empty + slot), 0));
    return uu;
  };
  auto producer_unit = [&](uint32_t k) -> int {   // whole producer warp
    if (leader) {
      int uu = 0;
      if (lane == 0) uu = claim(k);
      return __shfl_sync(0xffffffffu, uu, 0);
    }
    return next_unit(k, true);
  };

  // producer side (whole warp): lane 0 waits for a free slot and posts the
  // expected bytes (leader); the lanes then issue the slot's boxes
  auto take = [&](Ring& rg, uint32_t bytes, uint32_t& dst, uint32_t& fb) -> bool {
    const uint32_t slot = rg.kc % rg.slots;
    const uint32_t ph = (rg.kc / rg.slots) & 1u;
    bool ok = true;
    if (lane == 0) {
      ok = mbar_wait<false>(rg.empty0 + 8 * slot, ph ^ 1u, abort_flag, lim);
      if (ok && leader) mbar_arrive_expect_tx(rg.full0 + 8 * slot, 2u * bytes);
    }
    ok = __shfl_sync(0xffffffffu, ok, 0);
    dst = rg.base + slot * kSlotBytes;
    fb = mapa(rg.full0 + 8 * slot, 0);
    ++rg.kc;
    return ok;
  };
  // MMA side: wait for a filled slot
  auto ready = [&](Ring& rg, uint32_t& src, uint32_t& empty) -> bool {
    const uint32_t slot = rg.kc % rg.slots;
    const uint32_t ph = (rg.kc / rg.slots) & 1u;
    // e4m3: the converters arrive after generic-proxy writes (cluster scope)
    if (!__all_sync(0xffffffffu, mbar_wait<F8>(rg.full0 + 8 * slot, ph, abort_flag, lim))) return false;
    tc_fence_after();
    src = rg.base + slot * kSlotBytes;
    empty = rg.empty0 + 8 * slot;
    ++rg.kc;
    return true;
  };
  if (F8 && warp == kWarpProd) {
    // ============ TMA producer, e4m3 cache (both CTAs) ============
    // The same stages in the same order as the bf16 producer, but each CTA
    // loads raw e4m3 blocks ([64 rows x 64 bytes], one per lane) into its own
    // staging slot and local barrier; the converter warps widen them into the
    // operand ring.  Staging block b of a stage lands at b * 4 KB and is
    // widened to b * 8 KB: score stages use b = 2 * chunk + page, value
    // stages b = 2 * dims block + half.
    if constexpr (F8) {
      uint32_t kc = 0;
      auto take8 = [&](uint32_t nbox, uint32_t& dst, uint32_t& fb) -> bool {
        const uint32_t slot = kc % LY::kSlots;
        const uint32_t ph = (kc / LY::kSlots) & 1u;
        bool ok = true;
        if (lane == 0) {
          ok = mbar_wait<false>(bar(B::sempty8 + slot), ph ^ 1u, abort_flag, lim);
          if (ok) mbar_arrive_expect_tx(bar(B::sfull8 + slot), nbox * kBox8);
        }
        ok = __shfl_sync(0xffffffffu, ok, 0);
        dst = s_base + LY::kStaging + slot * kStage8;
        fb = bar(B::sfull8 + slot);
        ++kc;
        return ok;
      };
      if (lane == 0) {
        tma_prefetch_desc(&tm_cache);
        tma_prefetch_desc(&tm_q);
      }
      uint32_t uc = 0;
      bool ok = true;
      for (uint32_t k = 0; ok; ++k) {
      const int u = producer_unit(k);
      if (u == -2) { ok = false; break; }
      if (u < 0) break;
      const UnitInfo U = unit_at(u);
      if (U.n_tiles == 0) continue;
      const int r = U.r, b = U.b, lo = U.lo, hi = U.hi, n_tiles = U.n_tiles;
      if (lane == 0) {
        // the previous unit's score MMAs must be done with Q
        if (uc > 0) ok = mbar_wait<false>(bar(B::q_free), (uc - 1) & 1, abort_flag, lim);
        if (ok && !(p.withhold_q && leader && uc == 0)) {
          mbar_arrive_expect_tx(bar(B::q_full), kChunks * LY::kQChunk);
          for (int c = 0; c < kChunks; ++c)
            tma_load_3d(s_q + c * LY::kQChunk, &tm_q, 64 * c, (int)rank * HPW, r, bar(B::q_full));
        }
      }
      ok = __shfl_sync(0xffffffffu, ok, 0);
      if (!ok) break;
      auto load_s8 = [&](int i) -> bool {
        bool vv;
        const int pg = page_of(p, b, lo + kTile * i + 128 * (int)rank + 64 * (lane & 1), &vv);
        for (int st = 0; st < kSStages; ++st) {
          const int nc = st < kSStages - 1 ? 2 : 1;
          uint32_t dst, fb;
          if (!take8(2 * nc, dst, fb)) return false;
          if (lane < 2 * nc) tma_load_2d(dst + lane * kBox8, &tm_cache, 0, (pg * kChunks + 2 * st + (lane >> 1)) * 64, fb);
        }
        return true;
      };
      auto load_o8 = [&](int j) -> bool {
        for (int pg_i = 0; pg_i < 4; ++pg_i) {
          const int row0 = lo + kTile * j + 64 * pg_i;
          if (row0 >= hi) break;
          bool vld;
          const int pg = page_of(p, b, row0, &vld);
          uint32_t dst, fb;
          if (!take8(4, dst, fb)) return false;
          if (lane < 4) {
            const int blk = (256 * (lane >> 1) + 128 * (int)rank) / 64 + (lane & 1);
            tma_load_2d(dst + lane * kBox8, &tm_cache, 0, (pg * kChunks + blk) * 64, fb);
          }
        }
        return true;
      };
      ok = load_s8(0);
      if (ok && n_tiles > 1) ok = load_s8(1);
      for (int i = 0; i < n_tiles && ok; ++i) {
        if (i + 2 < n_tiles) ok = load_s8(i + 2);
        if (ok) ok = load_o8(i);
      }
      ++uc;
      }
    }
  } else if (F8 && warp >= kWarpConv0 && warp < kWarpConv0 + kConvWarps) {
    // ============ e4m3 -> f16 converters (both CTAs) ============
    // First Q (bf16 -> f16 in place, once per unit), then every stage in the
    // MMA's order: wait for the staging slot's bytes and the operand slot's
    // release, widen the codes exactly (e4m3 values are f16 values), write
    // them 128-byte swizzled, make them visible to the tensor core and arrive
    // on the leader's full barrier.  Value stages are also multiplied by the
    // row's dequantisation scale (one f16 rounding: the dequantised value);
    // for scores the softmax applies the scale to the row's dot products.
    if constexpr (F8) {
      const int ct = threadIdx.x - 32 * kWarpConv0;
      constexpr int kCT = 32 * kConvWarps;
      uint32_t kc = 0, uc = 0;
      bool ok = true;
      for (uint32_t k = 0; ok; ++k) {
      const int u = next_unit(k, true);
      if (u == -2) { ok = false; break; }
      if (u < 0) break;
      const UnitInfo U = unit_at(u);
      if (U.n_tiles == 0) continue;
      const int b = U.b, lo = U.lo, hi = U.hi, n_tiles = U.n_tiles;
      ok = __all_sync(0xffffffffu, mbar_wait<false>(bar(B::q_full), uc & 1, abort_flag, lim));
      if (ok) {
        for (int i = ct; i < kChunks * LY::kQChunk / 16; i += kCT) {
          uint4 v = *reinterpret_cast<const uint4*>(smem + LY::kQ + 16 * i);
          uint32_t* w = reinterpret_cast<uint32_t*>(&v);
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const float2 f = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&w[e]));
            const __half2 h = __floats2half2_rn(f.x, f.y);
            w[e] = *reinterpret_cast<const uint32_t*>(&h);
          }
          *reinterpret_cast<uint4*>(smem + LY::kQ + 16 * i) = v;
        }
        fence_proxy_async_cluster();     // read by the pair's MMAs
        __syncwarp();
        if (lane == 0) mbar_arrive_cluster(mapa(bar(B::q_ready), 0));
      }
      auto convert = [&](int nbox, int scale_page) -> bool {
        // scale_page >= 0: value stage of that page (lane l holds rows l, l + 32)
        float s_lo = 1.f, s_hi = 1.f;
        if (scale_page >= 0) {
          s_lo = p.cache_scale[(size_t)scale_page * 64 + lane];
          s_hi = p.cache_scale[(size_t)scale_page * 64 + 32 + lane];
        }
        const uint32_t slot = kc % LY::kSlots;
        const uint32_t ph = (kc / LY::kSlots) & 1u;
        ++kc;
        if (!__all_sync(0xffffffffu, mbar_wait<false>(bar(B::sfull8 + slot), ph, abort_flag, lim))) return false;
        if (!__all_sync(0xffffffffu, mbar_wait<false>(bar(B::empty + slot), ph ^ 1u, abort_flag, lim))) return false;
        const uint8_t* src = smem + LY::kStaging + slot * kStage8;
        uint8_t* dst = smem + LY::kRing + slot * kSlotBytes;
        // 16 codes (one quarter of a 64-byte row) per step
        for (int c = ct; c < nbox * 256; c += kCT) {
          const int box = c >> 8, row = (c >> 2) & 63, qq = c & 3;
          const uint4 codes = *reinterpret_cast<const uint4*>(src + box * kBox8 + row * 64 + qq * 16);
          const uint32_t* cw = reinterpret_cast<const uint32_t*>(&codes);
          const float sa = __shfl_sync(0xffffffffu, s_lo, row & 31);
          const float sb = __shfl_sync(0xffffffffu, s_hi, row & 31);
          const __half2 rs2 = __float2half2_rn(row < 32 ? sa : sb);
          uint32_t hw[8];
#pragma unroll
          for (int e = 0; e < 4; ++e) {
#pragma unroll
            for (int hf = 0; hf < 2; ++hf) {
              const __half2_raw r2 = __nv_cvt_fp8x2_to_halfraw2(
                  static_cast<__nv_fp8x2_storage_t>((cw[e] >> (16 * hf)) & 0xffffu), __NV_E4M3);
              __half2 h2 = *reinterpret_cast<const __half2*>(&r2);
              if (scale_page >= 0) h2 = __hmul2(h2, rs2);
              hw[2 * e + hf] = *reinterpret_cast<const uint32_t*>(&h2);
            }
          }
          uint8_t* rowp = dst + box * kBoxBytes + row * 128;
          *reinterpret_cast<uint4*>(rowp + (((2 * qq) ^ (row & 7)) << 4)) = make_uint4(hw[0], hw[1], hw[2], hw[3]);
          *reinterpret_cast<uint4*>(rowp + (((2 * qq + 1) ^ (row & 7)) << 4)) = make_uint4(hw[4], hw[5], hw[6], hw[7]);
        }
        fence_proxy_async_cluster();     // read by the pair's MMAs
        __syncwarp();
        if (lane == 0) {
          mbar_arrive_local(bar(B::sempty8 + slot));
          mbar_arrive_cluster(mapa(bar(B::full + slot), 0));
        }
        return true;
      };
      auto conv_s = [&]() -> bool {
        for (int st = 0; st < kSStages; ++st)
          if (!convert(st < kSStages - 1 ? 4 : 2, -1)) return false;
        return true;
      };
      auto conv_o = [&](int j) -> bool {
        for (int pg_i = 0; pg_i < 4; ++pg_i) {
          const int row0 = lo + kTile * j + 64 * pg_i;
          if (row0 >= hi) break;
          bool vld;
          const int pg = page_of(p, b, row0, &vld);
          if (!convert(4, pg)) return false;
        }
        return true;
      };
      if (ok) ok = conv_s();
      if (ok && n_tiles > 1) ok = conv_s();
      for (int i = 0; i < n_tiles && ok; ++i) {
        if (i + 2 < n_tiles) ok = conv_s();
        if (ok) ok = conv_o(i);
      }
      ++uc;
      }
    }
  } else if (warp == kWarpProd) {
    // ============ TMA producer (both CTAs), in the order the MMA consumes ============
    // S(0), S(1), then per tile i: S(i+2), O(i).  The pool is page-blocked
    // (nine contiguous [64 rows x 64 columns] blocks per page), viewed as 2-D
    // [blocks * 64 lines x 64 columns].  A score stage is blocks c, c+1 of this
    // CTA's two pages (lane l: block c + l/2 of page l%2, 8 KB each); a value
    // stage is one page's two dims blocks of this CTA (lane l: dims block l,
    // one contiguous 16 KB box each).  One ring in consumption order keeps the
    // most bytes in flight: separate score and value rings measured slower.
    if (lane == 0) {
      tma_prefetch_desc(&tm_cache);
      tma_prefetch_desc(&tm_cache2);
      tma_prefetch_desc(&tm_q);
    }
    uint32_t uc = 0;
    bool ok = true;
    for (uint32_t k = 0; ok; ++k) {
    const int u = producer_unit(k);
    if (u == -2) { ok = false; break; }
    if (u < 0) break;
    const UnitInfo U = unit_at(u);
    if (U.n_tiles == 0) continue;
    const int r = U.r, b = U.b, lo = U.lo, hi = U.hi, n_tiles = U.n_tiles;
    if (lane == 0) {
      // the previous unit's score MMAs must be done with Q (both halves)
      if (uc > 0) ok = mbar_wait<false>(bar(B::q_free), (uc - 1) & 1, abort_flag, lim);
      // (test hook: the leader leaves the query load of its first unit out, so
      // the MMA issuer's wait for it runs out and the launch aborts cleanly)
      if (ok && !(p.withhold_q && leader && uc == 0)) {
        const uint32_t q_bar = mapa(bar(B::q_full), 0);
        if (leader) mbar_arrive_expect_tx(bar(B::q_full), 2u * kChunks * LY::kQChunk);
        for (int c = 0; c < kChunks; ++c)
          tma_load_3d_pair(s_q + c * LY::kQChunk, &tm_q, 64 * c, (int)rank * HPW, r, q_bar);
      }
    }
    ok = __shfl_sync(0xffffffffu, ok, 0);
    if (!ok) break;
    // L2 residency: this CTA's score rows are re-read (by the peer and by
    // itself) for the value operand two tiles later, so they are loaded
    // evict-last; value loads are the rows' last use and go evict-first.
    const uint64_t pol_keep = kL2Hints ? policy_evict_last() : 0;
    const uint64_t pol_drop = kL2Hints ? policy_evict_first() : 0;
    auto load_s = [&](int i) -> bool {
      bool vv;
      const int pg = page_of(p, b, lo + kTile * i + 128 * (int)rank + 64 * (lane & 1), &vv);
      for (int st = 0; st < kSStages; ++st) {
        const int nc = st < kSStages - 1 ? 2 : 1;
        uint32_t dst, fb;
        if (!take(ring, nc * kChunkBytes, dst, fb)) return false;
        if (lane < 2 * nc) {
          const uint32_t d = dst + (lane >> 1) * kChunkBytes + (lane & 1) * kBoxBytes;
          const int y = (pg * kChunks + 2 * st + (lane >> 1)) * 64;
          if (kL2Hints) tma_load_2d_pair_hint(d, &tm_cache, 0, y, fb, pol_keep);
          else tma_load_2d_pair(d, &tm_cache, 0, y, fb);
        }
      }
      return true;
    };
    auto load_o = [&](int j) -> bool {
      for (int pg_i = 0; pg_i < 4; ++pg_i) {
        const int row0 = lo + kTile * j + 64 * pg_i;
        if (row0 >= hi) break;
        bool vld;
        const int pg = page_of(p, b, row0, &vld);
        uint32_t dst, fb;
        if (!take(ring, 2 * kChunkBytes, dst, fb)) return false;
        if (lane < 2) {
          const int y = (pg * kChunks + (256 * lane + 128 * (int)rank) / 64) * 64;
          if (kL2Hints) tma_load_2d_pair_hint(dst + lane * kChunkBytes, &tm_cache2, 0, y, fb, pol_drop);
          else tma_load_2d_pair(dst + lane * kChunkBytes, &tm_cache2, 0, y, fb);
        }
      }
      return true;
    };
    ok = load_s(0);
    if (ok && n_tiles > 1) ok = load_s(1);
    for (int i = 0; i < n_tiles && ok; ++i) {
      if (i + 2 < n_tiles) ok = load_s(i + 2);
      if (ok) ok = load_o(i);
    }
    ++uc;
    }
  } else if (warp == kWarpMma) {
    // ================= MMA issuer (leader CTA) =================
    // Per unit: S(0), S(1), then per tile i: S(i+2), O(i) -- the score GEMM
    // runs two tiles ahead so the softmax of tile i overlaps S(i+1), O(i-1),
    // S(i+2).  Across units the next unit's S(0), S(1) run while the softmax
    // warps read the previous unit's O^T out; its first O^T MMA waits for that.
    // Tiles are numbered globally (gt + i) for the S^T buffers, the P^T ring
    // and the per-tile barriers.
    if (leader) {
      // e4m3 cache: the operands are f16 (widened codes, Q and P in f16)
      constexpr uint32_t idS = idesc_f16(256, NH, false, false, F8);
      constexpr uint32_t idO = idesc_f16(256, NH, true, false, F8);
      uint32_t uc = 0, gt = 0;
      bool ok = true;
      for (uint32_t k = 0; ok; ++k) {
      const int u = next_unit(k, true);
      if (u == -2) { ok = false; break; }
      if (u < 0) break;
      const UnitInfo U = unit_at(u);
      if (U.n_tiles == 0) continue;
      const int lo = U.lo, hi = U.hi, n_tiles = U.n_tiles;
      ok = __all_sync(0xffffffffu, mbar_wait(bar(F8 ? B::q_ready : B::q_full), uc & 1, abort_flag, lim));
      if (!ok) break;
      tc_fence_after();
      auto issue_s = [&](int i) -> bool {
        const uint32_t gi = gt + i;
        const int sb = gi & 1;
        if (gi >= 2) {
          if (!__all_sync(0xffffffffu, mbar_wait(bar(B::s_free + sb), ((gi - 2) >> 1) & 1, abort_flag, lim))) return false;
          tc_fence_after();
        }
        const uint32_t d = tmem + (sb ? kColS1 : kColS0);
        for (int st = 0; st < kSStages; ++st) {
          uint32_t a0, empty;
          if (!ready(ring, a0, empty)) return false;
          const int nc = st < kSStages - 1 ? 2 : 1;
          for (int cc = 0; cc < nc; ++cc) {
            const int c = 2 * st + cc;
#pragma unroll
            for (int ks = 0; ks < 4; ++ks) {
              const uint64_t ad = smem_desc_sw128(a0 + cc * kChunkBytes + ks * 32, 16, 1024);
              const uint64_t bd = smem_desc_sw128(s_q + c * LY::kQChunk + ks * 32, 16, 1024);
              mma_pair_f16_w(d, ad, bd, idS, (c | ks) != 0);
            }
          }
          mma_commit_pair_w(empty, 0x3);
        }
        mma_commit_pair_w(bar(B::s_full + sb), 0x3);
        // the unit's last score GEMM: Q may be replaced once it completes
        if (i == n_tiles - 1) mma_commit_pair_w(bar(B::q_free), 0x3);
        return true;
      };
      auto issue_o = [&](int j) -> bool {
        const uint32_t gj = gt + j;
        if (!__all_sync(0xffffffffu, mbar_wait(bar(B::p_full), gj & 1, abort_flag, lim))) return false;
        // the accumulator is overwritten by this unit's first O^T MMA: the
        // previous unit's epilogue must have read it out
        if (j == 0 && uc > 0 && !__all_sync(0xffffffffu, mbar_wait(bar(B::epi_done), (uc - 1) & 1, abort_flag, lim))) return false;
        tc_fence_after();
        for (int pg_i = 0; pg_i < 4; ++pg_i) {
          // P^T chunk pg_i of global tile gj lives in slot (4 gj + pg_i) mod
          // kPSlots; its release is committed even for pages past the end
          const int pslot = (4 * gj + pg_i) % LY::kPSlots;
          if (lo + kTile * j + 64 * pg_i < hi) {
            uint32_t a0, empty;
            if (!ready(ring, a0, empty)) return false;
            for (int bb = 0; bb < 2; ++bb) {
#pragma unroll
              for (int ks = 0; ks < 4; ++ks) {
                const uint64_t ad = smem_desc_sw128(a0 + bb * kChunkBytes + ks * 2048, kBoxBytes, 1024);
                const uint64_t bd = smem_desc_sw128(s_p + pslot * LY::kPChunk + ks * 32, 16, 1024);
                mma_pair_f16_w(tmem + kColO + bb * 128, ad, bd, idO, (j | pg_i | ks) != 0);
              }
            }
            mma_commit_pair_w(empty, 0x3);
          }
          mma_commit_pair_w(bar(B::p_free + pslot), 0x3);
        }
        mma_commit_pair_w(bar(B::o_done), 0x3);
        return true;
      };
      ok = issue_s(0);
      if (ok && n_tiles > 1) ok = issue_s(1);
      for (int i = 0; i < n_tiles && ok; ++i) {
        if (i + 2 < n_tiles) ok = issue_s(i + 2);
        if (ok) ok = issue_o(i);
      }
      gt += n_tiles;
      ++uc;
      }
    }
  } else {
    // ================= softmax (both CTAs, warps 2-17) =================
    // Four warpgroups, each a quarter of the heads (HPG) for this CTA's 128
    // rows of the tile (thread = row).  Per tile:
    //   A  load the tile's scores into registers and release the S^T buffer;
    //      per-head max over the warp (shuffle butterfly), then over the 4 warps of the group
    //   -- warp 0 of the group exchanges maxima with the peer's group of the
    //      same heads and sets the new running max (and the rescale factors)
    //   B  P = 2^(u - m) written to the P^T operand of the CTA that owns
    //      these heads (CTA g/2), running row sums updated
    constexpr int HPG = LY::HPG;
    constexpr int C = HPG < 32 ? HPG : 32;
    const int g = (warp - kWarpSoft0) >> 2;    // warpgroup: heads [g*HPG, (g+1)*HPG)
    const int q = warp & 3;                    // TMEM lane quadrant
    const int tok = 32 * q + lane;             // row within this CTA's half of the tile
    const uint32_t lane_addr = static_cast<uint32_t>(32 * q) << 16;
    const int owner = g >> 1;                  // CTA whose P^T holds these heads
    const uint32_t p_dst = (owner == (int)rank) ? s_p : mapa(s_p, (uint32_t)owner);
    const bool p_remote = owner != (int)rank;
    const int hr0 = (g & 1) * HPG;             // first P^T row of these heads in the owner
    float* red_g = red + g * 4 * HPG;
    float* alpha = own_max;                    // reused after the tile max is consumed
    volatile int* changed_flag = reinterpret_cast<volatile int*>(misc + LY::kChanged) + g;
    const int kt = 128 * (int)rank + tok;      // row within the pair tile
    const int ke = kt & ~1;
    const int wcol = ke & 63;
    const int pchunk = ke >> 6;                // P^T chunk (64 rows of the tile) this warp writes
    const int st_id = threadIdx.x - 32 * kWarpSoft0;   // 0 .. 511
    uint32_t uc = 0, gt = 0;                   // units with tiles done, global tile count
    bool ok = true;
    for (uint32_t k = 0; ok; ++k) {
    const int u = next_unit(k, true);
    if (u == -2) { ok = false; break; }
    if (u < 0) break;
    const UnitInfo U = unit_at(u);
    const int r = U.r, s = U.s, b = U.b, lo = U.lo, hi = U.hi, n_tiles = U.n_tiles;
    if (n_tiles == 0) {
      // nothing visible in this split: lse = -inf (the leader CTA), o_part is
      // left unwritten (the merge gives such a split weight 0 and skips it)
      if (leader)
        for (int h = st_id; h < p.n_heads; h += 32 * 4 * kSoftGroups)
          p.lse_part[((size_t)r * p.n_heads + h) * S + s] = -INFINITY;
      continue;
    }
    // running row sums of this warp's 32 rows: chunk k, head C*k + lane % C
    float l_acc[HPG / C];
#pragma unroll
    for (int k = 0; k < HPG / C; ++k) l_acc[k] = 0.f;
    for (int i = 0; i < n_tiles; ++i) {
      const uint32_t gi = gt + i;              // global tile number: buffers and phases
      const int sb = gi & 1;
      ok = __all_sync(0xffffffffu, mbar_wait<false>(bar(B::s_full + sb), (gi >> 1) & 1, abort_flag, lim));
      if (!ok) break;
      tc_fence_after();
      const int row = lo + kTile * i + kt;
      bool vld = row < hi;
      float rsc = 1.f;                         // e4m3: the row's dequantisation scale
      if (vld) {
        bool pok;
        const int pg = page_of(p, b, row, &pok);
        if (!pok) { vld = false; flag_error(p.err, MLA_DEVERR_PAGE); }
        else if constexpr (F8) rsc = p.cache_scale[(size_t)pg * 64 + (row & 63)];
      }
      const float sl = vld ? p.scale_log2 * rsc : 0.f;
      // ---- A: scores into registers, release the buffer, per-head tile max
      float u[HPG];
      {
        const uint32_t sc = tmem + lane_addr + (sb ? kColS1 : kColS0) + g * HPG;
#pragma unroll
        for (int k = 0; k < HPG / C; ++k) tmem_ld<C>(sc + C * k, u + C * k);
        tmem_wait_ld();
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_cluster(mapa(bar(B::s_free + sb), 0));
#pragma unroll
      for (int h = 0; h < HPG; ++h) u[h] = vld ? u[h] * sl : -INFINITY;
      {
        // per-head max over the warp's 32 rows: a transposing butterfly
        // leaves head C*k + lane%C's max in lane `lane`
        float t[HPG];
#pragma unroll
        for (int h = 0; h < HPG; ++h) t[h] = u[h];
#pragma unroll
        for (int k = 0; k < HPG / C; ++k) {
          const float mx = transpose_max<C>(t + C * k, lane);
          if (lane < C) red_g[q * HPG + C * k + lane] = mx;
        }
      }
      named_barrier(1 + g, 128);
      const int xb = gi & 1;
      const float* m_prev = m_used + ((gi + 1) & 1) * NH + g * HPG;   // unused on a unit's first tile
      float* m_next = m_used + (gi & 1) * NH + g * HPG;
      if (q == 0) {
        // exchange tile maxima with the peer's group of the same heads: arm
        // this CTA's barrier for the peer's HPG values, send ours with st.async
        // (each store completes its bytes on the peer's barrier)
        if (lane == 0) mbar_arrive_expect_tx(bar(B::mx_full + xb), HPG * 4);
        __syncwarp();
        const uint32_t peer_bar = mapa(bar(B::mx_full + xb), peer);
        for (int h = lane; h < HPG; h += 32) {
          const float tm = fmaxf(fmaxf(red_g[h], red_g[HPG + h]), fmaxf(red_g[2 * HPG + h], red_g[3 * HPG + h]));
          own_max[g * HPG + h] = tm;
          st_async_f32(mapa(smem_u32(x_max + xb * NH + g * HPG + h), peer), tm, peer_bar);
        }
        if (__all_sync(0xffffffffu, mbar_wait(bar(B::mx_full + xb), (gi >> 1) & 1, abort_flag, lim))) {
          int ch = 0;
          for (int h = lane; h < HPG; h += 32) {
            const float mt = fmaxf(own_max[g * HPG + h], x_max[xb * NH + g * HPG + h]);
            const float mo = i == 0 ? -INFINITY : m_prev[h];
            const float mn = (mt > mo + kRescaleLog2) ? mt : mo;
            m_next[h] = mn;
            // rescale factor for sums and accumulator kept so far (0 when nothing was kept)
            alpha[g * HPG + h] = (mo == -INFINITY) ? 0.f : exp2_approx(mo - mn);
            ch |= (mn != mo);
          }
          ch = __any_sync(0xffffffffu, ch);
          if (lane == 0) *changed_flag = ch;
        }
      }
      named_barrier(1 + g, 128);
      if (*abort_flag) { ok = false; break; }
      const bool changed = *changed_flag != 0;
      // ---- B1: probabilities (fp32, in registers)
#pragma unroll
      for (int h = 0; h < HPG; ++h) {
        const float mn = m_next[h];
        u[h] = exp2_approx(u[h] - (mn == -INFINITY ? 0.f : mn));
      }
      // this warp's P^T chunk slot must have been released by the O^T MMAs
      // of its previous use (1 or 2 tiles back), and every phase of o_done is
      // observed in order: a parity wait cannot tell a barrier two phases
      // behind from one that is done, so skipping phases here would let the
      // rescale and the epilogue read the accumulator before the last O^T
      // MMAs complete
      const int pn = 4 * gi + pchunk;
      const int pslot = pn % LY::kPSlots;
      if (pn >= LY::kPSlots) {
        ok = __all_sync(0xffffffffu,
                        mbar_wait<false>(bar(B::p_free + pslot), ((pn / LY::kPSlots) - 1) & 1, abort_flag, lim));
        if (!ok) break;
      }
      const uint32_t row_base = pslot * LY::kPChunk + (wcol & 7) * 2;
      if (i >= 1) {
        ok = __all_sync(0xffffffffu, mbar_wait<false>(bar(B::o_done), (gi - 1) & 1, abort_flag, lim));
        if (!ok) break;
        tc_fence_after();
      }
      if (i >= 1 && changed) {
        {
          constexpr int CC = C < 16 ? C : 16;
#pragma unroll 1
          for (int bb = 0; bb < 2; ++bb) {
#pragma unroll 1
            for (int k = 0; k < HPG / CC; ++k) {
              const uint32_t oc = tmem + lane_addr + kColO + bb * 128 + g * HPG + CC * k;
              float o[CC];
              tmem_ld<CC>(oc, o);
              tmem_wait_ld();
#pragma unroll
              for (int h = 0; h < CC; ++h) o[h] *= alpha[g * HPG + CC * k + h];
              tmem_st<CC>(oc, o);
            }
          }
          tmem_wait_st();
        }
      }
      // ---- B2: P^T (bf16, pairs of rows per 32-bit store), running row sums
#pragma unroll
      for (int k = 0; k < HPG / C; ++k) {
        float* uk = u + C * k;
#pragma unroll
        for (int h = 0; h < C; h += 2) {
          const float send = (lane & 1) ? uk[h] : uk[h + 1];
          const float recv = __shfl_xor_sync(0xffffffffu, send, 1);
          const int hr = hr0 + C * k + ((lane & 1) ? h + 1 : h);
          const float mine = (lane & 1) ? uk[h + 1] : uk[h];
          uint32_t val;
          if constexpr (F8) {
            const __half2 pk = (lane & 1) ? __floats2half2_rn(recv, mine) : __floats2half2_rn(mine, recv);
            val = *reinterpret_cast<const uint32_t*>(&pk);
          } else {
            const __nv_bfloat162 pk = (lane & 1) ? __floats2bfloat162_rn(recv, mine) : __floats2bfloat162_rn(mine, recv);
            val = *reinterpret_cast<const uint32_t*>(&pk);
          }
          const uint32_t off = row_base + hr * 128 + ((((wcol >> 3) ^ (hr & 7))) << 4);
          if (p_remote) st_cluster_b32(p_dst + off, val);
          else asm volatile("st.shared.b32 [%0], %1;" ::"r"(p_dst + off), "r"(val) : "memory");
        }
        const float ls = transpose_reduce<C>(uk, lane);
        l_acc[k] = changed ? fmaf(l_acc[k], alpha[g * HPG + C * k + (lane % C)], ls) : l_acc[k] + ls;
      }
      tc_fence_before();
      fence_proxy_async_cluster();
      __syncwarp();
      if (lane == 0) mbar_arrive_cluster(mapa(bar(B::p_full), 0));
    }
    // ---- epilogue: normalise O^T by the row sums, write o_part and lse
    if (ok) ok = __all_sync(0xffffffffu, mbar_wait<false>(bar(B::o_done), (gt + n_tiles - 1) & 1, abort_flag, lim));
    if (ok) {
      tc_fence_after();
#pragma unroll
      for (int k = 0; k < HPG / C; ++k)
        if (lane < C) red_g[q * HPG + C * k + lane] = l_acc[k];
      named_barrier(1 + g, 128);
      float* inv_l = own_max;
      if (q == 0) {
        // exchange row sums with the peer's group (as the tile maxima)
        if (lane == 0) mbar_arrive_expect_tx(bar(B::l_full), HPG * 4);
        __syncwarp();
        const uint32_t peer_bar = mapa(bar(B::l_full), peer);
        for (int h = lane; h < HPG; h += 32) {
          const float lt = red_g[h] + red_g[HPG + h] + red_g[2 * HPG + h] + red_g[3 * HPG + h];
          l_own[g * HPG + h] = lt;
          st_async_f32(mapa(smem_u32(l_x + g * HPG + h), peer), lt, peer_bar);
        }
        if (__all_sync(0xffffffffu, mbar_wait(bar(B::l_full), uc & 1, abort_flag, lim))) {
          const float* m_fin = m_used + ((gt + n_tiles - 1) & 1) * NH + g * HPG;
          for (int h = lane; h < HPG; h += 32) {
            const int hg = g * HPG + h;
            const float lt = l_own[hg] + l_x[hg];
            inv_l[hg] = lt > 0.f ? 1.0f / lt : 0.f;
            if (leader && hg < p.n_heads)
              p.lse_part[((size_t)r * p.n_heads + hg) * S + s] =
                  lt > 0.f ? (m_fin[h] + log2f(lt)) * 0.69314718055994531f : -INFINITY;
          }
        }
      }
      named_barrier(1 + g, 128);
      if (!*abort_flag) {
        const size_t hstride = (size_t)S * MLA_D_C;
#pragma unroll 1
        for (int bb = 0; bb < 2; ++bb) {
          const int d = 256 * bb + 128 * (int)rank + tok;
#pragma unroll 1
          for (int k = 0; k < HPG / C; ++k) {
            const int h0 = g * HPG + C * k;
            float* op = p.o_part + ((size_t)r * p.n_heads * S + s) * MLA_D_C + d + (size_t)h0 * hstride;
            float o[C];
            tmem_ld<C>(tmem + lane_addr + kColO + bb * 128 + h0, o);
            tmem_wait_ld();
#pragma unroll
            for (int h = 0; h < C; ++h) {
              if (h0 + h < p.n_heads) *op = o[h] * inv_l[h0 + h];
              op += hstride;
            }
          }
        }
      }
      // this warp's part of O^T has been read: the pair's next unit may overwrite it
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_cluster(mapa(bar(B::epi_done), 0));
    }
    gt += n_tiles;
    ++uc;
    }
  }

  // ---- teardown
  if (*abort_flag) {
    if (threadIdx.x == 0) flag_error(p.err, MLA_DEVERR_TIMEOUT);
    // let copies and MMAs already in flight land before the memory is released
    const uint64_t t0 = globaltimer();
    while (globaltimer() - t0 < 2000000ull) {
    }
  }
  // the last pair to finish resets the launch's unit counter for the next launch
  if (leader && threadIdx.x == 0) {
    __threadfence();
    if (atomicAdd(p.done, 1u) == (unsigned)(n_pairs - 1)) {
      atomicExch(p.claim, 0u);
      atomicExch(p.done, 0u);
    }
  }
  tc_fence_before();
  __syncthreads();
  cluster_sync();
  if (warp == kWarpProd) {
    tc_fence_after();
    tmem_dealloc_pair(tmem, kTmemCols);
  }
}

// ------------------------------------------------------------------ host side
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
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

// Unit counters of the persistent decode: one (claim, done) pair per launch in
// flight, from kCounterSlots per device.  A launch starts with both at 0 and
// its last pair sets them back to 0, so consecutive launches reuse a slot
// without a reset.  The slot is chosen by the launch's o_part workspace: calls
// that write the same o_part must not overlap on the GPU anyway (they would
// race on the partials), and calls with different workspaces get different
// slots while at most kCounterSlots distinct workspaces are in use.  A CUDA
// graph captures the slot with the o_part it was captured with, so replays of
// one graph share a slot exactly when they share a workspace.
constexpr int kCounterSlots = 64;

__device__ unsigned g_unit_claim[kCounterSlots];
__device__ unsigned g_unit_done[kCounterSlots];

bool claim_slot(const void* workspace, unsigned** claim, unsigned** done) {
  static std::mutex mu;
  static const void* owner[kCounterSlots] = {};
  static unsigned next = 0;
  void* c = nullptr;
  void* d = nullptr;
  if (cudaGetSymbolAddress(&c, g_unit_claim) != cudaSuccess || cudaGetSymbolAddress(&d, g_unit_done) != cudaSuccess)
    return false;
  unsigned i = kCounterSlots;
  {
    std::lock_guard<std::mutex> lock(mu);
    for (unsigned k = 0; k < (unsigned)kCounterSlots; ++k)
      if (owner[k] == workspace) { i = k; break; }
    if (i == (unsigned)kCounterSlots) {
      i = next++ % kCounterSlots;
      owner[i] = workspace;
    }
  }
  *claim = static_cast<unsigned*>(c) + i;
  *done = static_cast<unsigned*>(d) + i;
  return true;
}

// CTA pairs that fit on the current device at one pair per two SMs
long long sm_pairs() {
  int dev = 0, sms = 0;
  if (cudaGetDevice(&dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || sms < 2)
    return 1;
  return sms / 2;
}

template <int NH, bool F8>
cudaError_t launch_nh(const DecodeArgs& a, const CUtensorMap& tc, const CUtensorMap& tc2, const CUtensorMap& tq,
                      cudaStream_t st) {
  using LY = Layout<NH, F8>;
  cudaError_t e = cudaFuncSetAttribute(decode_tc_kernel<NH, F8>, cudaFuncAttributeMaxDynamicSharedMemorySize, LY::kSmem);
  if (e != cudaSuccess) return e;
  TcParams p{a.n_heads, a.q_len, a.batch, a.block_table, a.max_pages, a.num_pages, a.seq_lens, a.num_splits,
             a.split_tokens, a.softmax_scale * 1.4426950408889634f, a.cache_scale, nullptr, nullptr,
             a.o_part, a.lse_part, a.err, g_wait_limit.load(), g_withhold_q.load()};
  // Persistent pairs, one per SM pair, claiming units from a counter of this
  // launch: set-up, Q loads, pipeline fill and the epilogue are amortised and
  // overlapped across units, and splits of unequal length still balance.
  const long long units = (long long)a.batch * a.q_len * a.num_splits;
  const long long P = sm_pairs();
  const long long pairs = units < P ? units : P;
  if (!claim_slot(a.o_part, &p.claim, &p.done)) return cudaErrorInvalidSymbol;
  dim3 grid((unsigned)(2 * pairs));
  decode_tc_kernel<NH, F8><<<grid, kThreadsT<F8>, LY::kSmem, st>>>(tc, tc2, tq, p);
  return cudaGetLastError();
}

}  // namespace

bool decode_tc_supported(const DecodeArgs& a) {
  return a.q_dtype == MLA_BF16 && (a.cache_dtype == MLA_BF16 || a.cache_dtype == MLA_E4M3) &&
         a.page_size == 64 && (long long)a.batch * a.q_len * a.num_splits * 2 < (1ll << 31);
}

cudaError_t launch_decode_tc(const DecodeArgs& a, cudaStream_t st) {
  EncodeTiledFn enc = encode_fn();
  if (!enc) return cudaErrorNotSupported;
  const int NH = a.n_heads <= 16 ? 16 : a.n_heads <= 32 ? 32 : a.n_heads <= 64 ? 64 : 128;
  const int HPW = NH / 2;
  CUtensorMap tc, tc2, tq;
  const bool f8 = a.cache_dtype == MLA_E4M3;
  // the page-blocked pool as 2-D [num_pages * 9 * 64 lines x 64 columns]:
  // bf16, 128-byte lines: boxes of 64 lines (one block) and of 128 lines (two
  // adjacent blocks); e4m3, 64-byte lines: boxes of one block, unswizzled
  if (f8) {
    cuuint64_t dims[2] = {64, (cuuint64_t)a.num_pages * kChunks * 64};
    cuuint64_t strides[1] = {64};
    cuuint32_t box[2] = {64, 64};
    cuuint32_t es[2] = {1, 1};
    if (enc(&tc, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(a.cache), dims, strides, box, es,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return cudaErrorInvalidValue;
    tc2 = tc;
  }
  for (int k = 0; k < 2 && !f8; ++k) {
    cuuint64_t dims[2] = {64, (cuuint64_t)a.num_pages * kChunks * 64};
    cuuint64_t strides[1] = {128};
    cuuint32_t box[2] = {64, k == 0 ? 64u : 128u};
    cuuint32_t es[2] = {1, 1};
    if (enc(k == 0 ? &tc : &tc2, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(a.cache), dims, strides, box,
            es, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return cudaErrorInvalidValue;
  }
  {
    cuuint64_t dims[3] = {MLA_D_ROW, (cuuint64_t)a.n_heads, (cuuint64_t)a.batch * a.q_len};
    cuuint64_t strides[2] = {MLA_D_ROW * 2, (cuuint64_t)a.n_heads * MLA_D_ROW * 2};
    cuuint32_t box[3] = {64, (cuuint32_t)HPW, 1};
    cuuint32_t es[3] = {1, 1, 1};
    if (enc(&tq, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(a.q_abs), dims, strides, box, es,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return cudaErrorInvalidValue;
  }
  if (f8) {
    switch (NH) {
      case 16: return launch_nh<16, true>(a, tc, tc2, tq, st);
      case 32: return launch_nh<32, true>(a, tc, tc2, tq, st);
      case 64: return launch_nh<64, true>(a, tc, tc2, tq, st);
      default: return launch_nh<128, true>(a, tc, tc2, tq, st);
    }
  }
  switch (NH) {
    case 16: return launch_nh<16, false>(a, tc, tc2, tq, st);
    case 32: return launch_nh<32, false>(a, tc, tc2, tq, st);
    case 64: return launch_nh<64, false>(a, tc, tc2, tq, st);
    default: return launch_nh<128, false>(a, tc, tc2, tq, st);
  }
}

}  // namespace mla

extern "C" mla_status mla_test_set_decode_wait(unsigned long long limit_cycles, int withhold_q_load) {
  if (limit_cycles == 0) limit_cycles = 4000000000ull;
  mla::g_wait_limit.store(limit_cycles);
  mla::g_withhold_q.store(withhold_q_load != 0);
  return MLA_OK;
}
