// Split-KV latent attention for 65..128 heads over a bf16 or e4m3 cache, on
// the tcgen05 tensor cores, with the heads split between the two CTAs of a
// pair.  Three instantiations:
//   bf16 cache, bf16 Q and P (kind::f16);
//   F8: e4m3 cache with bf16 queries: converter warps widen the staged codes
//       into the same f16 operand layout, Q and P are f16, and the softmax
//       applies each row's dequantisation scale to its scores;
//   D8: e4m3 cache with the query in two e4m3 terms (hi + lo on one scale
//       per head): both GEMMs on kind::f8f6f4 straight from the cache codes,
//       64-byte swizzled stages of half the size (twice as many), the
//       softmax weights written as two e4m3 terms with each row's scale
//       folded in relative to a running reference.
//
// What it computes ("DeepSeek-V2: MLA Explained", "MLA Full Formulas" part 3
// with the absorption of "Optimization Note"): for each head h of query row
// r and each cached row j of the split that the query sees,
//   z_j = scale * (q_abs[r,h,0:512] . c_j + q_abs[r,h,512:576] . k_j)
// then the split's normalised softmax-weighted mean of the latents c_j and
// its log-normaliser.
//
// How.  All heads share the cached rows, so both contractions are dense
// GEMMs per tile of 256 rows, issued for the CTA pair (cta_group::2) with
// M = 128 heads:
//   S[128 heads x 256 rows]  = Q[128 x 576] . K[256 x 576]^T    (N = 256)
//   O[128 heads x 512 dims] += P[128 x 256] . V[256 x 512]      (two MMAs of N = 256)
// With M = 128 over a pair, CTA r holds heads [64r, 64r+64) of Q (the A
// operand, 72 KB) and its TMEM receives S for those heads over all 256 rows
// of the tile: lanes 0-63 hold the 128 rows that CTA 0 loaded (the B operand
// is split by rows), lanes 64-127 the rows CTA 1 loaded.  The softmax of a
// head therefore never needs the other CTA: each of its four threads (two
// lane halves x two column halves) takes 64 scores, one page of the
// sequence, and they combine maxima and sums through shared memory.  Each
// thread writes its 64 probabilities as one 128-byte line of a K-major
// [64 heads x 64 rows] bf16 tile, the A operand of the value MMA for that
// page.  V is the B operand, split by dims: CTA r provides dims [128r,
// 128r+128) and [256+128r, 256+128r+128) of every row of the tile; its own
// rows come back from L2 (score loads are evict-last), the peer's rows were
// read from HBM by the peer.  The value MMAs accumulate O in TMEM, 128 lanes
// x 256 columns per CTA (lanes 0-63: the lower 128 dims of each 256-dim
// half, lanes 64-127: the upper 128).
//
// Cache rows stream through a ring of seven 16 KB shared-memory stages
// (e4m3: four, widened from six 8 KB staging slots of raw codes)
// filled by TMA (128-byte swizzle) in the order the MMA consumes them: per
// tile the nine score stages of tile i+1 follow the value stages of tile i,
// so the score GEMM runs a tile ahead of the value GEMM and the softmax of a
// tile overlaps the tensor work.  Pairs are persistent and claim (query
// row, split) units dynamically.  Every barrier wait is bounded: on a
// timeout the kernel flags MLA_DEVERR_TIMEOUT, lets its copies land, frees
// its tensor memory and returns.
//
// Warp roles per CTA: 0 TMA producer and TMEM allocator, 1 MMA issuer (the
// leader CTA issues for the pair), 2-9 softmax (warp w reads TMEM lanes
// 32 (w % 4) .. +31; warps 2-5 take score columns 0-63, warps 6-9 64-127),
// and with an e4m3 cache 10-13 converters (codes -> f16 operands).
//
// Hand-offs of shared-memory operands to the MMA issuer (P, and with an
// e4m3 cache Q and the widened stages) arrive on the leader's barriers with
// a CTA-scope release after a proxy fence: each CTA's half of a cta_group::2
// MMA reads that CTA's own shared memory on its own SM, so the leader only
// needs to know when to issue.  A cluster-scope release there stalled the
// arriving warp ~1.2K cycles (the e4m3 launch: 570 -> 425 us).
#include <math.h>

#include <mutex>

#include "mla_device.cuh"
#include "mla_internal.h"
#include "sm100.cuh"

namespace mla {
namespace {

using namespace sm100;

constexpr int kTile = 256;                // cached rows per pair tile (128 per CTA)
constexpr int kChunks = 9;                // 576 / 64 column chunks
constexpr int kHPC = 64;                  // heads per CTA
constexpr int kSlotBytes = 16384;         // one stage: one score chunk or one value box of this CTA
constexpr int kBox = 8192;                // [64 rows x 64 16-bit values]
constexpr int kBox8 = 4096;               // e4m3 cache: [64 rows x 64 codes]
constexpr int kStgBytes = 2 * kBox8;      // e4m3 cache: the raw codes of one stage
constexpr int kSlot8 = 2 * kBox8;         // 8-bit MMAs: one stage of codes ([128 rows x 64] or [64 rows x 128])
constexpr int kQ8Plane = kChunks * kBox8; // 8-bit MMAs: one term (hi or lo) of Q, 9 x [64 heads x 64 codes]
constexpr int kQChunk = kHPC * 128;       // [64 heads x 64 dims], 16-bit
constexpr int kPChunk = kHPC * 128;       // [64 heads x 64 rows], 16-bit: P of one page
constexpr int kWarpProd = 0, kWarpMma = 1, kWarpSoft0 = 2, kSoftWarps = 8;
constexpr int kWarpConv0 = kWarpSoft0 + kSoftWarps, kConvWarps = 4;   // e4m3 cache: converters
constexpr int kQN = 8;                    // unit queue depth
constexpr float kRescaleLog2 = 8.0f;      // lazy rescale threshold (log2 units)
constexpr float kRescaleLog2Q8 = 4.0f;    // 8-bit MMAs: probabilities stay <= 2^4, and times
constexpr float kPScale8 = 16.0f;         // 16 x row scale / reference <= 16 x 1.75 ...
constexpr float kScaleSlack8 = 1.75f;     // ... the reference is raised past 1.75x: <= 448
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kColS = 0;             // S of tile t at kColS + 128 (t & 1)
constexpr uint32_t kColO = 256;           // O: dims 0..255 at 256, dims 256..511 at 384

// offsets inside the misc area
constexpr int kMBars = 0;                 // 64 barriers
constexpr int kMTmem = 64 * 8;
constexpr int kMAbort = kMTmem + 4;
constexpr int kMRedMax = kMTmem + 16;     // float [2 tile parities][2 lane halves][2 column halves][64 heads]
constexpr int kMRedSum = kMRedMax + 2 * 4 * kHPC * 4;   // float [2 lane halves][2 column halves][64 heads]
constexpr int kMUnitQ = kMRedSum + 4 * kHPC * 4;
constexpr int kMStgSeq = kMUnitQ + 4 * kQN;   // int [8]: e4m3, the stage each staging slot was last filled for
constexpr int kMRedSc = kMStgSeq + 4 * 8;    // float [2 tile parities][8 softmax warps]: 8-bit MMAs
constexpr int kMiscBytes = kMRedSc + 4 * 2 * kSoftWarps;

// Shared memory, barriers and threads of the bf16 (F8 = D8 = false), the
// widening e4m3 (F8) and the 8-bit MMA e4m3 (D8) kernels.  With F8 the
// producer's copies land in a staging ring of raw codes and four converter
// warps widen them into the operand ring (one slot fewer, to make room for
// the staging).  With D8 the codes are the operands: stages are half the
// size, so the ring has twice the stages.
template <bool F8, bool D8 = false>
struct PairLayout {
  static_assert(!(F8 && D8), "one e4m3 form at a time");
  static constexpr int kSlotB = D8 ? kSlot8 : kSlotBytes;  // bytes of one operand stage
  static constexpr int kSlots = F8 ? kConvWarps : (D8 ? 14 : 7);   // operand ring stages
  static constexpr int kStg = F8 ? 6 : 0;                 // staging slots
  static constexpr int kThreads = 32 * (kWarpSoft0 + kSoftWarps + (F8 ? kConvWarps : 0));
  // bytes from the 1024-aligned base
  static constexpr int kOffQ = 0;                          // Q: 9 x 8 KB, K-major SW128 (D8: hi, lo 9 x 4 KB, SW64)
  static constexpr int kOffRing = kOffQ + kChunks * kQChunk;
  static constexpr int kOffP = kOffRing + kSlots * kSlotB;   // P: 4 pages x 8 KB (D8: hi, lo 4 KB each)
  static constexpr int kOffStg = kOffP + 4 * kPChunk;
  static constexpr int kOffMisc = kOffStg + kStg * kStgBytes;
  static constexpr int kSmem = kOffMisc + kMiscBytes + 1024;     // + alignment slack
  // barrier indices
  static constexpr int kBFull = 0;                  // [kSlots] leader: a stage is in both CTAs (TMA
                                                    // bytes; e4m3: the stage's converter warp of each CTA)
  static constexpr int kBEmpty = kSlots;            // [kSlots] both: the MMAs are done with the stage
  static constexpr int kBSFull = 2 * kSlots;        // [2] both: S of a tile is in TMEM
  static constexpr int kBODone = kBSFull + 2;       // both: the value MMAs of a tile are done
  static constexpr int kBPFull = kBODone + 1;       // leader: both CTAs' softmax wrote P (and rescaled O)
  static constexpr int kBQFull = kBPFull + 1;       // bf16: leader, both CTAs' Q landed; e4m3: local
  static constexpr int kBQFree = kBQFull + 1;       // both: the unit's score MMAs are done with Q
  static constexpr int kBEpiDone = kBQFree + 1;     // leader: both CTAs read O out (TMEM reusable)
  static constexpr int kBUqFull = kBEpiDone + 1;    // [kQN] both: unit queue slot written
  static constexpr int kBUqEmpty = kBUqFull + kQN;  // [kQN] leader: every consumer read the slot
  static constexpr int kBSoft = kBUqEmpty + kQN;    // [2] local: the softmax warps' own barriers
  static constexpr int kBStgFull = kBSoft + 2;      // [kStg] local: raw codes landed
  static constexpr int kBStgEmpty = kBStgFull + kStg;   // [kStg] local: the converters read them
  static constexpr int kBQReady = kBStgEmpty + kStg;    // leader: both CTAs' Q widened to f16
  static constexpr int kBEnd = kBQReady + 1;
  static_assert(kSmem <= 227 * 1024, "shared memory budget");
  static_assert(kBEnd <= 64, "barrier area");
  static_assert(kStg <= 8, "staging sequence area");
};

__device__ __forceinline__ int ld_acquire_shared(const int* p) {
  int v;
  asm volatile("ld.acquire.cta.shared::cta.b32 %0, [%1];" : "=r"(v) : "r"(smem_u32(p)) : "memory");
  return v;
}
__device__ __forceinline__ void st_release_shared(int* p, int v) {
  asm volatile("st.release.cta.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(p)), "r"(v) : "memory");
}

struct PairParams {
  int n_heads, q_len, batch;
  const int32_t* block_table;
  int max_pages, num_pages;
  const int32_t* seq_lens;
  int num_splits, split_tokens;
  int run;                     // splits per claimed unit (consecutive in (query row, split) order)
  float scale_log2;            // softmax_scale * log2(e)
  unsigned* claim;             // unit counter of this launch (0 at launch; reset by the last pair)
  unsigned* done;              // pairs finished
  float* o_part;
  float* lse_part;
  int32_t* err;
  unsigned long long wait_limit;
  int withhold_q;
  const float* cache_scale;    // e4m3 cache: per-row dequantisation scale [num_pages * 64]
  const float* q_scale;        // 8-bit MMAs: per (query row, head) scale of the two-term query [rows * n_heads]
};

// page id of a cached row of sequence b (0 for rows outside the table or the
// pool: those rows are masked, and page 0 is readable memory)
__device__ __forceinline__ int page_of(const PairParams& p, int b, int row, bool* ok) {
  const int pidx = row >> 6;
  int pg = -1;
  if (pidx < p.max_pages) pg = p.block_table[(size_t)b * p.max_pages + pidx];
  *ok = pg >= 0 && pg < p.num_pages;
  return *ok ? pg : 0;
}

__device__ __forceinline__ void st_cluster_b32(uint32_t addr, uint32_t v) {
  asm volatile("st.shared::cluster.b32 [%0], %1;" ::"r"(addr), "r"(v) : "memory");
}

__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
  const __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<const uint32_t*>(&v);
}
__device__ __forceinline__ uint32_t pack_f16(float lo, float hi) {
  const __half2 v = __floats2half2_rn(lo, hi);
  return *reinterpret_cast<const uint32_t*>(&v);
}

// tm_cache: boxes of one [64 rows x 64 columns] block (e4m3: [64 x 64 codes]);
// tm_cache2: boxes of two adjacent blocks (bf16 only); tm_q: q_abs boxes.
template <bool F8, bool D8 = false>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(PairLayout<F8, D8>::kThreads, 1)
    decode_pair_kernel(const __grid_constant__ CUtensorMap tm_cache, const __grid_constant__ CUtensorMap tm_cache2,
                       const __grid_constant__ CUtensorMap tm_q, const PairParams p) {
  using L = PairLayout<F8, D8>;
  constexpr int kSlots = L::kSlots, kStg = L::kStg;
  constexpr int kOffQ = L::kOffQ, kOffRing = L::kOffRing, kOffP = L::kOffP, kOffStg = L::kOffStg,
                kOffMisc = L::kOffMisc;
  constexpr int kBFull = L::kBFull, kBEmpty = L::kBEmpty, kBSFull = L::kBSFull, kBODone = L::kBODone,
                kBPFull = L::kBPFull, kBQFull = L::kBQFull, kBQFree = L::kBQFree, kBEpiDone = L::kBEpiDone,
                kBUqFull = L::kBUqFull, kBUqEmpty = L::kBUqEmpty, kBSoft = L::kBSoft, kBStgFull = L::kBStgFull,
                kBStgEmpty = L::kBStgEmpty, kBQReady = L::kBQReady;
  // queue readers: peer producer, MMA warp, softmax (and converter) warps of both CTAs
  constexpr int kQConsumers = 2 + 2 * kSoftWarps + (F8 ? 2 * kConvWarps : 0);
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t s_base = smem_u32(smem);
  const uint32_t s_q = s_base + kOffQ, s_ring = s_base + kOffRing;
  uint8_t* misc = smem + kOffMisc;
  const uint32_t s_misc = s_base + kOffMisc;
  auto bar = [&](int i) -> uint32_t { return s_misc + kMBars + 8 * i; };
  volatile int* abort_flag = reinterpret_cast<volatile int*>(misc + kMAbort);
  float* red_max = reinterpret_cast<float*>(misc + kMRedMax);
  float* red_sum = reinterpret_cast<float*>(misc + kMRedSum);
  float* red_sc = reinterpret_cast<float*>(misc + kMRedSc);
  int* unit_q = reinterpret_cast<int*>(misc + kMUnitQ);
  uint8_t* s_pbuf = smem + kOffP;
  const uint32_t s_p = s_base + kOffP;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint64_t lim = p.wait_limit;
  const uint32_t rank = cluster_rank();
  const uint32_t peer = rank ^ 1u;
  const bool leader = rank == 0;

  // ---- units: runs of `run` consecutive splits in (query row, split) order,
  // claimed by persistent pairs; a run that crosses into the next query row
  // is worked as two segments.  Every role walks the pair's same sequence of
  // segments, so barrier phases count globally (ring stages, tiles, segments).
  // A segment's splits are merged in TMEM: its partial is written at its
  // first split, and its other splits get lse = -inf (weight 0 in the merge).
  const int S = p.num_splits;
  const int n_flat = p.batch * p.q_len * S;
  const int n_units = (n_flat + p.run - 1) / p.run;
  const int n_pairs = gridDim.x >> 1;
  struct UnitInfo { int r, s, s1, b, lo, hi, n_tiles; };
  // the segment starting at flat split f of a unit that ends at f1
  auto seg_at = [&](int f, int f1) -> UnitInfo {
    UnitInfo x;
    x.r = f / S;
    x.s = f - x.r * S;
    x.s1 = min(S, x.s + (f1 - f));
    x.b = x.r / p.q_len;
    const int t = x.r % p.q_len;
    const int n_vis = p.seq_lens[x.b] - p.q_len + t + 1;
    x.lo = x.s * p.split_tokens;
    x.hi = (int)min((long long)x.s1 * p.split_tokens, (long long)n_vis);
    const int n_tok = x.hi - x.lo;
    x.n_tiles = n_tok > 0 ? (n_tok + kTile - 1) / kTile : 0;
    return x;
  };

  // ---- set-up
  if (threadIdx.x == 0) {
    for (int i = 0; i < kSlots; ++i) {
      mbar_init(bar(kBFull + i), F8 ? 2 : 1);
      mbar_init(bar(kBEmpty + i), 1);
    }
    for (int i = 0; i < kStg; ++i) {
      mbar_init(bar(kBStgFull + i), 1);
      mbar_init(bar(kBStgEmpty + i), 1);
    }
    if (F8) mbar_init(bar(kBQReady), 2 * kConvWarps);
    for (int i = 0; i < kStg; ++i) reinterpret_cast<int*>(misc + kMStgSeq)[i] = -1;
    mbar_init(bar(kBSFull), 1);
    mbar_init(bar(kBSFull + 1), 1);
    mbar_init(bar(kBODone), 1);
    mbar_init(bar(kBPFull), 2 * kSoftWarps);
    mbar_init(bar(kBQFull), 1);
    mbar_init(bar(kBQFree), 1);
    mbar_init(bar(kBEpiDone), 2 * kSoftWarps);
    for (int i = 0; i < kQN; ++i) {
      mbar_init(bar(kBUqFull + i), 1);
      mbar_init(bar(kBUqEmpty + i), kQConsumers);
    }
    mbar_init(bar(kBSoft), kSoftWarps);
    mbar_init(bar(kBSoft + 1), kSoftWarps);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == kWarpProd) tmem_alloc_pair(s_misc + kMTmem, kTmemCols);
  tc_fence_before();
  cluster_sync();
  tc_fence_after();
  const uint32_t tmem = *reinterpret_cast<volatile uint32_t*>(misc + kMTmem);
  // the set-up above may overlap the previous kernel on the stream; global
  // memory (the unit counter included) only after it has completed.  The
  // pair's first unit is claimed at once, so that the counter's round trip
  // overlaps the rest of the start.
  griddep_wait();
  griddep_launch_dependents();
  unsigned first_claim = 0;
  if (leader && threadIdx.x == 0) first_claim = atomicAdd(p.claim, 1u);

  // ---- the pair's unit sequence: the leader's producer claims units from the
  // launch's counter and posts them, in order, to a queue in both CTAs
  auto claim = [&](uint32_t k) -> int {      // leader producer, lane 0
    const uint32_t slot = k % kQN;
    if (k >= kQN && !mbar_wait(bar(kBUqEmpty + slot), ((k / kQN) - 1) & 1, abort_flag, lim)) return -2;
    const unsigned cu = k == 0 ? first_claim : atomicAdd(p.claim, 1u);
    const int uu = cu < (unsigned)n_units ? (int)cu : -1;
    *reinterpret_cast<volatile int*>(unit_q + slot) = uu;
    st_cluster_b32(mapa(smem_u32(unit_q + slot), peer), (uint32_t)uu);
    mbar_arrive_cluster(bar(kBUqFull + slot));
    mbar_arrive_cluster(mapa(bar(kBUqFull + slot), peer));
    return uu;
  };
  auto next_unit = [&](uint32_t k) -> int {  // whole warp
    const uint32_t slot = k % kQN;
    if (!__all_sync(0xffffffffu, mbar_wait(bar(kBUqFull + slot), (k / kQN) & 1, abort_flag, lim))) return -2;
    const int uu = *reinterpret_cast<volatile int*>(unit_q + slot);
    __syncwarp();
    if (lane == 0) mbar_arrive_cluster(mapa(bar(kBUqEmpty + slot), 0));
    return uu;
  };

  uint32_t kc = 0;   // ring stages handed out (producer) or consumed (MMA)
  if (warp == kWarpProd) {
    // ============ TMA producer (both CTAs), in the order the MMA consumes ============
    // S(0), then per tile i: S(i+1), O(i).  The pool is page-blocked (nine
    // contiguous [64 rows x 64 columns] blocks per page), viewed as 2-D
    // [blocks * 64 lines x 64 columns].  A score stage is column chunk c of
    // this CTA's two pages of the tile (block c of each page, 8 KB each);
    // a value stage is one page's pair of dims blocks 4 bb + 2 r, +1 of this
    // CTA (one contiguous 16 KB box).  e4m3 cache: the same blocks as raw
    // codes (4 KB each) into a staging slot of this CTA, for the converters.
    if (lane == 0) {
      tma_prefetch_desc(&tm_cache);
      if (!F8) tma_prefetch_desc(&tm_cache2);
      tma_prefetch_desc(&tm_q);
    }
    // score rows are re-read by the value stages of the pair (this CTA's for
    // its dims, the peer's for the other dims) one tile later: evict-last;
    // value loads are the rows' last use: evict-first
    const uint64_t pol_keep = policy_evict_last();
    const uint64_t pol_drop = policy_evict_first();
    uint32_t uc = 0;
    bool ok = true;
    for (uint32_t k = 0; ok; ++k) {
      int u;
      if (leader) {
        int uu = 0;
        if (lane == 0) uu = claim(k);
        u = __shfl_sync(0xffffffffu, uu, 0);
      } else {
        u = next_unit(k);
      }
      if (u == -2) { ok = false; break; }
      if (u < 0) break;
      const int f1 = min(n_flat, (u + 1) * p.run);
      for (int f = u * p.run; f < f1 && ok;) {
      const UnitInfo U = seg_at(f, f1);
      f += U.s1 - U.s;
      if (U.n_tiles == 0) continue;
      const int r = U.r, b = U.b, lo = U.lo, hi = U.hi, n_tiles = U.n_tiles;
      if (lane == 0) {
        // the previous unit's score MMAs must be done with Q (both halves)
        if (uc > 0) ok = mbar_wait<false>(bar(kBQFree), (uc - 1) & 1, abort_flag, lim);
        // (test hook: the leader leaves the query load of its first unit out,
        // so the MMA issuer's wait for it runs out and the launch aborts)
        if (ok && !(p.withhold_q && leader && uc == 0)) {
          if constexpr (F8) {
            // each CTA's half lands on its own barrier; the converters widen it to f16
            mbar_arrive_expect_tx(bar(kBQFull), kChunks * kQChunk);
            for (int c = 0; c < kChunks; ++c)
              tma_load_3d(s_q + c * kQChunk, &tm_q, 64 * c, (int)rank * kHPC, r, bar(kBQFull));
          } else if constexpr (D8) {
            // both terms of the query (planes 2r and 2r + 1 of the map), 64-byte swizzled
            const uint32_t q_bar = mapa(bar(kBQFull), 0);
            if (leader) mbar_arrive_expect_tx(bar(kBQFull), 2u * 2u * kQ8Plane);
            for (int hl = 0; hl < 2; ++hl)
              for (int c = 0; c < kChunks; ++c)
                tma_load_3d_pair(s_q + hl * kQ8Plane + c * kBox8, &tm_q, 64 * c, (int)rank * kHPC, 2 * r + hl, q_bar);
          } else {
            const uint32_t q_bar = mapa(bar(kBQFull), 0);
            if (leader) mbar_arrive_expect_tx(bar(kBQFull), 2u * kChunks * kQChunk);
            for (int c = 0; c < kChunks; ++c)
              tma_load_3d_pair(s_q + c * kQChunk, &tm_q, 64 * c, (int)rank * kHPC, r, q_bar);
          }
        }
      }
      ok = __shfl_sync(0xffffffffu, ok, 0);
      if (!ok) break;
      // One lane issues every copy of the segment: a per-stage hand-off
      // between lanes (shuffles, a converged wait) cost ~4 % of the launch.
      // The table entries of tile i + 2 are fetched while tile i is issued,
      // so their latency stays off the stream.
      if (lane == 0) {
        const int32_t* bt = p.block_table + (size_t)b * p.max_pages;
        const int pb = lo >> 6;      // the segment's first page index (lo is a multiple of 64)
        auto entry = [&](int pidx) -> int { return pidx < p.max_pages ? __ldg(bt + pidx) : -1; };
        // rows outside the table or the pool read page 0 (readable; they are masked)
        auto page = [&](int pg) -> int { return pg >= 0 && pg < p.num_pages ? pg : 0; };
        auto take = [&](uint32_t& dst, uint32_t& fb) -> bool {
          if constexpr (F8) {
            const uint32_t slot = kc % kStg;
            const uint32_t ph = (kc / kStg) & 1u;
            if (!mbar_wait<false>(bar(kBStgEmpty + slot), ph ^ 1u, abort_flag, lim)) return false;
            mbar_arrive_expect_tx(bar(kBStgFull + slot), kStgBytes);
            // the converter of this stage checks this before its parity wait (see there)
            st_release_shared(reinterpret_cast<int*>(misc + kMStgSeq) + slot, (int)kc);
            dst = s_base + kOffStg + slot * kStgBytes;
            fb = bar(kBStgFull + slot);
          } else {
            const uint32_t slot = kc % kSlots;
            const uint32_t ph = (kc / kSlots) & 1u;
            if (!mbar_wait<false>(bar(kBEmpty + slot), ph ^ 1u, abort_flag, lim)) return false;
            if (leader) mbar_arrive_expect_tx(bar(kBFull + slot), 2u * L::kSlotB);
            dst = s_ring + slot * L::kSlotB;
            fb = mapa(bar(kBFull + slot), 0);
          }
          ++kc;
          return true;
        };
        // score stages: column chunk c of this CTA's two pages of the tile
        auto load_s = [&](int pg0, int pg1) -> bool {
          for (int c = 0; c < kChunks; ++c) {
            uint32_t dst, fb;
            if (!take(dst, fb)) return false;
            if constexpr (F8) {
              tma_load_2d_hint(dst, &tm_cache, 0, (pg0 * kChunks + c) * 64, fb, pol_keep);
              tma_load_2d_hint(dst + kBox8, &tm_cache, 0, (pg1 * kChunks + c) * 64, fb, pol_keep);
            } else {
              tma_load_2d_pair_hint(dst, &tm_cache, 0, (pg0 * kChunks + c) * 64, fb, pol_keep);
              tma_load_2d_pair_hint(dst + (D8 ? kBox8 : kBox), &tm_cache, 0, (pg1 * kChunks + c) * 64, fb, pol_keep);
            }
          }
          return true;
        };
        // value stages: per page of tile j with visible rows, this CTA's two dims blocks pairs
        auto load_o = [&](int j, const int (&pg)[4]) -> bool {
#pragma unroll
          for (int pg_i = 0; pg_i < 4; ++pg_i) {
            if (lo + kTile * j + 64 * pg_i >= hi) break;
            for (int bb = 0; bb < 2; ++bb) {
              uint32_t dst, fb;
              if (!take(dst, fb)) return false;
              const int line = (pg[pg_i] * kChunks + 4 * bb + 2 * (int)rank) * 64;
              if constexpr (F8) {
                tma_load_2d_hint(dst, &tm_cache, 0, line, fb, pol_drop);
                tma_load_2d_hint(dst + kBox8, &tm_cache, 0, line + 64, fb, pol_drop);
              } else {
                tma_load_2d_pair_hint(dst, &tm_cache2, 0, line, fb, pol_drop);
              }
            }
          }
          return true;
        };
        int cur[4], nxt[4];
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          cur[q] = entry(pb + q);
          nxt[q] = entry(pb + 4 + q);
        }
        ok = load_s(page(rank ? cur[2] : cur[0]), page(rank ? cur[3] : cur[1]));
        for (int i = 0; i < n_tiles && ok; ++i) {
          int ahead[4];
#pragma unroll
          for (int q = 0; q < 4; ++q) ahead[q] = entry(pb + 4 * (i + 2) + q);
          if (i + 1 < n_tiles) ok = load_s(page(rank ? nxt[2] : nxt[0]), page(rank ? nxt[3] : nxt[1]));
          int pg[4];
#pragma unroll
          for (int q = 0; q < 4; ++q) pg[q] = page(cur[q]);
          if (ok) ok = load_o(i, pg);
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            cur[q] = nxt[q];
            nxt[q] = ahead[q];
          }
        }
      }
      ok = __shfl_sync(0xffffffffu, ok, 0);
      ++uc;
      }
    }
  } else if (warp == kWarpMma) {
    // ================= MMA issuer (leader CTA, whole warp, one elected lane) =================
    // Per unit: S(0), then per tile i: S(i+1), O(i).  S(i+1) goes to the other
    // TMEM buffer while the softmax of tile i reads S(i); S(i+2) reuses S(i)'s
    // columns after O(i), which waited for the softmax of tile i to finish
    // (tcgen05.mma operations of one thread execute in issue order).  The
    // value GEMM of tile i waits for P(i), which the softmax writes after
    // O(i-1) is done (one P buffer), so running the score GEMM further ahead
    // only delays O(i) (measured slower).
    if (leader) {
      // F8: the operands are f16 (widened codes, Q and P in f16); D8: e4m3
      constexpr uint32_t idS = D8 ? idesc_e4m3(128, 256, false, false) : idesc_f16(128, 256, false, false, F8);
      constexpr uint32_t idO = D8 ? idesc_e4m3(128, 256, false, true) : idesc_f16(128, 256, false, true, F8);
      auto ready = [&](uint32_t& src, uint32_t& empty) -> bool {
        const uint32_t slot = kc % kSlots;
        const uint32_t ph = (kc / kSlots) & 1u;
        if (!__all_sync(0xffffffffu, mbar_wait<false>(bar(kBFull + slot), ph, abort_flag, lim))) return false;
        tc_fence_after();
        src = s_ring + slot * L::kSlotB;
        empty = bar(kBEmpty + slot);
        ++kc;
        return true;
      };
      uint32_t uc = 0, gt = 0;
      bool ok = true;
      for (uint32_t k = 0; ok; ++k) {
        const int u = next_unit(k);
        if (u == -2) { ok = false; break; }
        if (u < 0) break;
        const int f1 = min(n_flat, (u + 1) * p.run);
        for (int f = u * p.run; f < f1 && ok;) {
        const UnitInfo U = seg_at(f, f1);
        f += U.s1 - U.s;
        if (U.n_tiles == 0) continue;
        const int lo = U.lo, hi = U.hi, n_tiles = U.n_tiles;
        ok = __all_sync(0xffffffffu, mbar_wait<false>(bar(F8 ? kBQReady : kBQFull), uc & 1, abort_flag, lim));
        if (!ok) break;
        tc_fence_after();
        auto issue_s = [&](int i) -> bool {
          const uint32_t t = gt + i;
          const uint32_t sb = t & 1u;
          const uint32_t d = tmem + kColS + 128 * sb;
          for (int c = 0; c < kChunks; ++c) {
            uint32_t a0, empty;
            if (!ready(a0, empty)) return false;
            if constexpr (D8) {
              // K = 32 codes per MMA (+32 bytes along the 64-byte lines), both
              // query terms into the same accumulator
              const uint64_t qd = smem_desc_sw64(s_q, 16, 512);
              const uint64_t kd = smem_desc_sw64(a0, 16, 512);
#pragma unroll
              for (int ks = 0; ks < 2; ++ks)
#pragma unroll
                for (int hl = 0; hl < 2; ++hl)
                  mma_pair_e4m3_w(d, qd + ((hl * kQ8Plane + c * kBox8 + ks * 32) >> 4), kd + ((ks * 32) >> 4), idS,
                                  (c | ks | hl) != 0);
            } else {
              const uint64_t qd = smem_desc_sw128(s_q, 16, 1024);
              const uint64_t kd = smem_desc_sw128(a0, 16, 1024);
#pragma unroll
              for (int ks = 0; ks < 4; ++ks)   // K = 16 per MMA: +32 bytes along the 128-byte lines
                mma_pair_f16_w(d, qd + ((c * kQChunk + ks * 32) >> 4), kd + ((ks * 32) >> 4), idS, (c | ks) != 0);
            }
            mma_commit_pair_w(empty, 0x3);
          }
          mma_commit_pair_w(bar(kBSFull + sb), 0x3);
          // the unit's last score GEMM: Q may be replaced once it completes
          if (i == n_tiles - 1) mma_commit_pair_w(bar(kBQFree), 0x3);
          return true;
        };
        auto issue_o = [&](int j) -> bool {
          const uint32_t t = gt + j;
          if (!__all_sync(0xffffffffu, mbar_wait<false>(bar(kBPFull), t & 1, abort_flag, lim))) return false;
          // the accumulator is overwritten by this unit's first value MMA: the
          // previous unit's epilogue must have read it out
          if (j == 0 && uc > 0 &&
              !__all_sync(0xffffffffu, mbar_wait(bar(kBEpiDone), (uc - 1) & 1, abort_flag, lim)))
            return false;
          tc_fence_after();
          for (int pg_i = 0; pg_i < 4; ++pg_i) {
            if (lo + kTile * j + 64 * pg_i >= hi) break;
            for (int bb = 0; bb < 2; ++bb) {
              uint32_t b0, empty;
              if (!ready(b0, empty)) return false;
              if constexpr (D8) {
                // 32 rows per MMA: +32 bytes of the P lines, +2 KB of V (8-row
                // groups of 512 bytes); the stage's two 64-dim blocks 4 KB apart;
                // both probability terms into the same accumulator
                const uint64_t pd = smem_desc_sw64(s_p, 16, 512);
                const uint64_t vd = smem_desc_sw64(b0, kBox8, 512);
#pragma unroll
                for (int ks = 0; ks < 2; ++ks)
#pragma unroll
                  for (int hl = 0; hl < 2; ++hl)
                    mma_pair_e4m3_w(tmem + kColO + 128 * bb, pd + ((pg_i * kPChunk + hl * kBox8 + ks * 32) >> 4),
                                    vd + ((ks * 2048) >> 4), idO, (j | pg_i | ks | hl) != 0);
              } else {
                const uint64_t pd = smem_desc_sw128(s_p, 16, 1024);
                const uint64_t vd = smem_desc_sw128(b0, kBox, 1024);
#pragma unroll
                for (int ks = 0; ks < 4; ++ks)   // 16 rows per MMA: +32 bytes of P lines, +2 KB of V lines
                  mma_pair_f16_w(tmem + kColO + 128 * bb, pd + ((pg_i * kPChunk + ks * 32) >> 4),
                                 vd + ((ks * 2048) >> 4), idO, (j | pg_i | ks) != 0);
              }
              mma_commit_pair_w(empty, 0x3);
            }
          }
          mma_commit_pair_w(bar(kBODone), 0x3);
          return true;
        };
        ok = issue_s(0);
        for (int i = 0; i < n_tiles && ok; ++i) {
          if (i + 1 < n_tiles) ok = issue_s(i + 1);
          if (ok) ok = issue_o(i);
        }
        gt += n_tiles;
        ++uc;
        }
      }
    }
  } else if (warp < kWarpConv0) {
    // ================= softmax (both CTAs, warps 2-9) =================
    // Thread (lane quadrant q4, column half ch, lane) owns head hh = 32 (q4 & 1)
    // + lane of this CTA and the 64 tile rows 128 (q4 >> 1) + 64 ch .. +63.
    const int q4 = warp & 3;
    const int half = q4 >> 1;                   // 0: TMEM lanes 0-63, 1: lanes 64-127
    const int hh = 32 * (q4 & 1) + lane;        // head within this CTA
    const int head = kHPC * (int)rank + hh;
    const int ch = (warp - kWarpSoft0) >> 2;    // score columns [64 ch, 64 ch + 64)
    const uint32_t lane_addr = static_cast<uint32_t>(32 * q4) << 16;
    const int part = 2 * half + ch;             // which of the head's four partial results (= page of the tile)
    // barriers among the eight softmax warps, on mbarriers so that every wait
    // is bounded: a warp that leaves on a timeout cannot strand the others
    uint32_t soft_ph[2] = {0, 0};
    auto soft_sync = [&](int which) -> bool {
      __syncwarp();
      if (lane == 0) mbar_arrive_local(bar(kBSoft + which));
      const bool okk = __all_sync(0xffffffffu, mbar_wait<false>(bar(kBSoft + which), soft_ph[which] & 1,
                                                                abort_flag, lim));
      ++soft_ph[which];
      return okk;
    };
    uint32_t uc = 0, gt = 0;
    bool ok = true;
    for (uint32_t k = 0; ok; ++k) {
      const int u = next_unit(k);
      if (u == -2) { ok = false; break; }
      if (u < 0) break;
      const int f1 = min(n_flat, (u + 1) * p.run);
      for (int f = u * p.run; f < f1 && ok;) {
      const UnitInfo U = seg_at(f, f1);
      f += U.s1 - U.s;
      const int r = U.r, s = U.s, b = U.b, lo = U.lo, hi = U.hi, n_tiles = U.n_tiles;
      // splits of the segment after its first: merged into the first (lse = -inf,
      // o_part unwritten: the merge gives them weight 0 and does not read them)
      if (part == 0 && head < p.n_heads)
        for (int s2 = s + 1; s2 < U.s1; ++s2) p.lse_part[((size_t)r * p.n_heads + head) * S + s2] = -INFINITY;
      if (n_tiles == 0) {
        // nothing visible in the segment: lse = -inf at its first split too
        if (part == 0 && head < p.n_heads) p.lse_part[((size_t)r * p.n_heads + head) * S + s] = -INFINITY;
        continue;
      }
      // D8: the scores are (q scale of the head) x (row scale) x the code
      // GEMM.  The weights of the value GEMM carry each row's scale relative
      // to a reference s_ref, times 16: s_ref is the largest row scale seen so
      // far in the segment, raised (with O rescaled) only when a tile's rows
      // exceed it by 1.75x, so every weight stays <= 16 x 16 x 1.75 = 448.
      // O is multiplied by s_ref / 16 in the epilogue.
      float slq = p.scale_log2, s_ref = 0.f;
      if constexpr (D8) {
        if (head < p.n_heads) slq *= __ldg(p.q_scale + (size_t)r * p.n_heads + head);
      }
      float m_run = -INFINITY, l_acc = 0.f;
      for (int i = 0; i < n_tiles; ++i) {
        const uint32_t t = gt + i;
        const uint32_t sb = t & 1u;
        // rows of this thread: one page of the sequence (its table entry is
        // read before the wait for the scores, off the critical path)
        const int row0 = lo + kTile * i + 128 * half + 64 * ch;
        int nvalid = min(max(hi - row0, 0), 64);
        float sc_lo = 1.f, sc_hi = 1.f;   // e4m3: the page's dequantisation scales (lane l: rows l, l + 32)
        if (nvalid > 0) {
          bool pok;
          const int pg = page_of(p, b, row0, &pok);
          if (!pok) {
            nvalid = 0;
            flag_error(p.err, MLA_DEVERR_PAGE);
          } else if constexpr (F8 || D8) {
            sc_lo = __ldg(p.cache_scale + (size_t)pg * 64 + lane);
            sc_hi = __ldg(p.cache_scale + (size_t)pg * 64 + 32 + lane);
          }
        }
        ok = __all_sync(0xffffffffu, mbar_wait<false>(bar(kBSFull + sb), (t >> 1) & 1, abort_flag, lim));
        if (!ok) break;
        tc_fence_after();
        const uint32_t scol = tmem + lane_addr + kColS + 128 * sb;
        float v[64];
        tmem_ld<32>(scol + 64 * ch, v);
        tmem_ld<32>(scol + 64 * ch + 32, v + 32);
        tmem_wait_ld();
        float mx = -INFINITY;
#pragma unroll
        for (int j = 0; j < 64; ++j) {
          float sl = slq;
          if constexpr (F8 || D8) sl *= __shfl_sync(0xffffffffu, j < 32 ? sc_lo : sc_hi, j & 31);
          v[j] = j < nvalid ? v[j] * sl : -INFINITY;
          mx = fmaxf(mx, v[j]);
        }
        // the four partial maxima of each head, double-buffered by tile parity:
        // a warp writes the next tile's slot only after passing this tile's
        // sync, so no warp can overwrite a slot that another is still reading
        float* rm = red_max + sb * 4 * kHPC;
        rm[part * kHPC + hh] = mx;
        if constexpr (D8) {   // the largest scale of this warp's visible rows, same buffering
          float tsm = fmaxf(lane < nvalid ? sc_lo : 0.f, lane + 32 < nvalid ? sc_hi : 0.f);
#pragma unroll
          for (int o = 16; o > 0; o >>= 1) tsm = fmaxf(tsm, __shfl_xor_sync(0xffffffffu, tsm, o));
          if (lane == 0) red_sc[sb * kSoftWarps + (warp - kWarpSoft0)] = tsm;
        }
        if (!(ok = soft_sync(0))) break;
        const float tmax = fmaxf(fmaxf(rm[hh], rm[kHPC + hh]), fmaxf(rm[2 * kHPC + hh], rm[3 * kHPC + hh]));
        const float m_new = (tmax > m_run + (D8 ? kRescaleLog2Q8 : kRescaleLog2)) ? tmax : m_run;
        const bool changed = m_new != m_run;
        // factor for the sums and the accumulator kept so far (0 when nothing was kept)
        const float alpha = (m_run == -INFINITY) ? 0.f : exp2_approx(m_run - m_new);
        m_run = m_new;
        const float msub = m_new == -INFINITY ? 0.f : m_new;
        float w_k = 0.f, s_fac = 1.f;   // D8: weight factor 16 / s_ref; O's factor for a raised s_ref
        bool s_up = false;
        if constexpr (D8) {
          const float* rs = red_sc + sb * kSoftWarps;
          float tsmax = rs[0];
#pragma unroll
          for (int w = 1; w < kSoftWarps; ++w) tsmax = fmaxf(tsmax, rs[w]);
          if (tsmax > kScaleSlack8 * s_ref) {
            s_up = s_ref > 0.f;
            s_fac = s_up ? s_ref / tsmax : 1.f;
            s_ref = tsmax;
          }
          w_k = s_ref > 0.f ? kPScale8 / s_ref : 0.f;
        }
        uint32_t pk[32];   // D8: pk[0..15] the hi codes of the 64 rows, pk[16..31] the lo codes
        float sum = 0.f;
        if constexpr (D8) {
          const float wlo = sc_lo * w_k, whi = sc_hi * w_k;
#pragma unroll
          for (int j = 0; j < 32; ++j) {
            const float p0 = exp2_approx(v[2 * j] - msub), p1 = exp2_approx(v[2 * j + 1] - msub);
            sum += p0 + p1;
            const float x0 = p0 * __shfl_sync(0xffffffffu, 2 * j < 32 ? wlo : whi, (2 * j) & 31);
            const float x1 = p1 * __shfl_sync(0xffffffffu, 2 * j + 1 < 32 ? wlo : whi, (2 * j + 1) & 31);
            uint32_t h2, l2;
            split_e4m3x2(x0, x1, h2, l2);
            if (j & 1) {
              pk[j >> 1] |= h2 << 16;
              pk[16 + (j >> 1)] |= l2 << 16;
            } else {
              pk[j >> 1] = h2;
              pk[16 + (j >> 1)] = l2;
            }
          }
        } else {
#pragma unroll
          for (int j = 0; j < 32; ++j) {
            const float p0 = exp2_approx(v[2 * j] - msub), p1 = exp2_approx(v[2 * j + 1] - msub);
            sum += p0 + p1;
            pk[j] = F8 ? pack_f16(p0, p1) : pack_bf16(p0, p1);
          }
        }
        l_acc = changed ? fmaf(l_acc, alpha, sum) : l_acc + sum;
        // every phase of o_done is observed in order (a parity wait cannot
        // tell a phase two behind from a completed one); O(i-1) done also
        // frees the P tiles for this tile's probabilities
        if (i >= 1) {
          ok = __all_sync(0xffffffffu, mbar_wait<false>(bar(kBODone), (t - 1) & 1, abort_flag, lim));
          if (!ok) break;
          tc_fence_after();
          if (s_up || __any_sync(0xffffffffu, changed)) {
            const float f = (changed ? alpha : 1.f) * s_fac;
            const uint32_t oc = tmem + lane_addr + kColO + 128 * ch;
#pragma unroll 1
            for (int c4 = 0; c4 < 4; ++c4) {
              float o[32];
              tmem_ld<32>(oc + 32 * c4, o);
              tmem_wait_ld();
#pragma unroll
              for (int j = 0; j < 32; ++j) o[j] *= f;
              tmem_st<32>(oc + 32 * c4, o);
            }
          }
        }
        // P of this thread's 64 rows (one page of the tile): line hh of the
        // page's K-major [64 heads x 64 rows] tile, 128-byte swizzled (D8: a
        // 64-byte line in each of the hi and lo tiles, 64-byte swizzled)
        if constexpr (D8) {
#pragma unroll
          for (int hl = 0; hl < 2; ++hl) {
            uint8_t* line = s_pbuf + part * kPChunk + hl * kBox8 + hh * 64;
#pragma unroll
            for (int q = 0; q < 4; ++q)
              *reinterpret_cast<uint4*>(line + ((q ^ ((hh >> 1) & 3)) << 4)) =
                  make_uint4(pk[16 * hl + 4 * q], pk[16 * hl + 4 * q + 1], pk[16 * hl + 4 * q + 2],
                             pk[16 * hl + 4 * q + 3]);
          }
        } else {
          uint8_t* line = s_pbuf + part * kPChunk + hh * 128;
#pragma unroll
          for (int q = 0; q < 8; ++q)
            *reinterpret_cast<uint4*>(line + ((q ^ (hh & 7)) << 4)) =
                make_uint4(pk[4 * q], pk[4 * q + 1], pk[4 * q + 2], pk[4 * q + 3]);
        }
        fence_proxy_async_cta();     // read by the tensor core
        tmem_wait_st();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive_cluster_cta(mapa(bar(kBPFull), 0));
      }
      // ---- epilogue: normalise O by the row sums, write o_part and lse
      if (ok) ok = __all_sync(0xffffffffu, mbar_wait<false>(bar(kBODone), (gt + n_tiles - 1) & 1, abort_flag, lim));
      if (ok) {
        tc_fence_after();
        red_sum[part * kHPC + hh] = l_acc;
        ok = soft_sync(0);
      }
      if (ok) {
        const float lt = red_sum[hh] + red_sum[kHPC + hh] + red_sum[2 * kHPC + hh] + red_sum[3 * kHPC + hh];
        const float inv_l = lt > 0.f ? (D8 ? s_ref / kPScale8 : 1.f) / lt : 0.f;
        if (part == 0 && head < p.n_heads)
          p.lse_part[((size_t)r * p.n_heads + head) * S + s] =
              lt > 0.f ? (m_run + log2f(lt)) * 0.69314718055994531f : -INFINITY;
        // this thread's O: dims 256 ch + 128 half + (0..127) of head `head`,
        // stored 32 dims at a time through a 4 KB [32 heads x 32 dims] tile
        // of this warp in the P area (idle until the next unit's first
        // probabilities, which these warps write): a store instruction then
        // covers four whole 128-byte lines (four heads) instead of 32 pieces
        // of 32 lines
        const uint32_t oc = tmem + lane_addr + kColO + 128 * ch;
        uint8_t* tile = s_pbuf + (warp - kWarpSoft0) * 4096;
        const int rd_head = lane >> 3, rd_q = lane & 7;   // reader: head 4 k + rd_head, 16-byte piece rd_q
        const int head0 = kHPC * (int)rank + 32 * (q4 & 1);   // this warp's first head
        const size_t head_stride = (size_t)S * MLA_D_C;         // floats between heads in o_part
        // the reader's first head (head0 + rd_head) at dims 256 ch + 128 half + 4 rd_q
        float* const o_rd = p.o_part + (((size_t)r * p.n_heads + head0 + rd_head) * S + s) * MLA_D_C + 256 * ch +
                            128 * half + 4 * rd_q;
#pragma unroll 1
        for (int c4 = 0; c4 < 4; ++c4) {
          float o[32];
          tmem_ld<32>(oc + 32 * c4, o);
          tmem_wait_ld();
#pragma unroll
          for (int q = 0; q < 8; ++q)
            *reinterpret_cast<float4*>(tile + lane * 128 + ((q ^ (lane & 7)) << 4)) =
                make_float4(o[4 * q] * inv_l, o[4 * q + 1] * inv_l, o[4 * q + 2] * inv_l, o[4 * q + 3] * inv_l);
          __syncwarp();
          float* op = o_rd + 32 * c4;
#pragma unroll 4
          for (int k4 = 0; k4 < 8; ++k4, op += 4 * head_stride) {
            const int j = 4 * k4 + rd_head;                    // head of this warp
            if (head0 + j < p.n_heads)
              *reinterpret_cast<float4*>(op) =
                  *reinterpret_cast<const float4*>(tile + j * 128 + ((rd_q ^ (j & 7)) << 4));
          }
          __syncwarp();
        }
        // this warp's part of O has been read: the pair's next unit may overwrite it
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive_cluster(mapa(bar(kBEpiDone), 0));
      }
      gt += n_tiles;
      ++uc;
      }
    }
  } else {
    // ============ e4m3 -> f16 converters (both CTAs, warps 10-13) ============
    // Per segment: Q (bf16 -> f16 in place, all four warps), then the stages
    // in the MMA's order, dealt round robin: warp w converts stages w, w + 4,
    // ... into operand slot w.  For its stage a warp waits for the staging
    // slot's codes and the operand slot's release, widens the codes exactly
    // (every e4m3 value is an f16 value), writes them 128-byte swizzled like
    // the bf16 copies, makes them visible to the tensor core and arrives on
    // the leader's full barrier.  Value stages are also multiplied by the
    // row's dequantisation scale (an f16 product); scores get the scale in
    // the softmax instead.
    if constexpr (F8) {
      const int cw = warp - kWarpConv0;               // 0..3
      const int ct = threadIdx.x - 32 * kWarpConv0;   // 0..127
      constexpr int kCT = 32 * kConvWarps;
      uint32_t uc = 0;
      bool ok = true;
      for (uint32_t k = 0; ok; ++k) {
        const int u = next_unit(k);
        if (u == -2) { ok = false; break; }
        if (u < 0) break;
        const int f1 = min(n_flat, (u + 1) * p.run);
        for (int f = u * p.run; f < f1 && ok;) {
        const UnitInfo U = seg_at(f, f1);
        f += U.s1 - U.s;
        if (U.n_tiles == 0) continue;
        const int b = U.b, lo = U.lo, hi = U.hi, n_tiles = U.n_tiles;
        if (!(ok = __all_sync(0xffffffffu, mbar_wait<false>(bar(kBQFull), uc & 1, abort_flag, lim)))) break;
        for (int i = ct; i < kChunks * kQChunk / 16; i += kCT) {
          uint4 v = *reinterpret_cast<const uint4*>(smem + kOffQ + 16 * i);
          uint32_t* w = reinterpret_cast<uint32_t*>(&v);
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const float2 f2 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&w[e]));
            w[e] = pack_f16(f2.x, f2.y);
          }
          *reinterpret_cast<uint4*>(smem + kOffQ + 16 * i) = v;
        }
        fence_proxy_async_cta();     // read by the tensor core
        __syncwarp();
        if (lane == 0) mbar_arrive_cluster_cta(mapa(bar(kBQReady), 0));
        // one stage: two [64 x 64] blocks of codes -> two [64 x 64] f16 blocks;
        // lane l handles 16 codes of rows (l >> 2) + 8 i, i = 0..15 (8 per block)
        auto convert = [&](int scale_page) -> bool {
          const uint32_t my = kc++;
          if ((int)(my % kConvWarps) != cw) return true;   // another warp's stage
          const uint32_t slot = my % kSlots, ph = (my / kSlots) & 1u;
          const uint32_t ss = my % kStg, sph = (my / kStg) & 1u;
          // value stage: lane l holds the scales of rows l and l + 32 of the page
          float s_lo = 1.f, s_hi = 1.f;
          if (scale_page >= 0) {
            s_lo = __ldg(p.cache_scale + (size_t)scale_page * 64 + lane);
            s_hi = __ldg(p.cache_scale + (size_t)scale_page * 64 + 32 + lane);
          }
          // Staging slots are shared by the converter warps (stage my uses slot
          // my % kStg, warp my % kConvWarps), so this warp may get here while the
          // slot's previous fill (stage my - kStg, another warp's) is still
          // pending; a parity wait would then match the phase before that and
          // pass early.  The producer records each fill's stage once the slot is
          // free again, which is after its previous phase completed: wait for that.
          {
            const int* seq = reinterpret_cast<const int*>(misc + kMStgSeq) + ss;
            const uint64_t t0 = clock64();
            bool okw = true;
            for (uint32_t n = 1; ld_acquire_shared(seq) != (int)my; ++n) {
              if ((n & 255u) == 0 && (*abort_flag || clock64() - t0 > lim)) {
                *abort_flag = 1;
                okw = false;
                break;
              }
            }
            if (!__all_sync(0xffffffffu, okw)) return false;
          }
          if (!__all_sync(0xffffffffu, mbar_wait<false>(bar(kBStgFull + ss), sph, abort_flag, lim))) return false;
          if (!__all_sync(0xffffffffu, mbar_wait<false>(bar(kBEmpty + slot), ph ^ 1u, abort_flag, lim))) return false;
          const uint8_t* src = smem + kOffStg + ss * kStgBytes;
          uint8_t* dst = smem + kOffRing + slot * kSlotBytes;
          const int qq = lane & 3;
#pragma unroll
          for (int i = 0; i < 16; ++i) {
            const int box = i >> 3, row = (lane >> 2) + 8 * (i & 7);
            const uint4 codes = *reinterpret_cast<const uint4*>(src + box * kBox8 + row * 64 + qq * 16);
            const uint32_t* cwd = reinterpret_cast<const uint32_t*>(&codes);
            const float sr = __shfl_sync(0xffffffffu, row < 32 ? s_lo : s_hi, row & 31);
            const __half2 rs2 = __float2half2_rn(sr);
            uint32_t hw[8];
#pragma unroll
            for (int e = 0; e < 4; ++e) {
#pragma unroll
              for (int hf = 0; hf < 2; ++hf) {
                const __half2_raw r2 = __nv_cvt_fp8x2_to_halfraw2(
                    static_cast<__nv_fp8x2_storage_t>((cwd[e] >> (16 * hf)) & 0xffffu), __NV_E4M3);
                __half2 h2 = *reinterpret_cast<const __half2*>(&r2);
                if (scale_page >= 0) h2 = __hmul2(h2, rs2);
                hw[2 * e + hf] = *reinterpret_cast<const uint32_t*>(&h2);
              }
            }
            uint8_t* rowp = dst + box * kBox + row * 128;
            *reinterpret_cast<uint4*>(rowp + (((2 * qq) ^ (row & 7)) << 4)) = make_uint4(hw[0], hw[1], hw[2], hw[3]);
            *reinterpret_cast<uint4*>(rowp + (((2 * qq + 1) ^ (row & 7)) << 4)) = make_uint4(hw[4], hw[5], hw[6], hw[7]);
          }
          fence_proxy_async_cta();     // read by the tensor core
          __syncwarp();
          if (lane == 0) {
            mbar_arrive_cluster_cta(mapa(bar(kBFull + slot), 0));
            mbar_arrive_local(bar(kBStgEmpty + ss));
          }
          return true;
        };
        auto conv_s = [&]() -> bool {
          for (int c = 0; c < kChunks; ++c)
            if (!convert(-1)) return false;
          return true;
        };
        auto conv_o = [&](int j) -> bool {
          for (int pg_i = 0; pg_i < 4; ++pg_i) {
            const int row0 = lo + kTile * j + 64 * pg_i;
            if (row0 >= hi) break;
            bool vld;
            const int pg = page_of(p, b, row0, &vld);
            for (int bb = 0; bb < 2; ++bb)
              if (!convert(pg)) return false;
          }
          return true;
        };
        ok = conv_s();
        for (int i = 0; i < n_tiles && ok; ++i) {
          if (i + 1 < n_tiles) ok = conv_s();
          if (ok) ok = conv_o(i);
        }
        ++uc;
        }
      }
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
// Unit counters, one (claim, done) pair per launch in flight, keyed by the
// launch's o_part workspace (see the decode_tc.cu counterpart for the rule).
constexpr int kCounterSlots = 64;
__device__ unsigned g_pair_claim[kCounterSlots];
__device__ unsigned g_pair_done[kCounterSlots];

bool claim_slot(const void* workspace, unsigned** claim, unsigned** done) {
  static std::mutex mu;
  static const void* owner[kCounterSlots] = {};
  static unsigned next = 0;
  void* c = nullptr;
  void* d = nullptr;
  if (cudaGetSymbolAddress(&c, g_pair_claim) != cudaSuccess || cudaGetSymbolAddress(&d, g_pair_done) != cudaSuccess)
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

}  // namespace

bool decode_pair_supported(const DecodeArgs& a) {
  const bool forms = (a.q_dtype == MLA_BF16 && (a.cache_dtype == MLA_BF16 || a.cache_dtype == MLA_E4M3)) ||
                     (a.q_dtype == MLA_E4M3 && a.cache_dtype == MLA_E4M3 && a.q_scale);
  return forms && a.page_size == 64 && a.n_heads > 64 && a.n_heads <= 128 &&
         (long long)a.batch * a.q_len * a.num_splits * 2 < (1ll << 31);
}

cudaError_t launch_decode_pair(const DecodeArgs& a, cudaStream_t st) {
  TensorMapEncodeFn enc = tensor_map_encoder();
  if (!enc) return cudaErrorNotSupported;
  const bool d8 = a.q_dtype == MLA_E4M3;                  // two-term e4m3 query: 8-bit MMAs
  const bool f8 = a.cache_dtype == MLA_E4M3 && !d8;       // bf16 query over e4m3: widened operands
  CUtensorMap tc, tc2, tq;
  if (d8) {
    // the e4m3 pool as 2-D [num_pages * 9 * 64 lines x 64 codes] of 64-byte
    // lines, 64-byte swizzled (the operand layout): boxes of one block and of
    // two adjacent blocks
    for (int k = 0; k < 2; ++k) {
      cuuint64_t dims[2] = {64, (cuuint64_t)a.num_pages * kChunks * 64};
      cuuint64_t strides[1] = {64};
      cuuint32_t box[2] = {64, k == 0 ? 64u : 128u};
      cuuint32_t es[2] = {1, 1};
      if (enc(k == 0 ? &tc : &tc2, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(a.cache), dims, strides, box,
              es, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_64B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
        return cudaErrorInvalidValue;
    }
  } else if (f8) {
    // the e4m3 pool as 2-D [num_pages * 9 * 64 lines x 64 codes] of 64-byte
    // lines, unswizzled (the converters swizzle): boxes of one block
    cuuint64_t dims[2] = {64, (cuuint64_t)a.num_pages * kChunks * 64};
    cuuint64_t strides[1] = {64};
    cuuint32_t box[2] = {64, 64};
    cuuint32_t es[2] = {1, 1};
    if (enc(&tc, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(a.cache), dims, strides, box, es,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return cudaErrorInvalidValue;
    tc2 = tc;
  } else {
    // the page-blocked pool as 2-D [num_pages * 9 * 64 lines x 64 columns] of
    // 128-byte lines: boxes of 64 lines (one block) and 128 lines (two adjacent blocks)
    for (int k = 0; k < 2; ++k) {
      cuuint64_t dims[2] = {64, (cuuint64_t)a.num_pages * kChunks * 64};
      cuuint64_t strides[1] = {128};
      cuuint32_t box[2] = {64, k == 0 ? 64u : 128u};
      cuuint32_t es[2] = {1, 1};
      if (enc(k == 0 ? &tc : &tc2, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(a.cache), dims, strides,
              box, es, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
        return cudaErrorInvalidValue;
    }
  }
  if (d8) {
    // the two-term query [rows, 2, heads, 576] codes as 3-D [2 rows planes x
    // heads x 576]: boxes of 64 codes x 64 heads of one plane, 64-byte swizzled
    // (heads past n_heads read as zeros)
    cuuint64_t dims[3] = {MLA_D_ROW, (cuuint64_t)a.n_heads, (cuuint64_t)a.batch * a.q_len * 2};
    cuuint64_t strides[2] = {MLA_D_ROW, (cuuint64_t)a.n_heads * MLA_D_ROW};
    cuuint32_t box[3] = {64, (cuuint32_t)kHPC, 1};
    cuuint32_t es[3] = {1, 1, 1};
    if (enc(&tq, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, const_cast<void*>(a.q_abs), dims, strides, box, es,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_64B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return cudaErrorInvalidValue;
  } else {
    // q_abs [rows, heads, 576]: boxes of 64 columns x 64 heads of one row
    // (heads past n_heads read as zeros)
    cuuint64_t dims[3] = {MLA_D_ROW, (cuuint64_t)a.n_heads, (cuuint64_t)a.batch * a.q_len};
    cuuint64_t strides[2] = {MLA_D_ROW * 2, (cuuint64_t)a.n_heads * MLA_D_ROW * 2};
    cuuint32_t box[3] = {64, (cuuint32_t)kHPC, 1};
    cuuint32_t es[3] = {1, 1, 1};
    if (enc(&tq, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(a.q_abs), dims, strides, box, es,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return cudaErrorInvalidValue;
  }
  const int smem = d8 ? PairLayout<false, true>::kSmem : f8 ? PairLayout<true>::kSmem : PairLayout<false>::kSmem;
  cudaError_t e =
      d8   ? cudaFuncSetAttribute(decode_pair_kernel<false, true>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem)
      : f8 ? cudaFuncSetAttribute(decode_pair_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem)
           : cudaFuncSetAttribute(decode_pair_kernel<false>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  // Runs of splits per claimed unit.  With at least four splits per CTA pair,
  // every pair gets one run of ceil(splits / pairs) consecutive splits: each
  // pair then writes one or two partials instead of one per split (the fp32
  // partials were 11 % of the bytes of the long workload's launch, and each
  // epilogue sits on the pair's critical path).  With fewer splits, as in
  // batches of short ragged sequences, single splits keep the dynamic
  // claiming balanced.
  const long long P = sm_pair_count();
  const long long n_flat = (long long)a.batch * a.q_len * a.num_splits;
  const int run = n_flat >= 4 * P ? (int)((n_flat + P - 1) / P) : 1;
  const long long units = (n_flat + run - 1) / run;
  PairParams p{a.n_heads, a.q_len, a.batch, a.block_table, a.max_pages, a.num_pages, a.seq_lens, a.num_splits,
               a.split_tokens, run, a.softmax_scale * 1.4426950408889634f, nullptr, nullptr, a.o_part, a.lse_part,
               a.err, g_wait_limit.load(), g_withhold_q.load(), a.cache_scale, a.q_scale};
  if (!claim_slot(a.o_part, &p.claim, &p.done)) return cudaErrorInvalidSymbol;
  const long long pairs = units < P ? units : P;
  if (d8)
    return launch_dependent(decode_pair_kernel<false, true>, dim3((unsigned)(2 * pairs)),
                            dim3(PairLayout<false, true>::kThreads), smem, st, tc, tc2, tq, p);
  if (f8)
    return launch_dependent(decode_pair_kernel<true>, dim3((unsigned)(2 * pairs)), dim3(PairLayout<true>::kThreads),
                            smem, st, tc, tc2, tq, p);
  return launch_dependent(decode_pair_kernel<false>, dim3((unsigned)(2 * pairs)), dim3(PairLayout<false>::kThreads),
                          smem, st, tc, tc2, tq, p);
}

}  // namespace mla
