/*
 * mla.h - C ABI of the B200 (sm_100a) absorbed Multi-head Latent Attention
 * decode library (libmla.so).
 *
 * The library computes one decode step of weight-absorbed MLA attention for
 * one layer, as defined by the DeepSeek-V2 Appendix C formulas ("DeepSeek-V2:
 * MLA Explained", section "MLA Full Formulas", parts 2 and 3) with the
 * absorption of "Optimization Note" on the same page: the key up-projection
 * W_UK is folded into the query and the value up-projection W_UV is applied
 * after the softmax sum, so attention runs directly over the cached rows.
 *
 * The cache ("KV Compression - DeepSeek-V3", section "How it works") holds one
 * row of 576 numbers per token: the RMSNorm'd 512-wide joint KV latent c_kv
 * followed by the 64-wide RoPE'd key k_pe shared by all heads.  Rows live in
 * pages of `page_size` = 64 tokens; a per-sequence block table maps a
 * sequence's page slot to a page of one pool.
 *
 * Pool layout (page-blocked): cache[num_pages][9][64][64] - each page is nine
 * contiguous blocks of [64 rows x 64 columns], block c holding columns
 * 64c..64c+63 of the page's 64 rows.  Element (slot = page*64 + row, column d)
 * sits at index ((page*9 + d/64)*64 + row)*64 + d%64.  Every tensor-core load
 * of the decode is then one contiguous 8 or 16 KB read.
 *
 * A decode step for B sequences with T new tokens each, H heads:
 *   mla_cache_append  new kv_a rows -> cache rows (RMSNorm, RoPE, cast/quantise)
 *   mla_absorb_q      q_nope, q_pe  -> q_abs = [W_UK^T q_nope ; q_pe]   (576 per head)
 *   mla_decode_fwd    q_abs, cache  -> split-KV partials (o_part, lse_part)
 *   (over an e4m3 cache with 65..128 heads, on 8-bit MMAs: mla_split_q_e4m3
 *    q_abs -> two-term e4m3 query, then mla_decode_fwd_q8 -> the same partials)
 *   mla_combine       partials      -> o_lat (512 per head), lse
 *   (mla_combine_shards: the same merge over the per-GPU results of sequences
 *    whose cached rows are sharded across GPUs)
 *   mla_out_uv        o_lat         -> out = W_UV o_lat                 (128 per head)
 * and the projections on either side of that core:
 *   mla_kv_proj_append  hidden states h -> kv_a = W_kv,a h -> cache rows (one kernel)
 *   mla_out_proj        out (all heads) -> u = W_O [o_1; ...; o_H]
 *
 * Conventions for every entry point
 *  - Pointers named as device pointers must be device memory (or managed
 *    memory) of the current device; the caller owns all memory.  No entry
 *    point allocates or frees device memory; the only device memory the
 *    library itself holds is the fixed scratch array of mla_decode_static.
 *  - Tensors are dense, row-major, with the shapes given; device pointers must
 *    be 16-byte aligned (the cache 128-byte aligned).
 *  - Calls are asynchronous on `stream`; a return of MLA_OK means the work was
 *    validated and enqueued.  Argument errors return before anything is
 *    enqueued.  MLA_ERR_CUDA reports a launch failure (details from
 *    mla_last_error_message()).  Bad data found on the device (a block-table
 *    entry outside the pool, a row outside the table) is skipped and recorded
 *    in `err_word` (when not NULL) as a bitwise OR of MLA_DEVERR_* flags; the
 *    caller reads it after synchronising.
 *  - No C++ exception crosses the ABI.  Entry points are thread-safe.
 */
#ifndef MLA_H_
#define MLA_H_

#include <stddef.h>
#include <stdint.h>
#include <cuda_runtime_api.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Fixed widths of the DeepSeek-V2/V3 attention shape ("KV Compression -
 * DeepSeek-V3", "How it works"; "DeepSeek-V2: MLA Explained", symbol list). */
#define MLA_D_C    512   /* joint KV latent width (kv_lora_rank) */
#define MLA_D_R     64   /* decoupled rope key width (qk_rope_head_dim) */
#define MLA_D_ROW  576   /* numbers cached per token per layer */
#define MLA_D_NOPE 128   /* per-head nope query width */
#define MLA_D_V    128   /* per-head value width */
#define MLA_PAGE    64   /* the supported page size in tokens */
#define MLA_MAX_HEADS 128

typedef enum {
  MLA_OK = 0,
  MLA_ERR_INVALID_ARG = 1,   /* a null pointer, a bad size or alignment */
  MLA_ERR_UNSUPPORTED = 2,   /* a valid but unsupported dtype / shape combination */
  MLA_ERR_CUDA = 3,          /* a CUDA runtime error while enqueuing */
  MLA_ERR_BAD_INDEX = 4,     /* host-checked index out of range */
  MLA_ERR_TIMEOUT = 5        /* a device wait ran out (reported via err_word) */
} mla_status;

typedef enum {
  MLA_F32 = 0,
  MLA_BF16 = 1,
  MLA_E4M3 = 2               /* OCP FP8 E4M3 (cache only), one fp32 scale per token */
} mla_dtype;

/* Device error flags OR-ed into err_word. */
#define MLA_DEVERR_PAGE     0x1  /* block-table entry < 0 or >= num_pages: row skipped */
#define MLA_DEVERR_POSITION 0x2  /* append position/sequence outside the table: row skipped */
#define MLA_DEVERR_TIMEOUT  0x4  /* a bounded device wait gave up: results invalid */

/* Short static string for a status code; never NULL. */
const char* mla_status_string(int status);

/* Detail of the last non-OK status returned on the calling thread ("" if none). */
const char* mla_last_error_message(void);

/* Library version: major*10000 + minor*100 + patch. */
int mla_version(void);

/*
 * mla_rope_table (host function, no GPU needed)
 * RoPE rotation table for the decoupled key ("DeepSeek-V2: MLA Explained",
 * "MLA Full Formulas" part 2, k^R_t = RoPE(W^KR h_t)).  Pair i (channels 2i,
 * 2i+1) of a row at position p turns by angle p * theta^(-2i/64); the angle,
 * cos and sin are evaluated in double precision and rounded to float.
 *   theta         rotary base (> 1), e.g. 10000
 *   max_pos       number of positions (>= 1)
 *   cos_out, sin_out  HOST arrays [max_pos, 32] float, caller-owned
 * Returns MLA_ERR_INVALID_ARG for null pointers or bad sizes.
 */
mla_status mla_rope_table(double theta, int max_pos, float* cos_out, float* sin_out);

/*
 * mla_decode_workspace_bytes (host function, no GPU needed)
 * Bytes of caller workspace mla_decode_fwd needs for its split partials:
 * o_part (fp32 [batch*q_len, n_heads, num_splits, 512]) plus lse_part (fp32
 * [batch*q_len, n_heads, num_splits]), i.e. batch*q_len*n_heads*num_splits*513*4.
 * Returns 0 for non-positive arguments.
 */
size_t mla_decode_workspace_bytes(int batch, int q_len, int n_heads, int num_splits);

/*
 * mla_cache_append
 * Writes the cache rows of new tokens ("KV Compression - DeepSeek-V3", "How it
 * works" and "Official code": split the 576-wide wkv_a output [512, 64],
 * RMSNorm the latent, RoPE the rope part, store both; "DeepSeek-V2: MLA
 * Explained", "Caching Strategy").  For new token n:
 *   c   = kv_a[n, 0:512],  cache_c = c / sqrt(mean(c^2) + eps) * norm_gain
 *   k   = kv_a[n, 512:576], cache_k[2i] = k[2i] cos - k[2i+1] sin,
 *                           cache_k[2i+1] = k[2i] sin + k[2i+1] cos  (table row positions[n])
 *   row = [cache_c ; cache_k] stored at slot
 *         block_table[seq_ids[n], positions[n] / page_size] * page_size + positions[n] % page_size
 *         of the page-blocked pool (see the layout above)
 *   E4M3 cache: a = max|row|, cache_scale[slot] = a / 448,
 *         codes = e4m3_rne_satfinite(row * (448 / a)); a = 0 stores zeros and scale 0.
 * Arithmetic is fp32.
 *   kv_a        device [n_new, 576], kv_dtype F32 or BF16
 *   seq_ids     device int32 [n_new], each in [0, batch)
 *   positions   device int32 [n_new], each in [0, max_pages_per_seq*page_size) and < rope_max_pos
 *   block_table device int32 [batch, max_pages_per_seq], entries in [0, num_pages)
 *   norm_gain   device float [512] or NULL (gain 1)
 *   eps         RMSNorm epsilon (>= 0)
 *   rope_cos, rope_sin device float [rope_max_pos, 32] (see mla_rope_table)
 *   cache       device [num_pages, 9, 64, 64] of cache_dtype (F32, BF16, E4M3), page-blocked
 *   cache_scale device float [num_pages, page_size] for E4M3, else ignored (may be NULL)
 *   err_word    device int32 or NULL; rows whose sequence, position or page is out of
 *               range are skipped and flagged (MLA_DEVERR_POSITION / MLA_DEVERR_PAGE)
 * Rows with the same (sequence, position) in one call race; distinct slots never do.
 */
mla_status mla_cache_append(const void* kv_a, mla_dtype kv_dtype, int n_new,
                            const int32_t* seq_ids, const int32_t* positions,
                            const int32_t* block_table, int batch, int max_pages_per_seq,
                            int page_size, const float* norm_gain, float eps,
                            const float* rope_cos, const float* rope_sin, int rope_max_pos,
                            void* cache, float* cache_scale, mla_dtype cache_dtype,
                            int num_pages, int32_t* err_word, cudaStream_t stream);

/*
 * mla_absorb_q
 * Absorbed query ("DeepSeek-V2: MLA Explained", "Optimization Note": W_UK
 * merged into the query; "MLA Full Formulas" part 1, q_{t,i} = [q^C; q^R]):
 *   q_abs[r, h, 0:512]   = sum_k W_UK[h, k, :] * q_nope[r, h, k]     (fp32 accumulate)
 *   q_abs[r, h, 512:576] = q_pe[r, h, :]
 *   q_nope device [rows, n_heads, 128], q_pe device [rows, n_heads, 64],
 *   w_uk   device [n_heads, 128, 512], q_abs device [rows, n_heads, 576]; all of `dtype`
 *   (F32 or BF16).  rows >= 1, 1 <= n_heads <= 128.
 *   BF16 runs on the tcgen05 tensor cores (a 128-row GEMM tile per head, fp32
 *   accumulation, rounded once to bf16); F32 runs on the CUDA cores.
 */
mla_status mla_absorb_q(const void* q_nope, const void* q_pe, const void* w_uk, void* q_abs,
                        int rows, int n_heads, mla_dtype dtype, cudaStream_t stream);

/*
 * mla_decode_fwd
 * Split-KV attention over the cache in latent space ("DeepSeek-V2: MLA
 * Explained", "MLA Full Formulas" part 3 with the absorption of
 * "Optimization Note").  For sequence b with seq_lens[b] = L_b cached rows
 * (the step's q_len new rows included), query t (row r = b*q_len + t) sits at
 * position L_b - q_len + t and sees rows j <= L_b - q_len + t.  Split s covers
 * rows [s*split_tokens, (s+1)*split_tokens).  For each (r, h, s):
 *   z_j = softmax_scale * (q_abs[r,h,0:512] . c_j + q_abs[r,h,512:576] . k_j)
 *         (E4M3 cache: c_j, k_j are codes times cache_scale[j])
 *   o_part[r,h,s,:] = sum_j e^{z_j - m} c_j / sum_j e^{z_j - m}   over the split's visible j
 *   lse_part[r,h,s] = m + ln sum_j e^{z_j - m}  (natural log)
 *   A split with no visible row gets lse_part = -inf; its o_part is left
 *   unwritten by the tensor-core paths (zero on the fp32 path), and
 *   mla_combine gives it weight 0 without reading it.
 *   The tensor-core path for more than 64 heads over a bf16 cache may work a
 *   run of consecutive splits of one query row as one unit (it does so when
 *   there are at least four splits per CTA pair of the GPU): it then writes
 *   the run's merged partial (the same formulas over the run's rows) at the
 *   run's first split and lse_part = -inf at its other splits, whose o_part
 *   stays unwritten.  mla_combine returns the same result either way.
 *   q_abs       device [batch*q_len, n_heads, 576], q_dtype F32 or BF16
 *   cache       device [num_pages, 9, 64, 64], page-blocked; cache_scale as for mla_cache_append
 *   block_table device int32 [batch, max_pages_per_seq]
 *   seq_lens    device int32 [batch], q_len <= L_b <= max_pages_per_seq*page_size
 *   num_splits * split_tokens must cover the longest sequence; split_tokens is
 *               a positive multiple of page_size
 *   o_part      device float [batch*q_len, n_heads, num_splits, 512]   (caller-owned workspace)
 *   lse_part    device float [batch*q_len, n_heads, num_splits]
 *   err_word    device int32 or NULL (MLA_DEVERR_PAGE, MLA_DEVERR_TIMEOUT)
 * Supported: page_size 64; q_dtype F32 with cache F32; q_dtype BF16 with cache
 * BF16 or E4M3.  Both BF16 forms run on the tcgen05 tensor cores (fp32
 * accumulation, one CTA pair per (query row, split)): a BF16 cache with bf16
 * operands; an E4M3 cache with f16 operands (the codes widened exactly, the
 * value rows multiplied by their scale once in f16, q_abs and the softmax
 * weights rounded to f16), so q_abs and the dequantised cache values must lie
 * within f16's range (|x| <= 65504; a larger q_abs value would turn into an
 * infinity and the scores of that query into NaN).
 * F32 runs exact fp32 on the CUDA cores.
 * Concurrency: the tensor-core path hands out its work through a small
 * counter that the library keys by o_part.  Calls that share o_part must not
 * overlap on the GPU (they would also race on the partials); calls with
 * different o_part buffers may run concurrently on different streams, as long
 * as at most 64 distinct o_part buffers are in use at the same time.  A CUDA
 * graph that captured this call keeps its o_part, so two replays of one graph
 * must not overlap.
 * Pool contract: the tensor-core path reads whole 64-row pages.  Rows of a
 * sequence's last page beyond its length, and page 0 (read in place of a
 * block-table entry outside the pool), enter the contraction with zero
 * weight, so they must hold finite values (no NaN codes for E4M3): allocate
 * the pool zero-filled.
 */
mla_status mla_decode_fwd(const void* q_abs, mla_dtype q_dtype, const void* cache,
                          const float* cache_scale, mla_dtype cache_dtype, int num_pages,
                          const int32_t* block_table, int max_pages_per_seq, int page_size,
                          const int32_t* seq_lens, int batch, int q_len, int n_heads,
                          int num_splits, int split_tokens, float softmax_scale,
                          float* o_part, float* lse_part, int32_t* err_word,
                          cudaStream_t stream);

/*
 * mla_split_q_e4m3
 * The two-term e4m3 form of bf16 absorbed queries: the query operand of
 * mla_decode_fwd_q8.  Not a step of the method itself: with an e4m3 cache
 * ("DeepSeek'in MLA'si latent attention ile KV cache'i %93 sikistiriyor",
 * cache section; OCP FP8 E4M3) both GEMMs of the decode can run on 8-bit
 * tensor-core MMAs, whose two operands are both 8-bit, and one e4m3 rounding
 * of the query (relative 2^-4) would move the scores too far.  Per (row r,
 * head h), in fp32 round-to-nearest-even:
 *   a = max|q_abs[r,h,:]|, inv = 448 / a (0 when a = 0), y = q_abs * inv
 *   q8[r, 0, h, :] = e4m3(y)              (hi; saturating)
 *   q8[r, 1, h, :] = e4m3(y - hi)         (lo; y - hi is exact)
 *   q_scale[r, h]  = a / 448
 * so that q_abs ~ q_scale * (hi + lo) to about 2^-8 relative.
 *   q_abs   device bf16 [rows, n_heads, 576]  (16-byte aligned; finite values: an infinite
 *           one turns the whole vector's codes into NaN)
 *   q8      device uint8 [rows, 2, n_heads, 576] e4m3 codes (16-byte aligned), caller-owned
 *   q_scale device float [rows, n_heads], caller-owned
 * rows >= 0 (0 is a no-op), 1 <= n_heads <= 128.
 */
mla_status mla_split_q_e4m3(const void* q_abs, int rows, int n_heads, void* q8, float* q_scale,
                            cudaStream_t stream);

/*
 * mla_decode_fwd_q8
 * mla_decode_fwd over an E4M3 cache with both GEMMs on 8-bit tensor-core
 * MMAs (tcgen05 kind::f8f6f4), for 65..128 heads: the same outputs and
 * conventions (o_part, lse_part, merged runs of splits, pool contract,
 * concurrency rule) with the query given in the two-term form of
 * mla_split_q_e4m3.  The scores are q_scale[r,h] * cache_scale[j] * the code
 * GEMM of (hi + lo) with row j's codes.  The value GEMM's weights are carried
 * as two e4m3 terms too: e^{z_j - m} * cache_scale[j] / s_ref * 16, where the
 * running maximum m is raised once a tile's scores exceed it by 4 (log2
 * units) and the reference s_ref is the largest row scale seen so far in the
 * unit of work, raised once a tile's scales exceed it by 1.75x (O rescaled
 * by the same factor), so every weight stays <= 448.  o_part then holds
 *   sum_j e^{z_j - m} (codes_j * cache_scale[j])[0:512] / sum_j e^{z_j - m}
 * to within about 2^-8 relative per weight.
 *   q8, q_scale  from mla_split_q_e4m3 for batch*q_len rows and n_heads
 *   other arguments as for mla_decode_fwd with cache_dtype E4M3
 * Supported: page_size 64, 65 <= n_heads <= 128 (else MLA_ERR_UNSUPPORTED).
 */
mla_status mla_decode_fwd_q8(const void* q8, const float* q_scale, const void* cache, const float* cache_scale,
                             int num_pages, const int32_t* block_table, int max_pages_per_seq, int page_size,
                             const int32_t* seq_lens, int batch, int q_len, int n_heads, int num_splits,
                             int split_tokens, float softmax_scale, float* o_part, float* lse_part,
                             int32_t* err_word, cudaStream_t stream);

/*
 * mla_combine
 * Log-sum-exp merge of split partials (the softmax sum of "MLA Full Formulas"
 * part 3 decomposed over disjoint row ranges):
 *   M = max_s lse_part[r,h,s];  w_s = e^{lse_s - M}  (0 for lse_s = -inf)
 *   o_lat[r,h,:] = sum_s w_s o_part[r,h,s,:] / sum_s w_s,   lse_out[r,h] = M + ln sum_s w_s
 *   o_part device float [rows, n_heads, num_splits, 512], lse_part [rows, n_heads, num_splits]
 *   o_lat  device [rows, n_heads, 512] of o_dtype (F32 or BF16)
 *   lse_out device float [rows, n_heads] or NULL
 */
mla_status mla_combine(const float* o_part, const float* lse_part, int rows, int n_heads,
                       int num_splits, void* o_lat, mla_dtype o_dtype, float* lse_out,
                       cudaStream_t stream);

/*
 * mla_combine_shards
 * The same log-sum-exp merge over the per-GPU results of sequences whose
 * cached rows are sharded across GPUs: shard g attended over its own disjoint
 * row range and merged its splits with mla_combine (o_dtype F32, lse_out
 * given), and the shards' results were gathered in shard order, e.g. by an
 * all-gather along the first dimension:
 *   M = max_g lse_shard[g,r,h];  w_g = e^{lse_g - M}  (0 for lse_g = -inf)
 *   o_lat[r,h,:] = sum_g w_g o_shard[g,r,h,:] / sum_g w_g,   lse_out[r,h] = M + ln sum_g w_g
 *   o_shard   device float [num_shards, rows, n_heads, 512]
 *   lse_shard device float [num_shards, rows, n_heads]
 *   o_lat     device [rows, n_heads, 512] of o_dtype (F32 or BF16)
 *   lse_out   device float [rows, n_heads] or NULL
 * A shard that saw no row of a query (lse = -inf) gets weight 0 and its o is
 * not read; a (row, head) no shard saw gives o_lat = 0 and lse_out = -inf.
 */
mla_status mla_combine_shards(const float* o_shard, const float* lse_shard, int num_shards, int rows,
                              int n_heads, void* o_lat, mla_dtype o_dtype, float* lse_out,
                              cudaStream_t stream);

/*
 * mla_combine_out_uv
 * mla_combine followed by mla_out_uv in one launch, for bf16 and few query
 * rows (each CTA reads one head's whole W_UV, so it suits steps of up to a few
 * rows; the projection itself is "MLA Full Formulas" part 2 applied after the
 * attention sum, as in mla_out_uv):
 *   o_lat[r,h,:] as mla_combine (stored bf16, rounded as mla_combine rounds it; o_lat may be NULL)
 *   out[r,h,:] = W_UV[h] o_lat[r,h,:]   (the bf16 o_lat, fp32 sums, stored bf16)
 *   o_part, lse_part as for mla_combine;  w_uv device bf16 [n_heads, 128, 512]
 *   o_lat device bf16 [rows, n_heads, 512] or NULL;  out device bf16 [rows, n_heads, 128]
 *   lse_out device float [rows, n_heads] or NULL
 */
mla_status mla_combine_out_uv(const float* o_part, const float* lse_part, int rows, int n_heads,
                              int num_splits, const void* w_uv, void* o_lat, void* out, float* lse_out,
                              cudaStream_t stream);

/*
 * mla_out_uv
 * Value up-projection applied after the softmax sum ("DeepSeek-V2: MLA
 * Explained", "MLA Full Formulas" part 2, v^C = W^UV c, moved past the sum per
 * "Optimization Note"):
 *   out[r, h, i] = sum_c W_UV[h, i, c] * o_lat[r, h, c]    (fp32 accumulate)
 *   o_lat device [rows, n_heads, 512], w_uv device [n_heads, 128, 512],
 *   out device [rows, n_heads, 128]; all of `dtype` (F32 or BF16).
 *   BF16 runs on the tcgen05 tensor cores (a 128-row GEMM tile per head and
 *   half of the outputs); F32 runs on the CUDA cores.
 */
mla_status mla_out_uv(const void* o_lat, const void* w_uv, void* out, int rows, int n_heads,
                      mla_dtype dtype, cudaStream_t stream);

/*
 * mla_out_proj
 * Output projection after the value up-projection ("DeepSeek-V2: MLA
 * Explained", "MLA Full Formulas" part 3: u_t = W_O [o_{t,1}; ...; o_{t,n_h}],
 * the heads concatenated in head order):
 *   u[r, j] = sum_{h, i} W_O[j, h*128 + i] * out[r, h, i]     (fp32 accumulate)
 *   out  device bf16 [rows, n_heads, 128]   (mla_out_uv's result; at decode
 *        row counts it is still in L2 when this call reads it)
 *   w_o  device bf16 [d_model, n_heads*128]
 *   u    device float [rows, d_model], overwritten
 *   d_model a multiple of 256.  Runs on the tcgen05 tensor cores as a split-K
 *   GEMM whose fp32 partial tiles are added into u (so bits may differ
 *   between runs in the last place); u is cleared first on the same stream.
 */
mla_status mla_out_proj(const void* out, const void* w_o, float* u, int rows, int n_heads, int d_model,
                        cudaStream_t stream);

/*
 * mla_kv_proj_workspace_bytes (host function, no GPU needed)
 * Bytes of caller workspace mla_kv_proj_append needs: the fp32 kv_a rows
 * [n_new, 576] plus one counter per 128 tokens.  0 for n_new <= 0.
 */
size_t mla_kv_proj_workspace_bytes(int n_new);

/*
 * mla_kv_proj_append
 * The joint KV down-projection and the cache append in one kernel ("KV
 * Compression - DeepSeek-V3", "How it works", Eq. (1):
 * [c_t^KV ; k~_t^R] = W_kv,a h_t, 576 wide, then split [512, 64], RMSNorm the
 * latent, RoPE the rope part, store; "Official code": wkv_a, kv_norm):
 *   kv_a[n, :] = sum_k W_kv,a[:, k] * h[n, k]                (fp32 accumulate)
 *   then exactly mla_cache_append's row writer on the fp32 kv_a rows.
 *   h       device bf16 [n_new, d_model];  w_kva device bf16 [576, d_model]
 *   d_model a multiple of 64
 *   workspace device, mla_kv_proj_workspace_bytes(n_new) bytes, 16-byte
 *           aligned, caller-owned; cleared by the call (on the stream); on
 *           completion its first n_new*576 floats hold the fp32 kv_a rows
 *   the other arguments as for mla_cache_append
 * A split-K GEMM on the tcgen05 tensor cores reduces into the workspace; the
 * last CTA to finish a tile of 128 tokens writes those tokens' cache rows.
 */
mla_status mla_kv_proj_append(const void* h, const void* w_kva, int n_new, int d_model, void* workspace,
                              const int32_t* seq_ids, const int32_t* positions, const int32_t* block_table,
                              int batch, int max_pages_per_seq, int page_size, const float* norm_gain, float eps,
                              const float* rope_cos, const float* rope_sin, int rope_max_pos, void* cache,
                              float* cache_scale, mla_dtype cache_dtype, int num_pages, int32_t* err_word,
                              cudaStream_t stream);

/*
 * mla_decode_static
 * Split-KV attention and its combine in one call that allocates nothing and
 * takes no workspace: the same result as mla_decode_fwd followed by
 * mla_combine, with the split partials kept in a scratch array that the
 * library itself holds in device memory.  This call has no counterpart in
 * the pages; it exists for callers that cannot allocate device memory on
 * their own, e.g. a plugin whose host framework owns every device allocation,
 * or a latency-critical serving loop where cudaMalloc's implicit device-wide
 * synchronisation would stall the other streams.
 *
 *   Arguments as for mla_decode_fwd, except that the partials are internal:
 *   o_lat   device [batch*q_len, n_heads, 512] of o_dtype (F32 or BF16)
 *   lse_out device float [batch*q_len, n_heads] or NULL
 *
 * Limits and sharing:
 *  - batch*q_len*n_heads*num_splits must not exceed MLA_STATIC_MAX_PARTIALS
 *    (8192 partial rows, 16.8 MB of fp32 scratch); larger requests return
 *    MLA_ERR_INVALID_ARG with the numbers in mla_last_error_message(), and
 *    nothing is enqueued.  Use mla_decode_fwd + mla_combine for them.
 *  - The scratch is a statically sized array in the library's device code:
 *    every GPU that loads the library holds it until the process exits.
 *  - The first call on each device looks up the array's device address
 *    (cudaGetSymbolAddress, no allocation) with that device current; make
 *    that first call before any stream capture begins.  The lookup is
 *    repeated only if the device's context was replaced (cudaDeviceReset),
 *    since the array then lives at a new address.
 *  - Every call uses the same array and it keeps the last call's contents.
 *    Each call writes every partial it reads before reading it, so nothing
 *    needs clearing.  Calls whose GPU work overlaps (on different streams,
 *    or from different host threads without ordering) race on the array.
 */
#define MLA_STATIC_MAX_PARTIALS 8192
mla_status mla_decode_static(const void* q_abs, mla_dtype q_dtype, const void* cache,
                             const float* cache_scale, mla_dtype cache_dtype, int num_pages,
                             const int32_t* block_table, int max_pages_per_seq, int page_size,
                             const int32_t* seq_lens, int batch, int q_len, int n_heads,
                             int num_splits, int split_tokens, float softmax_scale,
                             void* o_lat, mla_dtype o_dtype, float* lse_out, int32_t* err_word,
                             cudaStream_t stream);

/*
 * The non-absorbed ("level 2") decode, for comparison with the path above
 * ("HuggingFace version does NOT use efficient MLA caching", the ways MLA
 * inference can be run: level 2 caches the latent and decompresses per-head
 * keys and values at every step).  "DeepSeek-V2: MLA Explained", "MLA Full
 * Formulas" parts 2 and 3.  bf16 caches with 64-row pages only.
 *
 * mla_decompress_kv
 * For every row r of every page p of the pool (c = the row's 512 latent numbers):
 *   k_c[p, r, h, :] = W_UK[h] c,   v_c[p, r, h, :] = W_UV[h] c      (fp32 sums, stored bf16)
 *   cache       device bf16 [num_pages, 9, 64, 64] (the page-blocked pool), 128-byte aligned
 *   w_uk, w_uv  device bf16 [n_heads, 128, 512] (as in mla_absorb_q / mla_out_uv)
 *   k_c, v_c    device bf16 [num_pages, 64, n_heads, 128] each (num_pages * 64 * n_heads * 256 bytes)
 *   err_word    device int32 or NULL (MLA_DEVERR_TIMEOUT if a bounded wait ran out)
 * Errors: MLA_ERR_UNSUPPORTED for a cache that is not bf16 or page_size != 64.
 */
mla_status mla_decompress_kv(const void* cache, mla_dtype cache_dtype, int num_pages, int page_size,
                             const void* w_uk, const void* w_uv, int n_heads, void* k_c, void* v_c,
                             int32_t* err_word, cudaStream_t stream);

/*
 * mla_attend_naive
 * Standard attention per head over the decompressed keys and values.  Query
 * row r = b*q_len + t of sequence b sees the rows j <= seq_lens[b] - q_len + t
 * (as in mla_decode_fwd); with k_j the row's rope key (cache columns 512..575):
 *   z_j = softmax_scale * (q_nope[r,h,:] . k_c[j,h,:] + q_pe[r,h,:] . k_j)
 *   out[r,h,:] = sum_j e^{z_j - m} v_c[j,h,:] / sum_j e^{z_j - m},   lse[r,h] = m + ln sum_j e^{z_j - m}
 *   q_nope      device bf16 [batch*q_len, n_heads, 128];  q_pe  device bf16 [batch*q_len, n_heads, 64]
 *   cache, k_c, v_c as produced for mla_decompress_kv; block_table, seq_lens as in mla_decode_fwd
 *   out         device bf16 [batch*q_len, n_heads, 128];  lse  device float [batch*q_len, n_heads] or NULL
 *   err_word    device int32 or NULL (MLA_DEVERR_PAGE for table entries outside the pool; those rows are skipped)
 * out equals the absorbed path's mla_out_uv result up to rounding.
 */
mla_status mla_attend_naive(const void* q_nope, const void* q_pe, const void* cache, mla_dtype cache_dtype,
                            const void* k_c, const void* v_c, int num_pages, const int32_t* block_table,
                            int max_pages_per_seq, int page_size, const int32_t* seq_lens, int batch,
                            int q_len, int n_heads, float softmax_scale, void* out, float* lse,
                            int32_t* err_word, cudaStream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* MLA_H_ */
