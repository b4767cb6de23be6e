/*
 * csa2.h -- C ABI of libcsa2: the CSA2 hierarchical sparse-attention decode
 * path (DeepSeek V4.1-Flash) on one NVIDIA B200 (sm_100a).
 *
 * The path has five steps, and each step below cites the web page that
 * describes it:
 *   1. a full-mode indexer scores every context position for the query;
 *   2. it keeps a candidate pool of up to 16,384 positions;
 *   3. reindex layers re-score only that pool and keep the top 512;
 *   4. reuse layers take an earlier layer's selection unchanged;
 *   5. attention runs over the selected positions plus the most recent 128
 *      tokens, reading a main KV cache stored in FP4 that is dequantised in
 *      the kernel.
 *
 * Sources: "DeepSeek V4.1-Flash: 552B runs like 16B" (the-agent-daily.org),
 * Act 2 and Act 3; "How DeepSeek V4.1 Flash Actually Works: A Deep Dive"
 * (youtubesummary.com), "The three KV-cache optimizations", item 2;
 * "DeepSeek Has Done It Again..." (youtubesummary.com), "Architecture and
 * inference efficiency", bullet "Sparse attention for long context";
 * "DeepSeek V4.1 Flash: the most insane optimization so far" (artofsm.art);
 * "Deepseek just did the impossible" (summarytube.com), "Memory and Compute
 * Optimization".
 *
 * The pages fix no number formats or head sizes.  This library fixes them:
 *   - The indexer is int8 with int8 head weights, so scores are exact
 *     integers:  score[s] = sum_h w[h] * max(0, sum_d q[h][d] * key[s][d]).
 *   - The KV cache is FP4 E2M1 in blocks of 32 values, each block with one
 *     FP8 E4M3 scale (OCP MX / OFP8 definitions).  K = V = the dequantised
 *     row (one latent row per position, shared by all query heads).
 *   - Queries and outputs are bf16.  Attention accumulates in fp32.
 *
 * Conventions for every entry point
 *   - Every pointer is a DEVICE pointer unless it is marked "host".  The caller
 *     allocates and owns every buffer.  The library never allocates or frees
 *     memory and never synchronises.  Apart from the fixed scratch array of
 *     csa2_topk_pool_noalloc (see there), its only global state is one-time,
 *     per-device set-up (kernel attributes, occupancy figures), held in
 *     atomics, so first calls from several host threads do not race.  Calls
 *     that use distinct workspaces and streams are independent.
 *   - All work is enqueued on `stream` (a cudaStream_t; NULL means the legacy
 *     default stream).  Nothing is complete when the call returns.
 *     Every call only enqueues kernels, so it can be captured into a CUDA
 *     graph.  Make one ordinary call first, which does one-time kernel set-up.
 *   - The return value reports argument errors and launch errors at once.
 *     Errors found on the device (bad index, score overflow, wait timeout) are
 *     written to `*status`, a caller-owned device int32 that the caller zeroes.
 *     The first error wins.  Read it after your own synchronisation.
 *     No kernel traps or asserts.  When a kernel hits an error, it records
 *     the error and skips the faulty access.
 *   - `ws`/`ws_bytes` is a caller-provided device scratch buffer, at least as
 *     large as the matching *_workspace() function says, and 256-byte
 *     aligned.  Its contents need no initialisation.  It must not be used by
 *     another call that runs concurrently.
 *   - Positions: query i belongs to sequence seq_of_query[i] (NULL means
 *     sequence i) and sits at position query_pos[i].  It sees the cached
 *     rows 0..query_pos[i], and the cache already holds the current token.
 *   - Selections (pools, top-k) list positions in ascending order.  Ties in
 *     score go to the lower position.  The slots after the count are -1.
 */
#ifndef CSA2_H
#define CSA2_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* ------------------------------------------------------------ status codes */
enum {
  CSA2_OK = 0,
  CSA2_ERR_INVALID_ARG = 1,       /* NULL/misaligned pointer, bad size or mode   */
  CSA2_ERR_UNSUPPORTED = 2,       /* shape outside the supported set (see below) */
  CSA2_ERR_WORKSPACE = 3,         /* ws_bytes smaller than the *_workspace() size */
  CSA2_ERR_CUDA = 4,              /* a CUDA launch or runtime call failed          */
  CSA2_ERR_SCORE_RANGE = 5,       /* device: 128*sum|w|*sum|q| >= 2^31, so an int32 score could wrap */
  CSA2_ERR_INDEX_RANGE = 6,       /* device: a position, page or row out of range  */
  CSA2_ERR_TIMEOUT = 7,           /* device: a bounded wait gave up (never expected) */
  CSA2_ERR_ORDER = 8              /* device: candidate positions not strictly ascending */
};

/* Layer modes of the CSA2 plan. */
enum { CSA2_FULL = 0, CSA2_REINDEX = 1, CSA2_REUSE = 2 };

/* ------------------------------------------------------------ cached rows
 * A view of per-position rows (index keys, FP4 codes or FP4 scales).
 * Position p of sequence s lives at physical row
 *   paged      : page_table[s*max_pages + p/page_rows]*page_rows + p%page_rows
 *   contiguous : s*seq_rows + p                       (page_table == NULL)
 * and row r starts at (const char*)base + r*row_bytes.  Every row index is
 * checked against n_rows on the device (CSA2_ERR_INDEX_RANGE).
 * Alignment: base 16 B, row_bytes a multiple of 16 B for index keys and FP4
 * codes, and a multiple of 4 B for FP4 scales.  page_rows must be a multiple
 * of 64.
 */
typedef struct csa2_rows {
  const void* base;
  int64_t row_bytes;
  int64_t n_rows;
  const int32_t* page_table;   /* device int32 [n_seq][max_pages] or NULL */
  int32_t page_rows;
  int32_t max_pages;
  int64_t seq_rows;
} csa2_rows;

/* ------------------------------------------------------------ step 1 (+2)
 * csa2_index_full: the full-mode indexer ("the first full-mode indexing layer
 * searches the large context and builds a candidate pool": "DeepSeek
 * V4.1-Flash: 552B runs like 16B", Act 2; "scans full context once and
 * generates up to 16,384 candidate positions": "How DeepSeek V4.1 Flash
 * Actually Works", three KV-cache optimizations, item 2).
 *
 *   q            int8  [nq][H][D]   indexer query heads
 *   w            int8  [nq][H]      integer head weights
 *   keys         index-key rows, D int8 per row (csa2_rows above)
 *   seq_of_query int32 [nq] or NULL;  query_pos int32 [nq]
 *   max_ctx      host: every query_pos[i] < max_ctx (checked on device)
 *   scores       int32 [nq][ld_scores] or NULL: score of every position
 *                0..query_pos[i] (ld_scores >= max_ctx); the rest is untouched
 *   P, pool_idx, pool_cnt   P > 0: int32 [nq][P] pool (the P best positions),
 *                           int32 [nq] count = min(P, pos+1)
 *   K, sel_idx, sel_cnt     K > 0: int32 [nq][K] the K best positions (the
 *                           top-K of the pool under the same scores, i.e. the
 *                           global top-K) and their count
 * Every query scores its own causal prefix 0..query_pos[i], so a prefill
 * chunk (many queries of one sequence at consecutive positions) is one call;
 * with P = 0 and K > 0 each query keeps its top-K of the whole prefix.  From
 * 16 queries on, consecutive queries of one sequence share key tiles in
 * groups of four.
 * Supported: D in {64, 128}; 1 <= H <= 128; 1 <= nq <= 4096; P, K in
 * [0, 65536].
 * Errors on the device: SCORE_RANGE, INDEX_RANGE.
 */
int32_t csa2_index_full(const int8_t* q, const int8_t* w, const csa2_rows* keys,
                        const int32_t* seq_of_query, const int32_t* query_pos,
                        int32_t nq, int32_t H, int32_t D, int32_t max_ctx,
                        int32_t* scores, int64_t ld_scores,
                        int32_t P, int32_t* pool_idx, int32_t* pool_cnt,
                        int32_t K, int32_t* sel_idx, int32_t* sel_cnt,
                        void* ws, size_t ws_bytes, int32_t* status, void* stream);
size_t csa2_index_full_workspace(int32_t nq, int32_t max_ctx, int32_t P, int32_t K);

/* ------------------------------------------------------------ step 2
 * csa2_topk_pool: exact top-k over int32 scores, ties to the lower position,
 * result in ascending position order (the pool of step 2 and the 512-of-pool
 * selection; same sources as step 1).
 *
 *   scores    int32 [nq][ld]        candidate scores
 *   n_valid   int32 [nq] or NULL    candidates of query i (<= n_max); NULL: n_max
 *   cand_pos  int32 [nq][ld] or NULL  position of each candidate, strictly
 *             ascending within the valid prefix (CSA2_ERR_ORDER otherwise);
 *             NULL: candidate j is position j
 *   k         wanted count; out_idx int32 [nq][k], out_cnt int32 [nq]
 * Supported: 1 <= nq <= 65535, 0 <= n_max <= 2^30, 1 <= k <= 65536.
 */
int32_t csa2_topk_pool(const int32_t* scores, int64_t ld, const int32_t* n_valid,
                       const int32_t* cand_pos, int32_t nq, int32_t n_max, int32_t k,
                       int32_t* out_idx, int32_t* out_cnt,
                       void* ws, size_t ws_bytes, int32_t* status, void* stream);
size_t csa2_topk_pool_workspace(int32_t nq, int32_t n_max, int32_t k);

/* csa2_topk_pool_noalloc: csa2_topk_pool without a caller workspace.  The
 * pages have no counterpart to this call; it exists for callers that cannot
 * allocate device memory.  Plugin code inside a host framework may receive only
 * its input and output buffers, and a serving loop may have reserved all
 * device memory up front (cudaMalloc can block on the device and fragment
 * that reservation).
 * Arguments, results and errors are those of csa2_topk_pool, minus ws/ws_bytes.
 * Scratch: one fixed device array inside the library, CSA2_NOALLOC_SCRATCH_BYTES
 * long.  Every GPU that loads the library holds it until the process exits.
 * n_max <= 16384 needs no scratch.  Larger sizes must satisfy
 * csa2_topk_pool_workspace(nq, n_max, k) <= CSA2_NOALLOC_SCRATCH_BYTES;
 * otherwise the call returns CSA2_ERR_WORKSPACE and launches nothing.  That
 * allows 8 queries of up to 10^6 candidates each, or 7 of up to 2^24.
 * The call allocates and frees nothing.  Its first call on a device looks up
 * the array's address there (cudaGetSymbolAddress), so make that first call
 * before any stream capture on that device.  The address is kept per device
 * together with the context it was found in; after a device reset (a new
 * context, the module loaded again) the next call looks it up again, and that
 * call too must come before any stream capture.
 * Every call uses the same array and clears the parts that must start at
 * zero.  Calls that overlap on the GPU (other streams, other threads) race on
 * it, so serialise them.
 */
#define CSA2_NOALLOC_SCRATCH_BYTES (4u << 20)
int32_t csa2_topk_pool_noalloc(const int32_t* scores, int64_t ld, const int32_t* n_valid,
                               const int32_t* cand_pos, int32_t nq, int32_t n_max, int32_t k,
                               int32_t* out_idx, int32_t* out_cnt, int32_t* status, void* stream);

/* ------------------------------------------------------------ step 3
 * csa2_reindex: score only the pool positions with this layer's query,
 * weights and index keys, and keep the best K ("later layers search only that
 * much smaller pool": "DeepSeek V4.1-Flash: 552B runs like 16B", Act 2;
 * "search within that shortlist": "How DeepSeek V4.1 Flash Actually Works",
 * item 2).
 *
 *   q, w, keys, seq_of_query   as csa2_index_full
 *   pool_idx  int32 [nq][P] ascending positions, pool_cnt int32 [nq]
 *   sel_idx   int32 [nq][K] out, sel_cnt int32 [nq] out
 *   scores    int32 [nq][P] or NULL: score of each pool entry (slot order)
 * Supported: D in {64, 128}; 1 <= H <= 128; 1 <= nq <= 65535; 1 <= P <= 65536; 1 <= K <= P.
 */
int32_t csa2_reindex(const int8_t* q, const int8_t* w, const csa2_rows* keys,
                     const int32_t* seq_of_query, const int32_t* pool_idx,
                     const int32_t* pool_cnt, int32_t nq, int32_t H, int32_t D,
                     int32_t P, int32_t K, int32_t* sel_idx, int32_t* sel_cnt,
                     int32_t* scores, void* ws, size_t ws_bytes, int32_t* status,
                     void* stream);
size_t csa2_reindex_workspace(int32_t nq, int32_t P, int32_t K);

/* ------------------------------------------------------------ step 5
 * csa2_sparse_attn_fp4: softmax attention over S = selection U window, each
 * position counted once.  The window is [max(0, pos-window+1), pos].  Keys
 * and values are the same dequantised FP4 latent row ("512 most relevant KV
 * entries, plus a local 128-token window": "How DeepSeek V4.1 Flash Actually
 * Works", item 2; "DeepSeek Has Done It Again...", sparse attention bullet;
 * FP4 main KV: "DeepSeek V4.1-Flash: 552B runs like 16B", Act 3).
 *
 *   q        bf16 [nq][Hq][D] (bit patterns as uint16)
 *   codes    FP4 code rows: D/2 bytes, element 2i in the low nibble of byte i
 *   scales   E4M3 scale rows: D/32 bytes, byte j scales elements 32j..32j+31
 *   sel_idx  int32 [nq][K] ascending positions (-1 after sel_cnt[i]);
 *            sel_cnt int32 [nq]
 *   softmax_scale  host; <= 0 means 1/sqrt(D)
 *   out      bf16 [nq][Hq][D];  lse float [nq][Hq] or NULL (natural log of
 *            the softmax denominator, including the scale)
 * Supported: D in {128, 512}; Hq in {8, 16, ..., 128} (a multiple of 8);
 * 0 <= K <= 65536; 0 <= window <= 1024 (0: S is the selection alone, as for a
 * context shard that holds none of the query's window rows).
 */
int32_t csa2_sparse_attn_fp4(const uint16_t* q, const csa2_rows* codes, const csa2_rows* scales,
                             const int32_t* seq_of_query, const int32_t* query_pos,
                             const int32_t* sel_idx, const int32_t* sel_cnt,
                             int32_t nq, int32_t Hq, int32_t D, int32_t K, int32_t window,
                             float softmax_scale, uint16_t* out, float* lse,
                             void* ws, size_t ws_bytes, int32_t* status, void* stream);
size_t csa2_sparse_attn_workspace(int32_t nq, int32_t Hq, int32_t D, int32_t K, int32_t window);

/* csa2_attn_combine: attention over the union of R disjoint row sets, from
 * the R partial results over each set.  Softmax over the union is each part's
 * softmax rescaled by its share of the total mass, so with lse_r the natural
 * log of part r's softmax denominator (the `lse` output of
 * csa2_sparse_attn_fp4):
 *     LSE = log sum_r exp(lse_r),   out = sum_r exp(lse_r - LSE) o_r.
 * This is the last step of a context-sharded decode: each part (a GPU that
 * owns a slice of the cache) attends to the rows of S it holds; the pages
 * scale context by selection ("DeepSeek V4.1-Flash: 552B runs like 16B",
 * Act 2), and the selected rows then live on whichever slice holds them.
 *   o_parts    bf16 [R][nq][Hq][D] (16-byte aligned)
 *   lse_parts  float [R][nq][Hq]; -inf: that part holds no row of the query
 *   out        bf16 [nq][Hq][D] (16-byte aligned); lse_out float [nq][Hq]
 *              or NULL (-inf when no part holds a row)
 * Accumulation is fp32.  Supported: 1 <= R <= 4096, 8 <= D <= 1024 with D a
 * multiple of 8.  Nothing is allocated; no workspace.
 */
int32_t csa2_attn_combine(const uint16_t* o_parts, const float* lse_parts, int32_t R, int32_t nq, int32_t Hq,
                          int32_t D, uint16_t* out, float* lse_out, int32_t* status, void* stream);

/* csa2_sparse_attn_fp4_local: csa2_sparse_attn_fp4 for a layer that keeps its
 * own cache of the most recent tokens beside the FP4 main cache (V4 kept a
 * separate per-layer local KV of the latest 128 tokens besides the global KV,
 * and V4.1 keeps that local cache while a session is active: "How DeepSeek
 * V4.1 Flash Actually Works", the three KV-cache optimizations, item 3).  The
 * window positions are read from it, every other position of S from the FP4
 * cache.  The pages give the local cache no format; here it holds bf16 rows.
 *   local_kv  bf16 rows of D values (row_bytes >= 2 D, a multiple of 16),
 *             contiguous (page_table NULL); seq_rows = R >= window is the
 *             ring length: position p of sequence s is row s*R + (p mod R).
 *             The caller keeps it current: for every query it holds the
 *             rows of that query's window positions.
 * Other arguments, the workspace (csa2_sparse_attn_workspace) and errors as
 * csa2_sparse_attn_fp4; a local_kv of the wrong shape is CSA2_ERR_INVALID_ARG.
 */
int32_t csa2_sparse_attn_fp4_local(const uint16_t* q, const csa2_rows* codes, const csa2_rows* scales,
                                   const csa2_rows* local_kv, const int32_t* seq_of_query,
                                   const int32_t* query_pos, const int32_t* sel_idx, const int32_t* sel_cnt,
                                   int32_t nq, int32_t Hq, int32_t D, int32_t K, int32_t window,
                                   float softmax_scale, uint16_t* out, float* lse,
                                   void* ws, size_t ws_bytes, int32_t* status, void* stream);

/* ------------------------------------------------------------ steps 1-5 as a plan
 * csa2_layer_plan: one decode step through L layers of modes FULL, REINDEX or
 * REUSE ("Full -> Reindex -> Reuse pipeline": "DeepSeek V4.1-Flash: 552B runs
 * like 16B", Act 2; "full, reindex, and reuse modes": "DeepSeek V4.1 Flash:
 * the most insane optimization so far"; layers share indices: "Deepseek just
 * did the impossible", Memory and Compute Optimization).
 * modes[0] must be FULL.  A REINDEX layer re-scores the pool of the most
 * recent FULL layer.  A REUSE layer attends with the selection of the most
 * recent FULL or REINDEX layer (no index work at all).
 * Supported: 1 <= L <= 16 layers, nq * L <= 65535 (one attention launch
 * covers every layer), the per-op limits of the calls above.
 */
typedef struct csa2_layer {
  const int8_t* q;          /* FULL/REINDEX: int8 [nq][H][D_idx] */
  const int8_t* w;          /* FULL/REINDEX: int8 [nq][H]        */
  csa2_rows keys;           /* FULL/REINDEX: index-key rows      */
  const uint16_t* q_attn;   /* bf16 [nq][Hq][D]                  */
  csa2_rows codes;          /* FP4 code rows of this layer       */
  csa2_rows scales;         /* FP4 scale rows of this layer      */
  uint16_t* out;            /* bf16 [nq][Hq][D]                  */
  float* lse;               /* float [nq][Hq] or NULL            */
  int32_t* pool_idx;        /* FULL: [nq][P] out or NULL (kept in ws then) */
  int32_t* pool_cnt;        /* FULL: [nq] out or NULL            */
  int32_t* sel_idx;         /* FULL/REINDEX: [nq][K] out or NULL */
  int32_t* sel_cnt;         /* FULL/REINDEX: [nq] out or NULL    */
  csa2_rows local_kv;       /* the layer's local window cache (see
                               csa2_sparse_attn_fp4_local); base NULL: the
                               window reads the FP4 cache           */
} csa2_layer;

typedef struct csa2_plan_shape {
  int32_t nq, H, D_idx, Hq, D, P, K, window, max_ctx;
  float softmax_scale;             /* <= 0: 1/sqrt(D) */
  const int32_t* seq_of_query;     /* device [nq] or NULL */
  const int32_t* query_pos;        /* device [nq] */
  int32_t group_queries;           /* nonzero: consecutive queries of one sequence
                                      (a speculative-verify block) share each key tile
                                      of the index scans in groups of four, from 2
                                      queries on; zero: every query scans alone (a
                                      batch of distinct sequences: one query per
                                      segment, with the fused histogram) */
} csa2_plan_shape;

int32_t csa2_layer_plan(const int32_t* modes /* host [L] */, int32_t L,
                        const csa2_layer* layers /* host [L] */,
                        const csa2_plan_shape* shape /* host */,
                        void* ws, size_t ws_bytes, int32_t* status, void* stream);
size_t csa2_layer_plan_workspace(const int32_t* modes, int32_t L, const csa2_plan_shape* shape);

/* ------------------------------------------------------------ FP4 cache write
 * csa2_fp4_quantize: store float rows as FP4 E2M1 with E4M3 block scales (the
 * write side of the FP4 main KV cache: "DeepSeek V4.1-Flash: 552B runs like
 * 16B", Act 3; "compressed from FP8 (8 bits) to FP4 (4 bits)": "How DeepSeek
 * V4.1 Flash Actually Works", item 2).  For each block of 32 values:
 *   scale = E4M3 nearest to max|x|/6 (ties to even, saturating at 448);
 *   code  = E2M1 nearest to x/scale (ties to even, saturating at +-6);
 *   scale 0 gives all-zero codes, and a value rounding to 0 is stored as +0.
 *   x        float [n_rows][ld_x] (first D used)
 *   dst_rows int32 [n_rows] or NULL: row r is written to physical row
 *            dst_rows[r] of codes/scales (NULL: row r)
 *   codes    uint8, rows of ld_codes bytes; scales uint8, rows of ld_scales bytes
 * Supported: D a multiple of 32 in [32, 4096].
 */
int32_t csa2_fp4_quantize(const float* x, int64_t n_rows, int32_t D, int64_t ld_x,
                          const int32_t* dst_rows, uint8_t* codes, int64_t ld_codes,
                          uint8_t* scales, int64_t ld_scales, int64_t n_dst_rows,
                          int32_t* status, void* stream);
/* csa2_fp4_quantize_bf16: the same for bf16 rows (x: bf16 bit patterns as
 * uint16, ld_x a multiple of 8), the format a layer produces its KV in.  A
 * bf16 value is exactly a float, so both calls store the same codes for the
 * same values. */
int32_t csa2_fp4_quantize_bf16(const uint16_t* x, int64_t n_rows, int32_t D, int64_t ld_x,
                               const int32_t* dst_rows, uint8_t* codes, int64_t ld_codes,
                               uint8_t* scales, int64_t ld_scales, int64_t n_dst_rows,
                               int32_t* status, void* stream);

/* ------------------------------------------------------------ helpers */
const char* csa2_status_string(int32_t status);  /* static string, never NULL */
int32_t csa2_version(void);                       /* major*10000 + minor*100 + patch */

/* ------------------------------------------------------------ bounded waits
 * csa2_selftest_wait: a diagnostic of the give-up path of the library's
 * waits.  Every wait between the CTAs of a kernel (the grid barrier of the
 * select, reindex and attention kernels) and of the TMA and tensor-core
 * pipelines (the mbarrier wait) stops after a time limit (2 s in the
 * kernels), records CSA2_ERR_TIMEOUT and lets its kernel return, so that a
 * wait which cannot end never hangs the device.  This call runs one such wait
 * on something that never happens, with a short limit:
 *   kind 0  the grid barrier, on *counter (device uint32, zeroed by the
 *           caller; the call adds 1 to it and waits for 2);
 *   kind 1  the mbarrier wait (counter unused, may be NULL).
 *   limit_ns  host: how long the wait tries, at most 10^10 (10 s).
 * After about limit_ns the kernel records CSA2_ERR_TIMEOUT in *status and
 * returns; the device stays usable.
 */
int32_t csa2_selftest_wait(int32_t kind, uint64_t limit_ns, uint32_t* counter, int32_t* status,
                           void* stream);

/* ------------------------------------------------------------ phase tracing
 * In the traced build of the library (libcsa2_trace.so, compiled with
 * -DCSA2_TRACE) the kernels carry phase markers: one thread of every CTA
 * records two uint64 values at each marked point of its kernel, the global
 * timer (ns) and the SM clock cycles since it entered the kernel.
 *   csa2_trace_table_bytes  size of the table: uint64
 *                           [8 kernels][1024 CTAs][16 points][2]; kernels are
 *                           0 index score, 1 select, 2 fused reindex,
 *                           3 attention, 4 row select, 5 zeroing; point 0 is
 *                           kernel entry.  CTA = x + X*(y + Y*z) of its grid;
 *                           CTAs past 1024 are not recorded.
 *   csa2_trace_attach       table: device memory of that size (8-byte aligned),
 *                           zeroed by the caller, or NULL to stop recording.
 *                           It applies to the current device.  Points a
 *                           kernel did not reach stay zero, and each launch
 *                           overwrites the entries of the one before.
 * The normal build compiles the markers to nothing; there csa2_trace_attach
 * returns CSA2_ERR_UNSUPPORTED and touches nothing.
 */
size_t csa2_trace_table_bytes(void);
int32_t csa2_trace_attach(void* table);

#ifdef __cplusplus
}
#endif
#endif /* CSA2_H */
