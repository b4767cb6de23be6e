// Internal launchers shared by the C ABI layer (api.cu) and the kernels.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <atomic>

#include "csa2.h"

#ifdef CSA2_TRACE
#include <nvtx3/nvToolsExt.h>
#endif

// In the traced build every C entry point opens a named NVTX range, so that a
// profiler can attribute each kernel launch to the C call that made it (a
// plan call nests the calls it makes).  The normal build has none.
#ifdef CSA2_TRACE
namespace csa2 {
struct ApiRange {
  explicit ApiRange(const char* name) { nvtxRangePushA(name); }
  ~ApiRange() { nvtxRangePop(); }
};
}  // namespace csa2
#define CSA2_API_RANGE(name) ::csa2::ApiRange api_range_(name)
#else
#define CSA2_API_RANGE(name) ((void)0)
#endif

namespace csa2 {

// Aligned carving of the caller's workspace.
struct Carver {
  char* base;
  size_t used = 0;
  explicit Carver(void* b) : base(static_cast<char*>(b)) {}
  template <class T>
  T* take(size_t n) {
    used = (used + 255) & ~size_t(255);
    T* p = base ? reinterpret_cast<T*>(base + used) : nullptr;
    used += n * sizeof(T);
    return p;
  }
};

// Options for the launches inside one layer-plan call (per host thread):
//   pdl        launch the index-score, select, reindex and attention kernels
//              as programmatic dependents of the kernel before them;
//   prezeroed  the top-k, reindex and attention scratch was zeroed by the
//              caller (in the kernel launched just before);
//   group      index scans group the queries of a sequence from 2 queries on
//              (a verify block), not only from 16;
//   plan       the call comes from a layer plan: its index scans group queries
//              only when `group` says so (a decode batch of distinct sequences
//              keeps one query per segment and the fused histogram).
struct LaunchOpts {
  bool pdl = false;
  bool prezeroed = false;
  bool group = false;
  bool plan = false;
};
LaunchOpts& launch_opts();
struct LaunchOptsScope {   // sets the options for its lifetime
  LaunchOpts saved;
  explicit LaunchOptsScope(LaunchOpts o) : saved(launch_opts()) { launch_opts() = o; }
  ~LaunchOptsScope() { launch_opts() = saved; }
};
// Zeroes up to kMaxZeroRegions regions (4-byte multiples) in one launch.
constexpr int kMaxZeroRegions = 4;
cudaError_t launch_zero(void* const* ptrs, const size_t* bytes, int n, cudaStream_t st);
// Launches `kernel` with the cooperative and programmatic-dependence
// attributes asked for.  A programmatic launch the device refuses is retried
// once without the attribute, and programmatic launches stay off from then on.
//
// The kernels whose CTAs meet at grid barriers (select, fused reindex,
// attention groups) are launched WITHOUT the cooperative attribute: on B200 a
// cooperative grid starts only after the grid before it has completed, which
// removes the programmatic-launch overlap (2.0-2.6 us per kernel boundary
// against 0.8 us without it).  Their co-residency rests instead on two facts:
// each launcher checks that the grid fits on the device at once (occupancy
// query), and each of these kernels calls pdl_trigger() only after its own
// pdl_wait(), so the grid after it is launched only when every one of its CTAs
// is already resident.  A grid barrier that still waits too long (another
// process filling the device) gives up after its bounded wait and records
// CSA2_ERR_TIMEOUT.
cudaError_t launch_ex(const void* kernel, void** args, dim3 grid, dim3 block, size_t smem, cudaStream_t st,
                      bool cooperative, bool pdl);
template <class... Args>
cudaError_t launch_k(void (*kernel)(Args...), dim3 grid, dim3 block, size_t smem, cudaStream_t st,
                     bool cooperative, bool pdl, Args... args) {
  void* argv[] = {static_cast<void*>(&args)...};
  return launch_ex(reinterpret_cast<const void*>(kernel), argv, grid, block, smem, st, cooperative, pdl);
}

// Radix top-k scratch for nq queries and up to two thresholds per query.
struct TopkScratch {
  uint32_t* hist;        // [nq][kBuckets]                 (zeroed before the histogram pass)
  uint32_t* chunk_cnt;   // [nq][2][n_chunks] x 64 bit     published chunk counts (flag, count)
  uint64_t* cand;        // [nq][2][cand_cap]              keys with bucket >= b*, in position order
  uint32_t* cand_cnt;    // [nq][2]
  uint64_t* kth;         // [nq][2]                        key of the k-th best candidate
  int32_t* thresh;       // [nq][2][2]                     bucket b*, members above b*
  uint32_t* sel_hdr;     // [nq][4]    select: barrier count, tie counts (follows hist; zeroed with it)
  uint64_t* sel_ties;    // [nq][2][kSelTieCap]            select: ties of the threshold bucket
  uint32_t* sel_mcnt;    // [nq][2][kSelMaxG]              select: members per CTA
  uint32_t* sel_radix;   // [nq][2][8][256]                select: digit counts (flat distributions)
  int32_t n_chunks;
  int32_t cand_cap;
};
constexpr int kChunk = 4096;          // positions per chunk in the multi-CTA passes
constexpr int kCandCap = 24576;       // ordered candidates (bucket >= b*) kept per (query, k)

// Select kernel (topk_select.cu): one CTA of kSelNT threads per kSelSpan
// candidates of a row; rows of more than kSelSpan candidates use co-resident
// CTAs that meet at grid barriers.
constexpr int kSelNT = 1024;
constexpr int kSelPer = 16;
constexpr int kSelSpan = kSelNT * kSelPer;
constexpr int kSelTieCap = 4096;
constexpr int kSelMaxG = 256;
// Bytes from TopkScratch::hist that must be zero before the histogram pass
// and the select kernel (the histograms and the select header).
inline size_t topk_zero_bytes(int32_t nq) { return (size_t)nq * (kBuckets + 4) * sizeof(uint32_t); }

size_t topk_scratch_bytes(int32_t nq, int32_t n_max);
TopkScratch carve_topk(Carver& c, int32_t nq, int32_t n_max);

// K1: scores of every visible position for every query (tcgen05 int8), plus
// the bucket histogram.  hist may be NULL.  *hist_built (if given) says
// whether the histogram was built: launches of many queries leave it out.
cudaError_t launch_index_score(const int8_t* q, const int8_t* w, const csa2_rows& keys,
                               const int32_t* seq_of_query, const int32_t* query_pos,
                               int32_t nq, int32_t H, int32_t D, int32_t max_ctx,
                               int32_t* scores, int64_t ld, uint32_t* hist, int32_t* status,
                               cudaStream_t st, bool* hist_built = nullptr);

// Radix top-k over score rows.  ks[0..n_k) are the wanted counts (n_k <= 2,
// ks[0] >= ks[1]); outputs go to out_idx[t]/out_cnt[t].  If hist_ready, the
// histogram in `s.hist` is already filled (by K1); otherwise it is built here.
struct TopkOut {
  int32_t* idx;
  int32_t* cnt;
  int32_t k;
};
cudaError_t launch_topk_large(const int32_t* scores, int64_t ld, const int32_t* n_valid,
                              const int32_t* query_pos, const int32_t* cand_pos, int32_t nq,
                              int32_t n_max, const TopkOut* outs, int32_t n_k,
                              const TopkScratch& s, bool hist_ready, int32_t* status,
                              cudaStream_t st);

// Top-k for up to kSmallMax candidates per query: one select CTA per query.
constexpr int kSmallMax = 16384;
static_assert(kSmallMax <= kSelSpan, "the small path is one select CTA per query");
cudaError_t launch_topk_small(const int32_t* scores, int64_t ld, const int32_t* n_valid,
                              const int32_t* cand_pos, int32_t nq, int32_t n_max, int32_t k,
                              int32_t* out_idx, int32_t* out_cnt, int32_t* status,
                              cudaStream_t st);

// Exact top-k of many long rows (up to kRowSelMax candidates), one CTA per
// row that builds its own histogram (topk_rows.cu).
constexpr int kRowPer = 256;                  // candidates per thread
constexpr int kRowSelMax = 1024 * kRowPer;    // per row
cudaError_t launch_row_select(const int32_t* scores, int64_t ld, const int32_t* n_valid,
                              const int32_t* query_pos, const int32_t* cand_pos, int32_t nq, int32_t n_max,
                              const TopkOut* outs, int32_t n_k, int32_t* status, cudaStream_t st);
// Whether launch_select can take these rows in one pass of co-resident CTAs.
bool select_fits(int32_t nq, int32_t n_max);

// Exact top-k of nq score rows in position order, for one or two k.  hist,
// when given, is the complete bucket histogram of each row and s the scratch
// whose select header is zero; without them n_max must be at most kSelSpan.
// Returns cudaErrorNotSupported when the rows need more CTAs than fit on the
// device at once (the caller then takes the multi-pass path).
cudaError_t launch_select(const int32_t* scores, int64_t ld, const int32_t* n_valid,
                          const int32_t* query_pos, const int32_t* cand_pos, int32_t nq, int32_t n_max,
                          const TopkOut* outs, int32_t n_k, const uint32_t* hist, const TopkScratch* s,
                          int32_t* status, cudaStream_t st);


// K3 scoring part: scores of the pool entries (slot order) for each query.
cudaError_t launch_reindex_score(const int8_t* q, const int8_t* w, const csa2_rows& keys,
                                 const int32_t* seq_of_query, const int32_t* pool_idx,
                                 const int32_t* pool_cnt, int32_t nq, int32_t H, int32_t D,
                                 int32_t P, int32_t* scores, int32_t* status, cudaStream_t st);

// K3 fused: scores and top-K of up to kMaxReindexJobs reindex layers that
// search the same pool, in one launch: co-resident CTAs that meet at grid
// barriers, or, for batches too large to be co-resident with pools of up to
// kRLastMaxP slots, the last CTA of each pool to finish its scores selects.
constexpr int kMaxReindexJobs = 8;
struct ReindexJobDesc {
  const int8_t* q;           // [nq][H][D]
  const int8_t* w;           // [nq][H]
  const csa2_rows* keys;
  int32_t* scores;           // [nq][P] or nullptr
  int32_t* sel_idx;          // [nq][K]
  int32_t* sel_cnt;          // [nq] or nullptr
};
struct ReindexSelScratch {
  int32_t n_probs;           // (layer, query) pairs it holds
  uint32_t* hist;            // [n_probs][kBuckets], then hdr: zeroed by the launcher
  uint32_t* hdr;             // [n_probs][4]
  uint64_t* ties;
  uint32_t* mcnt;
  uint32_t* radix;
  int32_t* sc;               // [n_probs][P] the pool's scores, when the job keeps none
};
constexpr int kRLastMaxP = 16384;
size_t reindex_select_scratch_bytes(int32_t n_probs, int32_t P);
ReindexSelScratch carve_reindex_select(Carver& c, int32_t n_probs, int32_t P);
// Returns cudaErrorNotSupported, having queued nothing, when pools above
// kRLastMaxP slots need more CTAs than can be co-resident, or the head count
// is above 64; the caller then scores and selects in separate launches.
cudaError_t launch_reindex_select(const ReindexJobDesc* jobs, int32_t n_jobs, const int32_t* seq_of_query,
                                  const int32_t* pool_idx, const int32_t* pool_cnt, int32_t nq, int32_t H,
                                  int32_t D, int32_t P, int32_t K, const ReindexSelScratch& r,
                                  int32_t* status, cudaStream_t st);

// K3 on thread-block clusters (reindex_cluster.cu): scores and top-K of up to
// kMaxReindexJobs reindex layers of one pool, one cluster per (layer, query),
// no grid barrier and no scratch.  Returns cudaErrorNotSupported, having
// queued nothing, for pools above 16 x 1024 slots, more than 64 heads, or
// when no cluster of the size needed fits the device.
cudaError_t launch_reindex_cluster(const ReindexJobDesc* jobs, int32_t n_jobs, const int32_t* seq_of_query,
                                   const int32_t* pool_idx, const int32_t* pool_cnt, int32_t nq, int32_t H,
                                   int32_t D, int32_t P, int32_t K, int32_t* status, cudaStream_t st);

// K4: FP4 sparse attention (local_kv: the layer's local window cache, or nullptr).
size_t attn_scratch_bytes(int32_t nq, int32_t Hq, int32_t D, int32_t K, int32_t window);
cudaError_t launch_sparse_attn(const uint16_t* q, const csa2_rows& codes, const csa2_rows& scales,
                               const csa2_rows* local_kv, const int32_t* seq_of_query, const int32_t* query_pos,
                               const int32_t* sel_idx, const int32_t* sel_cnt, int32_t nq,
                               int32_t Hq, int32_t D, int32_t K, int32_t window, float scale,
                               uint16_t* out, float* lse, void* ws, size_t ws_bytes,
                               int32_t* status, cudaStream_t st);

// Combine of R partial attention results (o_r, lse_r) over disjoint row sets
// of the same queries into attention over their union (attn_combine.cu).
cudaError_t launch_attn_combine(const uint16_t* o, const float* lse, int32_t R, int32_t nq, int32_t Hq, int32_t D,
                                uint16_t* out, float* lse_out, cudaStream_t st);

// K7: FP4 quantiser.
cudaError_t launch_fp4_quantize(const void* x, bool bf16, int64_t n_rows, int32_t D, int64_t ld_x,
                                const int32_t* dst_rows, uint8_t* codes, int64_t ld_codes,
                                uint8_t* scales, int64_t ld_scales, int64_t n_dst_rows,
                                int32_t* status, cudaStream_t st);

int sm_count();

// Self-test of the bounded waits (selftest.cu).
cudaError_t launch_wait_selftest(int32_t kind, uint64_t limit_ns, uint32_t* counter, int32_t* status,
                                 cudaStream_t st);

#ifdef CSA2_TRACE
// The traced build: each translation unit with phase markers sets its table.
cudaError_t trace_attach_index(uint64_t* table);
cudaError_t trace_attach_select(uint64_t* table);
cudaError_t trace_attach_reindex(uint64_t* table);
cudaError_t trace_attach_attn(uint64_t* table);
cudaError_t trace_attach_rows(uint64_t* table);
cudaError_t trace_attach_zero(uint64_t* table);
cudaError_t trace_attach_rcluster(uint64_t* table);
#endif

// One-time, per-device set-up (a kernel's shared-memory limit, an occupancy
// figure) is cached in atomics: host threads that make their first calls at
// the same time at worst repeat the set-up, and never race.
using SetupMask = std::atomic<unsigned long long>;   // bit d: done on device d

// Raises a kernel's dynamic shared-memory limit once per device.
template <class F>
cudaError_t ensure_smem(F* kernel, int bytes, SetupMask& done_mask) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 64 && ((done_mask >> dev) & 1ull)) return cudaSuccess;
  e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
  if (e == cudaSuccess && dev < 64) done_mask |= 1ull << dev;
  return e;
}

// Attention jobs that share shapes, positions and sizes (one per layer).
struct AttnJobDesc {
  const uint16_t* q;
  const csa2_rows* codes;
  const csa2_rows* scales;
  const int32_t* sel_idx;
  const int32_t* sel_cnt;
  uint16_t* out;
  float* lse;
  const csa2_rows* local_kv = nullptr;   // the layer's local window cache (bf16 ring), or none
};
constexpr int kMaxAttnJobs = 16;
void attn_bar_region(void* ws, int32_t n_jobs, int32_t nq, int32_t Hq, int32_t D, void** ptr, size_t* bytes);
cudaError_t launch_sparse_attn_jobs(const AttnJobDesc* jobs, int n_jobs, const int32_t* seq_of_query,
                                    const int32_t* query_pos, int32_t nq, int32_t Hq, int32_t D,
                                    int32_t K, int32_t window, float scale, void* ws, int32_t* status,
                                    cudaStream_t st);

}  // namespace csa2
