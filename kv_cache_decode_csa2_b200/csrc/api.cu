// The C ABI of libcsa2 (declared in include/csa2.h): argument checks,
// workspace sizing and carving, and kernel dispatch.  Nothing here allocates,
// frees or synchronises; every call only enqueues work on the caller's stream.
#include <math.h>
#include <string.h>

#include "csa2_device.cuh"
#include "internal.h"

using namespace csa2;

namespace {

bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

bool rows_ok(const csa2_rows* v, int64_t min_row_bytes, int64_t row_align) {
  if (!v || !v->base || v->n_rows < 1 || v->n_rows >= (1ll << 31)) return false;
  if (v->row_bytes < min_row_bytes || v->row_bytes % row_align) return false;
  if (!aligned(v->base, 16)) return false;
  if (v->page_table) {
    if (v->page_rows < 64 || v->page_rows % 64 || v->max_pages < 1) return false;
  } else if (v->seq_rows < 0) {
    return false;
  }
  return true;
}

int32_t cuda_status(cudaError_t e) { return e == cudaSuccess ? CSA2_OK : CSA2_ERR_CUDA; }

size_t index_full_ws(int32_t nq, int32_t max_ctx, int32_t P, int32_t K, void* base, int32_t** scores,
                     TopkScratch* ts) {
  Carver c(base);
  int32_t* sc = c.take<int32_t>((size_t)nq * (size_t)max_ctx);
  TopkScratch t{};
  if (P > 0 || K > 0) t = carve_topk(c, nq, max_ctx);
  if (scores) *scores = sc;
  if (ts) *ts = t;
  return c.used + 256;
}

// Reindex scratch for n_jobs layers over one pool: the fused launch's
// histograms and lists, and (for batches too large to be co-resident) one
// layer's scores and top-k scratch, reused layer after layer.
size_t reindex_ws(int32_t nq, int32_t P, int32_t n_jobs, void* base, int32_t** scores, TopkScratch* ts,
                  ReindexSelScratch* rs) {
  Carver c(base);
  ReindexSelScratch r = carve_reindex_select(c, nq * n_jobs, P);
  int32_t* sc = c.take<int32_t>((size_t)nq * (size_t)P);
  TopkScratch t{};
  if (P > kSmallMax) t = carve_topk(c, nq, P);
  if (scores) *scores = sc;
  if (ts) *ts = t;
  if (rs) *rs = r;
  return c.used + 256;
}

// Scores and top-K of reindex layers that search the same pool: one fused
// launch when its CTAs fit on the device at once, else per layer a scoring
// launch and a select launch.
int32_t run_reindex(const ReindexJobDesc* jobs, int32_t n_jobs, const int32_t* seq_of_query,
                    const int32_t* pool_idx, const int32_t* pool_cnt, int32_t nq, int32_t H, int32_t D, int32_t P,
                    int32_t K, void* ws, int32_t* status, cudaStream_t st) {
  int32_t* sc_ws;
  TopkScratch ts;
  ReindexSelScratch rs;
  reindex_ws(nq, P, n_jobs, ws, &sc_ws, &ts, &rs);
  // The co-resident fused launch when every pool's CTAs fit on the device at
  // once; else one cluster per (layer, query) (no grid barrier, any number of
  // pools); else scores and a select per layer.  The cluster form is second:
  // it gathers each pool's rows with 16 SMs instead of 64 and exchanges
  // through distributed shared memory, which measured slower for one query.
  cudaError_t e = launch_reindex_select(jobs, n_jobs, seq_of_query, pool_idx, pool_cnt, nq, H, D, P, K, rs,
                                        status, st);
  if (e != cudaErrorNotSupported) return cuda_status(e);
  (void)cudaGetLastError();
  e = launch_reindex_cluster(jobs, n_jobs, seq_of_query, pool_idx, pool_cnt, nq, H, D, P, K, status, st);
  if (e != cudaErrorNotSupported) return cuda_status(e);
  (void)cudaGetLastError();
  for (int j = 0; j < n_jobs; ++j) {
    const ReindexJobDesc& d = jobs[j];
    int32_t* sc = d.scores ? d.scores : sc_ws;
    e = launch_reindex_score(d.q, d.w, *d.keys, seq_of_query, pool_idx, pool_cnt, nq, H, D, P, sc, status, st);
    if (e != cudaSuccess) return CSA2_ERR_CUDA;
    if (P <= kSmallMax) {
      e = launch_topk_small(sc, P, pool_cnt, pool_idx, nq, P, K, d.sel_idx, d.sel_cnt, status, st);
    } else {
      TopkOut o{d.sel_idx, d.sel_cnt, K};
      e = launch_topk_large(sc, P, pool_cnt, nullptr, pool_idx, nq, P, &o, 1, ts, false, status, st);
    }
    if (e != cudaSuccess) return CSA2_ERR_CUDA;
  }
  return CSA2_OK;
}

}  // namespace

extern "C" {

const char* csa2_status_string(int32_t s) {
  switch (s) {
    case CSA2_OK: return "ok";
    case CSA2_ERR_INVALID_ARG: return "invalid argument";
    case CSA2_ERR_UNSUPPORTED: return "unsupported shape";
    case CSA2_ERR_WORKSPACE: return "workspace too small";
    case CSA2_ERR_CUDA: return "CUDA error";
    case CSA2_ERR_SCORE_RANGE: return "indexer scores may overflow int32";
    case CSA2_ERR_INDEX_RANGE: return "position, page or row out of range";
    case CSA2_ERR_TIMEOUT: return "bounded wait timed out";
    case CSA2_ERR_ORDER: return "candidate positions not strictly ascending";
    default: return "unknown status";
  }
}

int32_t csa2_version(void) { return 200; }   // 0.2.0: csa2_layer gained local_kv

int32_t csa2_selftest_wait(int32_t kind, uint64_t limit_ns, uint32_t* counter, int32_t* status, void* stream) {
  if (!status || (kind != 0 && kind != 1) || limit_ns > 10000000000ull) return CSA2_ERR_INVALID_ARG;
  if (kind == 0 && (!counter || !aligned(counter, 4))) return CSA2_ERR_INVALID_ARG;
  return cuda_status(launch_wait_selftest(kind, limit_ns, counter, status, static_cast<cudaStream_t>(stream)));
}

size_t csa2_trace_table_bytes(void) {
  return (size_t)kTraceKernels * kTraceCtas * kTracePhases * 2 * sizeof(uint64_t);
}

int32_t csa2_trace_attach(void* table) {
#ifdef CSA2_TRACE
  if (table && !aligned(table, 8)) return CSA2_ERR_INVALID_ARG;
  uint64_t* t = static_cast<uint64_t*>(table);
  cudaError_t (*const attach[])(uint64_t*) = {trace_attach_index, trace_attach_select, trace_attach_reindex,
                                               trace_attach_attn,  trace_attach_rows,   trace_attach_zero,
                                               trace_attach_rcluster};
  for (auto f : attach)
    if (f(t) != cudaSuccess) return CSA2_ERR_CUDA;
  return CSA2_OK;
#else
  (void)table;
  return CSA2_ERR_UNSUPPORTED;   // phase markers are compiled in only in the traced build
#endif
}

size_t csa2_index_full_workspace(int32_t nq, int32_t max_ctx, int32_t P, int32_t K) {
  if (nq < 1 || max_ctx < 1) return 0;
  return index_full_ws(nq, max_ctx, P, K, nullptr, nullptr, nullptr);
}

int32_t csa2_index_full(const int8_t* q, const int8_t* w, const csa2_rows* keys,
                        const int32_t* seq_of_query, const int32_t* query_pos, int32_t nq,
                        int32_t H, int32_t D, int32_t max_ctx, int32_t* scores, int64_t ld_scores,
                        int32_t P, int32_t* pool_idx, int32_t* pool_cnt, int32_t K,
                        int32_t* sel_idx, int32_t* sel_cnt, void* ws, size_t ws_bytes,
                        int32_t* status, void* stream) {
  CSA2_API_RANGE("csa2_index_full");
  if (!q || !w || !query_pos || !status || !aligned(q, 16)) return CSA2_ERR_INVALID_ARG;
  if (nq < 1 || max_ctx < 1 || P < 0 || K < 0 || P > 65536 || K > 65536) return CSA2_ERR_INVALID_ARG;
  if (nq > 4096) return CSA2_ERR_UNSUPPORTED;   // the index-score kernel's work list holds 4096 queries
  if (D != 64 && D != 128) return CSA2_ERR_UNSUPPORTED;
  if (H < 1 || H > 128 || nq > 4096) return CSA2_ERR_UNSUPPORTED;
  if (!rows_ok(keys, D, 16)) return CSA2_ERR_INVALID_ARG;
  if (scores && ld_scores < max_ctx) return CSA2_ERR_INVALID_ARG;
  if ((P > 0 && !pool_idx) || (K > 0 && !sel_idx)) return CSA2_ERR_INVALID_ARG;
  if (!ws || !aligned(ws, 256) || ws_bytes < csa2_index_full_workspace(nq, max_ctx, P, K))
    return CSA2_ERR_WORKSPACE;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  int32_t* sc_ws;
  TopkScratch ts;
  index_full_ws(nq, max_ctx, P, K, ws, &sc_ws, &ts);
  int32_t* sc = scores ? scores : sc_ws;
  const int64_t ld = scores ? ld_scores : max_ctx;
  const bool topk = P > 0 || K > 0;
  if (topk && !launch_opts().prezeroed) {
    cudaError_t e = cudaMemsetAsync(ts.hist, 0, topk_zero_bytes(nq), st);
    if (e != cudaSuccess) return CSA2_ERR_CUDA;
  }
  bool hist_built = false;
  cudaError_t e = launch_index_score(q, w, *keys, seq_of_query, query_pos, nq, H, D, max_ctx, sc, ld,
                                     topk ? ts.hist : nullptr, status, st, &hist_built);
  if (e != cudaSuccess) return CSA2_ERR_CUDA;
  if (!topk) return CSA2_OK;
  TopkOut outs[2];
  int n = 0;
  if (P > 0) outs[n++] = TopkOut{pool_idx, pool_cnt, P};
  if (K > 0) outs[n++] = TopkOut{sel_idx, sel_cnt, K};
  return cuda_status(launch_topk_large(sc, ld, nullptr, query_pos, nullptr, nq, max_ctx, outs, n, ts,
                                       hist_built, status, st));
}

size_t csa2_topk_pool_workspace(int32_t nq, int32_t n_max, int32_t k) {
  (void)k;
  if (nq < 1) return 0;
  if (n_max <= kSmallMax) return 256;
  return topk_scratch_bytes(nq, n_max);
}

int32_t csa2_topk_pool(const int32_t* scores, int64_t ld, const int32_t* n_valid,
                       const int32_t* cand_pos, int32_t nq, int32_t n_max, int32_t k,
                       int32_t* out_idx, int32_t* out_cnt, void* ws, size_t ws_bytes,
                       int32_t* status, void* stream) {
  CSA2_API_RANGE("csa2_topk_pool");
  if (!out_idx || !status || nq < 1 || n_max < 0 || n_max > (1 << 30) || k < 1 || k > 65536)
    return CSA2_ERR_INVALID_ARG;
  if (n_max > 0 && (!scores || ld < n_max)) return CSA2_ERR_INVALID_ARG;
  if (nq > 65535) return CSA2_ERR_UNSUPPORTED;   // queries index a grid dimension
  if (ws_bytes < csa2_topk_pool_workspace(nq, n_max, k) || (n_max > kSmallMax && (!ws || !aligned(ws, 256))))
    return CSA2_ERR_WORKSPACE;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (n_max <= kSmallMax)
    return cuda_status(launch_topk_small(scores, ld, n_valid, cand_pos, nq, n_max, k, out_idx, out_cnt,
                                         status, st));
  Carver c(ws);
  TopkScratch ts = carve_topk(c, nq, n_max);
  TopkOut o{out_idx, out_cnt, k};
  return cuda_status(launch_topk_large(scores, ld, n_valid, nullptr, cand_pos, nq, n_max, &o, 1, ts,
                                       false, status, st));
}

size_t csa2_reindex_workspace(int32_t nq, int32_t P, int32_t K) {
  (void)K;
  if (nq < 1 || P < 1) return 0;
  return reindex_ws(nq, P, 1, nullptr, nullptr, nullptr, nullptr);
}

int32_t csa2_reindex(const int8_t* q, const int8_t* w, const csa2_rows* keys,
                     const int32_t* seq_of_query, const int32_t* pool_idx, const int32_t* pool_cnt,
                     int32_t nq, int32_t H, int32_t D, int32_t P, int32_t K, int32_t* sel_idx,
                     int32_t* sel_cnt, int32_t* scores, void* ws, size_t ws_bytes, int32_t* status,
                     void* stream) {
  CSA2_API_RANGE("csa2_reindex");
  if (!q || !w || !pool_idx || !pool_cnt || !sel_idx || !status || !aligned(q, 16))
    return CSA2_ERR_INVALID_ARG;
  if (nq < 1 || P < 1 || P > 65536 || K < 1 || K > P) return CSA2_ERR_INVALID_ARG;
  if (D != 64 && D != 128) return CSA2_ERR_UNSUPPORTED;
  if (H < 1 || H > 128 || nq > 65535) return CSA2_ERR_UNSUPPORTED;
  if (!rows_ok(keys, D, 16)) return CSA2_ERR_INVALID_ARG;
  if (!ws || !aligned(ws, 256) || ws_bytes < csa2_reindex_workspace(nq, P, K)) return CSA2_ERR_WORKSPACE;
  const ReindexJobDesc job{q, w, keys, scores, sel_idx, sel_cnt};
  return run_reindex(&job, 1, seq_of_query, pool_idx, pool_cnt, nq, H, D, P, K, ws, status,
                     static_cast<cudaStream_t>(stream));
}

size_t csa2_sparse_attn_workspace(int32_t nq, int32_t Hq, int32_t D, int32_t K, int32_t window) {
  if (nq < 1 || Hq < 1 || D < 1 || K < 0 || window < 0) return 0;
  return attn_scratch_bytes(nq, Hq, D, K, window);
}

static int32_t check_attn(const uint16_t* q, const csa2_rows* codes, const csa2_rows* scales,
                          const int32_t* query_pos, int32_t nq, int32_t Hq, int32_t D, int32_t K,
                          int32_t window, const uint16_t* out) {
  if (!q || !query_pos || !out || !aligned(q, 16) || !aligned(out, 16)) return CSA2_ERR_INVALID_ARG;
  if (nq < 1 || nq > 65535 || K < 0 || K > 65536 || window < 0 || window > 1024) return CSA2_ERR_INVALID_ARG;
  if (D != 128 && D != 512) return CSA2_ERR_UNSUPPORTED;
  if (Hq < 8 || Hq > 128 || Hq % 8) return CSA2_ERR_UNSUPPORTED;
  if (!rows_ok(codes, D / 2, 16) || !rows_ok(scales, D / 32, 1)) return CSA2_ERR_INVALID_ARG;
  return CSA2_OK;
}

// A local window cache: contiguous bf16 rows of D values, a ring of at least
// `window` rows per sequence.
static bool local_ok(const csa2_rows* v, int32_t D, int32_t window) {
  return rows_ok(v, 2 * (int64_t)D, 16) && !v->page_table && v->seq_rows >= window;
}

static int32_t run_attn(const uint16_t* q, const csa2_rows* codes, const csa2_rows* scales,
                        const csa2_rows* local_kv, const int32_t* seq_of_query, const int32_t* query_pos,
                        const int32_t* sel_idx, const int32_t* sel_cnt, int32_t nq, int32_t Hq, int32_t D,
                        int32_t K, int32_t window, float softmax_scale, uint16_t* out, float* lse, void* ws,
                        size_t ws_bytes, int32_t* status, void* stream) {
  int32_t r = check_attn(q, codes, scales, query_pos, nq, Hq, D, K, window, out);
  if (r != CSA2_OK) return r;
  if (!status || (K > 0 && !sel_idx)) return CSA2_ERR_INVALID_ARG;
  if (local_kv && !local_ok(local_kv, D, window)) return CSA2_ERR_INVALID_ARG;
  if (!ws || !aligned(ws, 256) || ws_bytes < csa2_sparse_attn_workspace(nq, Hq, D, K, window))
    return CSA2_ERR_WORKSPACE;
  const float scale = softmax_scale > 0.f ? softmax_scale : 1.0f / sqrtf((float)D);
  return cuda_status(launch_sparse_attn(q, *codes, *scales, local_kv, seq_of_query, query_pos, sel_idx, sel_cnt,
                                        nq, Hq, D, K, window, scale, out, lse, ws, ws_bytes, status,
                                        static_cast<cudaStream_t>(stream)));
}

int32_t csa2_sparse_attn_fp4(const uint16_t* q, const csa2_rows* codes, const csa2_rows* scales,
                             const int32_t* seq_of_query, const int32_t* query_pos,
                             const int32_t* sel_idx, const int32_t* sel_cnt, int32_t nq, int32_t Hq,
                             int32_t D, int32_t K, int32_t window, float softmax_scale, uint16_t* out,
                             float* lse, void* ws, size_t ws_bytes, int32_t* status, void* stream) {
  CSA2_API_RANGE("csa2_sparse_attn_fp4");
  return run_attn(q, codes, scales, nullptr, seq_of_query, query_pos, sel_idx, sel_cnt, nq, Hq, D, K, window,
                  softmax_scale, out, lse, ws, ws_bytes, status, stream);
}

int32_t csa2_sparse_attn_fp4_local(const uint16_t* q, const csa2_rows* codes, const csa2_rows* scales,
                                   const csa2_rows* local_kv, const int32_t* seq_of_query,
                                   const int32_t* query_pos, const int32_t* sel_idx, const int32_t* sel_cnt,
                                   int32_t nq, int32_t Hq, int32_t D, int32_t K, int32_t window,
                                   float softmax_scale, uint16_t* out, float* lse, void* ws, size_t ws_bytes,
                                   int32_t* status, void* stream) {
  CSA2_API_RANGE("csa2_sparse_attn_fp4_local");
  if (!local_kv) return CSA2_ERR_INVALID_ARG;
  return run_attn(q, codes, scales, local_kv, seq_of_query, query_pos, sel_idx, sel_cnt, nq, Hq, D, K, window,
                  softmax_scale, out, lse, ws, ws_bytes, status, stream);
}

// ------------------------------------------------------------------ layer plan
namespace {

struct PlanWs {
  size_t index_ws, reindex_ws, attn_ws;
  void* index_base;
  void* reindex_base;
  void* attn_base;
  int32_t* pool[kMaxAttnJobs];
  int32_t* pool_cnt[kMaxAttnJobs];
  int32_t* sel[kMaxAttnJobs];
  int32_t* sel_cnt[kMaxAttnJobs];
  size_t total;
};

PlanWs carve_plan(const int32_t* modes, int32_t L, const csa2_plan_shape* s, void* base) {
  PlanWs p{};
  Carver c(base);
  p.index_ws = csa2_index_full_workspace(s->nq, s->max_ctx, s->P, s->K);
  p.index_base = c.take<char>(p.index_ws);
  int n_reindex = 0;
  for (int i = 0; i < L; ++i) n_reindex += modes[i] == CSA2_REINDEX;
  const int group = n_reindex < kMaxReindexJobs ? n_reindex : kMaxReindexJobs;
  p.reindex_ws = group ? reindex_ws(s->nq, s->P, group, nullptr, nullptr, nullptr, nullptr) : 0;
  p.reindex_base = c.take<char>(p.reindex_ws);
  p.attn_ws = csa2_sparse_attn_workspace(s->nq, s->Hq, s->D, s->K, s->window) * (size_t)L;
  p.attn_base = c.take<char>(p.attn_ws);
  for (int i = 0; i < L; ++i) {
    if (modes[i] == CSA2_FULL) {
      p.pool[i] = c.take<int32_t>((size_t)s->nq * s->P);
      p.pool_cnt[i] = c.take<int32_t>((size_t)s->nq);
    }
    if (modes[i] == CSA2_FULL || modes[i] == CSA2_REINDEX) {
      p.sel[i] = c.take<int32_t>((size_t)s->nq * s->K);
      p.sel_cnt[i] = c.take<int32_t>((size_t)s->nq);
    }
  }
  p.total = c.used + 256;
  return p;
}

bool plan_modes_ok(const int32_t* modes, int32_t L) {
  if (!modes || L < 1 || L > kMaxAttnJobs || modes[0] != CSA2_FULL) return false;
  for (int i = 0; i < L; ++i)
    if (modes[i] != CSA2_FULL && modes[i] != CSA2_REINDEX && modes[i] != CSA2_REUSE) return false;
  return true;
}

}  // namespace

size_t csa2_layer_plan_workspace(const int32_t* modes, int32_t L, const csa2_plan_shape* shape) {
  if (!plan_modes_ok(modes, L) || !shape || shape->nq < 1 || shape->max_ctx < 1 || shape->P < 1 ||
      shape->K < 1)
    return 0;
  return carve_plan(modes, L, shape, nullptr).total;
}

int32_t csa2_layer_plan(const int32_t* modes, int32_t L, const csa2_layer* layers,
                        const csa2_plan_shape* s, void* ws, size_t ws_bytes, int32_t* status,
                        void* stream) {
  CSA2_API_RANGE("csa2_layer_plan");
  if (!plan_modes_ok(modes, L) || !layers || !s || !status) return CSA2_ERR_INVALID_ARG;
  if (s->P < 1 || s->K < 1 || s->K > s->P || !s->query_pos) return CSA2_ERR_INVALID_ARG;
  if ((int64_t)s->nq * L > 65535) return CSA2_ERR_UNSUPPORTED;   // one attention launch: a grid z of nq * L
  for (int i = 0; i < L; ++i) {
    const csa2_layer& ly = layers[i];
    int32_t r = check_attn(ly.q_attn, &ly.codes, &ly.scales, s->query_pos, s->nq, s->Hq, s->D, s->K,
                           s->window, ly.out);
    if (r != CSA2_OK) return r;
    if (ly.local_kv.base && !local_ok(&ly.local_kv, s->D, s->window)) return CSA2_ERR_INVALID_ARG;
    if (modes[i] != CSA2_REUSE) {
      if (!ly.q || !ly.w || !aligned(ly.q, 16)) return CSA2_ERR_INVALID_ARG;
      if (s->D_idx != 64 && s->D_idx != 128) return CSA2_ERR_UNSUPPORTED;
      if (s->H < 1 || s->H > 128 || s->nq > 4096) return CSA2_ERR_UNSUPPORTED;
      if (!rows_ok(&ly.keys, s->D_idx, 16)) return CSA2_ERR_INVALID_ARG;
    }
  }
  const size_t need = csa2_layer_plan_workspace(modes, L, s);
  if (!ws || !aligned(ws, 256) || ws_bytes < need) return CSA2_ERR_WORKSPACE;
  PlanWs p = carve_plan(modes, L, s, ws);
  cudaStream_t st = static_cast<cudaStream_t>(stream);

  // Which buffers every layer reads and writes.  A REINDEX layer searches the
  // pool of the latest FULL layer; a REUSE layer attends to the selection of
  // the latest FULL or REINDEX layer.
  int32_t* pool_of[kMaxAttnJobs];
  int32_t* pool_cnt_of[kMaxAttnJobs];
  int32_t* sel_of[kMaxAttnJobs];
  int32_t* sel_cnt_of[kMaxAttnJobs];
  for (int i = 0; i < L; ++i) {
    const csa2_layer& ly = layers[i];
    if (modes[i] == CSA2_FULL) {
      pool_of[i] = ly.pool_idx ? ly.pool_idx : p.pool[i];
      pool_cnt_of[i] = ly.pool_cnt ? ly.pool_cnt : p.pool_cnt[i];
    } else {
      pool_of[i] = pool_of[i - 1];
      pool_cnt_of[i] = pool_cnt_of[i - 1];
    }
    if (modes[i] == CSA2_REUSE) {
      sel_of[i] = sel_of[i - 1];
      sel_cnt_of[i] = sel_cnt_of[i - 1];
    } else {
      sel_of[i] = ly.sel_idx ? ly.sel_idx : p.sel[i];
      sel_cnt_of[i] = ly.sel_cnt ? ly.sel_cnt : p.sel_cnt[i];
    }
  }
  // One launch zeroes all scratch of the step up front when every piece is
  // used once (one FULL layer, at most one reindex launch), so the kernels of
  // the step then follow one another as programmatic dependents.
  int n_full = 0, n_reindex = 0;
  for (int i = 0; i < L; ++i) {
    n_full += modes[i] == CSA2_FULL;
    n_reindex += modes[i] == CSA2_REINDEX;
  }
  LaunchOpts opts;
  opts.group = s->group_queries != 0;
  opts.plan = true;
  if (n_full == 1 && n_reindex <= kMaxReindexJobs) {
    void* zp[3];
    size_t zb[3];
    int nz = 0;
    TopkScratch ts;
    index_full_ws(s->nq, s->max_ctx, s->P, s->K, p.index_base, nullptr, &ts);
    zp[nz] = ts.hist;
    zb[nz++] = topk_zero_bytes(s->nq);
    if (n_reindex > 0) {
      zp[nz] = p.reindex_base;   // the fused launch's histograms and headers lead its scratch
      zb[nz++] = (size_t)n_reindex * s->nq * (kBuckets + 4) * sizeof(uint32_t);
    }
    attn_bar_region(p.attn_base, L, s->nq, s->Hq, s->D, &zp[nz], &zb[nz]);
    ++nz;
    if (launch_zero(zp, zb, nz, st) != cudaSuccess) return CSA2_ERR_CUDA;
    opts.pdl = true;
    opts.prezeroed = true;
  }
  LaunchOptsScope scope(opts);
  // Every FULL layer, then in one launch the REINDEX layers that search its pool.
  for (int i = 0; i < L; ++i) {
    if (modes[i] != CSA2_FULL) continue;
    const csa2_layer& ly = layers[i];
    int32_t r = csa2_index_full(ly.q, ly.w, &ly.keys, s->seq_of_query, s->query_pos, s->nq, s->H, s->D_idx,
                                s->max_ctx, nullptr, 0, s->P, pool_of[i], pool_cnt_of[i], s->K, sel_of[i],
                                sel_cnt_of[i], p.index_base, p.index_ws, status, stream);
    if (r != CSA2_OK) return r;
    ReindexJobDesc rj[kMaxReindexJobs];
    int n = 0;
    for (int j = i + 1; j <= L; ++j) {
      const bool end = j == L || modes[j] == CSA2_FULL;
      if (!end && modes[j] == CSA2_REINDEX)
        rj[n++] = ReindexJobDesc{layers[j].q, layers[j].w, &layers[j].keys, nullptr, sel_of[j], sel_cnt_of[j]};
      if (n > 0 && (end || n == kMaxReindexJobs)) {
        r = run_reindex(rj, n, s->seq_of_query, pool_of[i], pool_cnt_of[i], s->nq, s->H, s->D_idx, s->P, s->K,
                        p.reindex_base, status, st);
        if (r != CSA2_OK) return r;
        n = 0;
      }
      if (end) break;
    }
  }
  // REUSE layers with outputs of their own get a copy of the selection they use.
  AttnJobDesc jobs[kMaxAttnJobs];
  for (int i = 0; i < L; ++i) {
    const csa2_layer& ly = layers[i];
    if (modes[i] == CSA2_REUSE) {
      if (ly.sel_idx && ly.sel_idx != sel_of[i]) {
        if (cudaMemcpyAsync(ly.sel_idx, sel_of[i], (size_t)s->nq * s->K * 4, cudaMemcpyDeviceToDevice, st) !=
            cudaSuccess)
          return CSA2_ERR_CUDA;
      }
      if (ly.sel_cnt && ly.sel_cnt != sel_cnt_of[i]) {
        if (cudaMemcpyAsync(ly.sel_cnt, sel_cnt_of[i], (size_t)s->nq * 4, cudaMemcpyDeviceToDevice, st) !=
            cudaSuccess)
          return CSA2_ERR_CUDA;
      }
    }
    jobs[i] = AttnJobDesc{ly.q_attn, &ly.codes,  &ly.scales, sel_of[i], sel_cnt_of[i],
                          ly.out,    ly.lse,     ly.local_kv.base ? &ly.local_kv : nullptr};
  }
  const float scale = s->softmax_scale > 0.f ? s->softmax_scale : 1.0f / sqrtf((float)s->D);
  return cuda_status(launch_sparse_attn_jobs(jobs, L, s->seq_of_query, s->query_pos, s->nq, s->Hq, s->D, s->K,
                                             s->window, scale, p.attn_base, status, st));
}

// ------------------------------------------------------------------ combine of partial attention
int32_t csa2_attn_combine(const uint16_t* o_parts, const float* lse_parts, int32_t R, int32_t nq, int32_t Hq,
                          int32_t D, uint16_t* out, float* lse_out, int32_t* status, void* stream) {
  CSA2_API_RANGE("csa2_attn_combine");
  if (!o_parts || !lse_parts || !out || !status || !aligned(o_parts, 16) || !aligned(out, 16))
    return CSA2_ERR_INVALID_ARG;
  if (R < 1 || R > 4096 || nq < 1 || Hq < 1 || (int64_t)nq * Hq > (1 << 26)) return CSA2_ERR_INVALID_ARG;
  if (D < 8 || D > 1024 || D % 8) return CSA2_ERR_UNSUPPORTED;
  return cuda_status(launch_attn_combine(o_parts, lse_parts, R, nq, Hq, D, out, lse_out,
                                         static_cast<cudaStream_t>(stream)));
}

// ------------------------------------------------------------------ FP4 cache write
// fp32 or bf16 rows, each starting on 16 bytes: ld_x a multiple of the values per 16 bytes.
static int32_t run_fp4_quantize(const void* x, bool bf16, int64_t n_rows, int32_t D, int64_t ld_x,
                                const int32_t* dst_rows, uint8_t* codes, int64_t ld_codes, uint8_t* scales,
                                int64_t ld_scales, int64_t n_dst_rows, int32_t* status, void* stream) {
  const int64_t per16 = bf16 ? 8 : 4;   // values per 16 bytes
  if (!status || n_rows < 0 || (n_rows > 0 && (!x || !codes || !scales))) return CSA2_ERR_INVALID_ARG;
  if (D < 32 || D > 4096 || D % 32) return CSA2_ERR_UNSUPPORTED;
  if (ld_x < D || ld_x % per16 || !aligned(x, 16) || !aligned(codes, 16) || ld_codes < D / 2 || ld_codes % 16 ||
      ld_scales < D / 32 || n_dst_rows < 1)
    return CSA2_ERR_INVALID_ARG;
  return cuda_status(launch_fp4_quantize(x, bf16, n_rows, D, ld_x, dst_rows, codes, ld_codes, scales, ld_scales,
                                         n_dst_rows, status, static_cast<cudaStream_t>(stream)));
}

int32_t csa2_fp4_quantize(const float* x, int64_t n_rows, int32_t D, int64_t ld_x, const int32_t* dst_rows,
                          uint8_t* codes, int64_t ld_codes, uint8_t* scales, int64_t ld_scales,
                          int64_t n_dst_rows, int32_t* status, void* stream) {
  CSA2_API_RANGE("csa2_fp4_quantize");
  return run_fp4_quantize(x, false, n_rows, D, ld_x, dst_rows, codes, ld_codes, scales, ld_scales, n_dst_rows,
                          status, stream);
}

int32_t csa2_fp4_quantize_bf16(const uint16_t* x, int64_t n_rows, int32_t D, int64_t ld_x,
                               const int32_t* dst_rows, uint8_t* codes, int64_t ld_codes, uint8_t* scales,
                               int64_t ld_scales, int64_t n_dst_rows, int32_t* status, void* stream) {
  CSA2_API_RANGE("csa2_fp4_quantize_bf16");
  return run_fp4_quantize(x, true, n_rows, D, ld_x, dst_rows, codes, ld_codes, scales, ld_scales, n_dst_rows,
                          status, stream);
}

}  // extern "C"
