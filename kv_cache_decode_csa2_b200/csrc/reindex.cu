// K3: reindex scoring.  A reindex layer re-scores only the candidate pool
// ("later layers search only that much smaller pool instead of rescanning
// everything": "DeepSeek V4.1-Flash: 552B runs like 16B", Act 2).
//
// One CTA per (query, 128 pool slots).  The CTA gathers the pool rows of this
// layer's index keys by position into a swizzled K-major tile (16-byte cp.async
// per chunk: a pool row is one 128-byte line).  It runs one tcgen05 int8 MMA
// group, D[128 slots x N heads] in TMEM, and applies the ReLU and head-weight
// epilogue of the full-mode scorer.
//
// reindex_select_kernel goes on to the top-K of the layer in the same launch.
// The CTAs of a pool (every CTA holds 128 of its scores, one per thread) are
// co-resident and meet at bounded grid barriers; batches of pools too large
// to be co-resident let the CTA of each pool that finishes its scores last
// select alone (see LAST below).  They build the bucket
// histogram of the pool in global memory, find the threshold bucket b*, rank
// the ties at b* (the pool's tie list, staged in shared memory), and write the
// members in slot order, which is position order because pool positions
// ascend.  One launch serves every reindex layer that searches the same pool.
// reindex_score_kernel alone (scores, then the select kernel) serves the
// batches too large to be co-resident.
#include "csa2_device.cuh"
#include "internal.h"
#include "select_common.cuh"

namespace csa2 {

CSA2_TRACE_UNIT(reindex)

namespace {

struct ReindexArgs {
  const int8_t* q;
  const int8_t* w;
  const int32_t* seq_of_query;
  const int32_t* pool_idx;
  const int32_t* pool_cnt;
  const uint8_t* base;
  int64_t row_bytes;
  RowMap rows;
  int32_t H, P;
  int32_t* scores;
  int32_t* status;
};

__device__ __forceinline__ void cp_async16(void* dst, const void* src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(smem_u32(dst)), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async_wait_all() { asm volatile("cp.async.wait_all;" ::: "memory"); }

template <int D, int N>
__global__ void __launch_bounds__(128) reindex_score_kernel(const ReindexArgs a) {
  constexpr uint32_t TMEM_COLS = N <= 32 ? 32 : (N <= 64 ? 64 : 128);
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* atile = smem;                       // 128 x D
  uint8_t* bmat = atile + 128 * D;             // N x D
  int32_t* w_s = reinterpret_cast<int32_t*>(bmat + N * D);
  uint64_t* bar = reinterpret_cast<uint64_t*>(w_s + 128);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bar + 1);

  const int q = blockIdx.y;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  int32_t cnt = __ldg(a.pool_cnt + q);
  cnt = cnt < 0 ? 0 : (cnt > a.P ? a.P : cnt);
  const int32_t slot0 = blockIdx.x * 128;
  if (slot0 >= cnt) return;
  const int32_t seq = a.seq_of_query ? __ldg(a.seq_of_query + q) : q;

  if (warp == 0) {
    tmem_alloc(tmem_slot, TMEM_COLS);
    tmem_relinquish();
  }
  if (tid == 0) {
    mbar_init(bar, 1);
    fence_mbar_init();
  }
  // gather: row r of the tile <- index-key row of pool slot slot0 + r
  {
    const int r = tid;
    const int32_t slot = slot0 + r;
    const uint8_t* src = nullptr;
    if (slot < cnt) {
      const int32_t pos = __ldg(a.pool_idx + (int64_t)q * a.P + slot);
      const int64_t row = pos >= 0 ? map_row(a.rows, seq, pos) : -1;
      if (row < 0) record_error(a.status, CSA2_ERR_INDEX_RANGE);
      else src = a.base + row * a.row_bytes;
    }
#pragma unroll
    for (int c = 0; c < D / 16; ++c) {
      uint8_t* dst = atile + swizzled_chunk(r, c, D);
      if (src) cp_async16(dst, src + 16 * c);
      else *reinterpret_cast<int4*>(dst) = make_int4(0, 0, 0, 0);
    }
  }
  const int8_t* qsrc = a.q + (int64_t)q * a.H * D;
  for (int idx = tid; idx < N * (D / 16); idx += 128) {
    const int r = idx / (D / 16), c = idx % (D / 16);
    int4 v = make_int4(0, 0, 0, 0);
    if (r < a.H) v = __ldg(reinterpret_cast<const int4*>(qsrc + r * D) + c);
    *reinterpret_cast<int4*>(bmat + swizzled_chunk(r, c, D)) = v;
  }
  if (tid < N) w_s[tid] = tid < a.H ? (int32_t)__ldg(a.w + (int64_t)q * a.H + tid) : 0;
  cp_async_wait_all();
  fence_async_smem();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  if (tid == 0) {
    constexpr uint32_t idesc = idesc_i8(128, N);
    const uint32_t a_addr = smem_u32(atile), b_addr = smem_u32(bmat);
#pragma unroll
    for (int k = 0; k < D / 32; ++k)
      mma_i8(tmem_base, smem_desc_kmajor(a_addr + 32 * k, D), smem_desc_kmajor(b_addr + 32 * k, D),
             idesc, k > 0 ? 1u : 0u);
    mma_commit(bar);
  }
  // every thread waits; the result is warp-uniform before the collective loads
  volatile int32_t never = 0;
  const bool ok = __all_sync(0xffffffffu, mbar_wait(bar, 0, &never));
  if (ok) {
    tc_fence_after();
    const uint32_t taddr = tmem_base + ((uint32_t)(warp * 32) << 16);
    int32_t s = 0;
    if constexpr (N == 16) {
      uint32_t r16[16];
      tmem_ld16(taddr, r16);
      tmem_wait_ld();
#pragma unroll
      for (int h = 0; h < 16; ++h) s += w_s[h] * max((int32_t)r16[h], 0);
    } else {
#pragma unroll 1
      for (int g = 0; g < N / 32; ++g) {
        uint32_t r32[32];
        tmem_ld32(taddr + 32 * g, r32);
        tmem_wait_ld();
#pragma unroll
        for (int h = 0; h < 32; ++h) s += w_s[g * 32 + h] * max((int32_t)r32[h], 0);
      }
    }
    const int32_t slot = slot0 + warp * 32 + lane;
    if (slot < cnt) a.scores[(int64_t)q * a.P + slot] = s;
  } else if (tid == 0) {
    record_error(a.status, CSA2_ERR_TIMEOUT);
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem_base, TMEM_COLS);
  }
}

template <int D, int N>
cudaError_t launch_r(const ReindexArgs& a, int nq, cudaStream_t st) {
  const size_t smem = 1024 + 128 * D + N * D + 128 * 4 + 64;
  static SetupMask done{0};
  cudaError_t e = ensure_smem(reindex_score_kernel<D, N>, (int)smem, done);
  if (e != cudaSuccess) return e;
  const dim3 grid((a.P + 127) / 128, nq);
  reindex_score_kernel<D, N><<<grid, 128, smem, st>>>(a);
  return cudaGetLastError();
}


// ------------------------------------------------------------------ fused scoring + top-K
constexpr int kRTieCap = 2048;   // ties of one pool ranked in shared memory (more: radix select)

struct RSelJob {
  const int8_t* q;
  const int8_t* w;
  const uint8_t* base;
  int64_t row_bytes;
  RowMap rows;
  int32_t* scores;    // [nq][P] or nullptr
  int32_t* sel_idx;   // [nq][K]
  int32_t* sel_cnt;   // [nq] or nullptr
};

struct RSelArgs {
  RSelJob job[kMaxReindexJobs];
  const int32_t* seq_of_query;
  const int32_t* pool_idx;
  const int32_t* pool_cnt;
  int32_t H, P, K, nq, G;
  uint32_t* hist;     // [probs][kBuckets]   zeroed before the launch
  uint32_t* hdr;      // [probs][4]          zeroed before the launch: barrier count, tie count
  uint64_t* ties;     // [probs][kRTieCap]
  uint32_t* mcnt;     // [probs][G]
  uint32_t* radix;    // [probs][8][256]
  int32_t* sc;        // [probs][P] scores of pools whose job keeps none (last-CTA select)
  int32_t* status;
};

// Dynamic shared memory: the T tiles of 128 pool rows and the query (then the
// pool's ties), w, this CTA's ties, the MMA barrier and the TMEM address.
// LAST: the region holds, after scoring, the pool's scores and the padded
// histogram (then the ties) of the selecting CTA.
template <int D, int N, int T, bool LAST>
struct RSelLayout {
  static constexpr int NT = 128 * T;
  static constexpr size_t tiles = (size_t)(T * 128 * D + N * D);
  static constexpr size_t ties_or_hist = LAST ? (size_t)kRLastMaxP * 4 + (size_t)(kBuckets + kBuckets / 32) * 4
                                         : (size_t)kRTieCap * 8 > (size_t)kBuckets * 4 ? (size_t)kRTieCap * 8
                                                                                        : (size_t)kBuckets * 4;
  static constexpr size_t region = tiles > ties_or_hist ? tiles : ties_or_hist;   // reused after scoring
  static constexpr size_t smem = 1024 + region + 128 * 4 + NT * 8 + 64;
  static constexpr uint32_t cols = T * N <= 32 ? 32 : T * N <= 64 ? 64 : T * N <= 128 ? 128 : 256;
};

// T tiles of 128 pool slots per CTA (one slot per thread): the device holds
// one such CTA per SM, so T sets how many pools fit in one launch.
//
// LAST: every CTA publishes its scores and counts itself in with one
// acquire-release add; the CTA that arrives last (it then sees every score of
// the pool) selects the pool's top-K alone: kRLastE consecutive slots per
// thread in registers, the bucket histogram in shared memory, the ties at
// the threshold bucket ranked in shared memory, one block scan for the
// output slots.  Nothing waits on another CTA, so the grid need not be
// co-resident, and the CTAs that are not last leave as soon as they have
// published, which lets the next launch start on their SMs.
constexpr int kRLastE = 64;                              // slots per thread of the selecting CTA
constexpr int kRLastHist = kBuckets + kBuckets / 32;     // padded histogram words
template <int D, int N, int T, bool LAST>
__global__ void __launch_bounds__(128 * T, LAST ? 2 : 1) reindex_select_kernel(const __grid_constant__ RSelArgs a) {
  using Lay = RSelLayout<D, N, T, LAST>;
  constexpr int NT = Lay::NT;
  constexpr uint32_t TMEM_COLS = Lay::cols;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* atile = smem;                                   // T x 128 x D   (scoring)
  uint8_t* bmat = atile + T * 128 * D;                     // N x D         (scoring)
  uint64_t* rowties = reinterpret_cast<uint64_t*>(smem);   // the pool's ties (after scoring)
  int32_t* w_s = reinterpret_cast<int32_t*>(smem + Lay::region);
  uint64_t* own = reinterpret_cast<uint64_t*>(w_s + 128);  // this CTA's ties (at most NT)
  uint64_t* bar = own + NT;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bar + 1);
  __shared__ uint64_t wtmp[NT / 32];
  __shared__ int32_t bstar_s, above_s;
  __shared__ uint32_t own_cnt, wcnt[NT / 32];
  __shared__ unsigned long long kthr_s;
  __shared__ RadixSmem rsm;

  const int x = blockIdx.x, q = blockIdx.y, jb = blockIdx.z;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const RSelJob& J = a.job[jb];
  const int prob = jb * a.nq + q;
  const int G = a.G;
  // trace points: 1 own inputs staged, 2 grid before done, 3 pool rows
  // gathered, 4 scored, 5 histogram barrier (LAST: scores published), 6
  // threshold bucket, 7 tie barrier, 8 ties ranked, 9 count barrier, 10
  // written (LAST: 6, 8 and 10 in the selecting CTA only)
  CSA2_TRACE_BEGIN(kTrReindex, tid == 0);
  if (tid == 0) {
    bstar_s = -1;
    above_s = 0;
    own_cnt = 0;
    kthr_s = ~0ull;
  }

  // ---- prologue on this layer's own inputs: TMEM, the MMA barrier, the
  // query rows (B operand) and the head weights
  if (warp == 0) {
    tmem_alloc(tmem_slot, TMEM_COLS);
    tmem_relinquish();
  }
  if (tid == 0) {
    mbar_init(bar, 1);
    fence_mbar_init();
  }
  {
    const int8_t* qsrc = J.q + (int64_t)q * a.H * D;
    for (int idx = tid; idx < N * (D / 16); idx += NT) {
      const int r = idx / (D / 16), c = idx % (D / 16);
      int4 v = make_int4(0, 0, 0, 0);
      if (r < a.H) v = __ldg(reinterpret_cast<const int4*>(qsrc + r * D) + c);
      *reinterpret_cast<int4*>(bmat + swizzled_chunk(r, c, D)) = v;
    }
    if (tid < N) w_s[tid] = tid < a.H ? (int32_t)__ldg(J.w + (int64_t)q * a.H + tid) : 0;
  }
  CSA2_MARK(kTrReindex, 1, tid == 0);
  pdl_wait();      // the pool comes from the grid before
  pdl_trigger();
  CSA2_MARK(kTrReindex, 2, tid == 0);

  int32_t cnt = __ldg(a.pool_cnt + q);
  cnt = cnt < 0 ? 0 : (cnt > a.P ? a.P : cnt);
  const int32_t slot0 = x * NT, slot = slot0 + tid;
  const bool has = slot0 < cnt;   // CTA-uniform: this CTA holds pool entries
  const bool valid = slot < cnt;
  const int32_t* pidx = a.pool_idx + (int64_t)q * a.P;
  const int32_t pos = valid ? __ldg(pidx + slot) : -1;
  const int32_t prev = (valid && slot > 0) ? __ldg(pidx + slot - 1) : INT32_MIN;
  if (valid && pos <= prev) record_error(a.status, CSA2_ERR_ORDER);   // pool positions ascend

  // ---- scores of this CTA's NT pool entries (one per thread)
  int32_t s = 0;
  if (has) {
    const int32_t seq = a.seq_of_query ? __ldg(a.seq_of_query + q) : q;
    {
      const uint8_t* src = nullptr;
      if (valid) {
        const int64_t row = pos >= 0 ? map_row(J.rows, seq, pos) : -1;
        if (row < 0) record_error(a.status, CSA2_ERR_INDEX_RANGE);
        else src = J.base + row * J.row_bytes;
      }
      uint8_t* tile = atile + (tid >> 7) * 128 * D;
#pragma unroll
      for (int c = 0; c < D / 16; ++c) {
        uint8_t* dst = tile + swizzled_chunk(tid & 127, c, D);
        if (src) cp_async16(dst, src + 16 * c);
        else *reinterpret_cast<int4*>(dst) = make_int4(0, 0, 0, 0);
      }
    }
    cp_async_wait_all();
    fence_async_smem();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  CSA2_MARK(kTrReindex, 3, tid == 0);
  const uint32_t tmem_base = *tmem_slot;
  if (has) {
    if (tid == 0) {
      constexpr uint32_t idesc = idesc_i8(128, N);
      const uint32_t a_addr = smem_u32(atile), b_addr = smem_u32(bmat);
#pragma unroll
      for (int t = 0; t < T; ++t)   // tile t accumulates in TMEM columns [t N, t N + N)
#pragma unroll
        for (int k = 0; k < D / 32; ++k)
          mma_i8(tmem_base + t * N, smem_desc_kmajor(a_addr + t * 128 * D + 32 * k, D),
                 smem_desc_kmajor(b_addr + 32 * k, D), idesc, k > 0 ? 1u : 0u);
      mma_commit(bar);
    }
    volatile int32_t never = 0;
    const bool ok = __all_sync(0xffffffffu, mbar_wait(bar, 0, &never));
    if (ok) {
      tc_fence_after();
      // warp w reads TMEM lanes 32 (w % 4) .. (a warp's lane quarter) of tile w / 4
      const uint32_t taddr = tmem_base + ((uint32_t)((warp & 3) * 32) << 16) + (uint32_t)((warp >> 2) * N);
      if constexpr (N == 16) {
        uint32_t r16[16];
        tmem_ld16(taddr, r16);
        tmem_wait_ld();
#pragma unroll
        for (int h = 0; h < 16; ++h) s += w_s[h] * max((int32_t)r16[h], 0);
      } else {
#pragma unroll 1
        for (int g = 0; g < N / 32; ++g) {
          uint32_t r32[32];
          tmem_ld32(taddr + 32 * g, r32);
          tmem_wait_ld();
#pragma unroll
          for (int h = 0; h < 32; ++h) s += w_s[g * 32 + h] * max((int32_t)r32[h], 0);
        }
      }
    } else if (tid == 0) {
      record_error(a.status, CSA2_ERR_TIMEOUT);
    }
  }
  tc_fence_before();
  __syncthreads();   // also: the tiles are free for the tie list from here on
  CSA2_MARK(kTrReindex, 4, tid == 0);
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem_base, TMEM_COLS);
  }
  if constexpr (LAST) {
    static_assert(NT * kRLastE >= kRLastMaxP, "the selecting CTA holds a whole pool");
    int32_t* srow = J.scores ? J.scores + (int64_t)q * a.P : a.sc + (size_t)prob * a.P;
    uint32_t* hdr = a.hdr + (size_t)prob * 4;
    if (valid) srow[slot] = s;
    __shared__ uint32_t last_s;
    __syncthreads();   // the CTA's scores are stored before thread 0's release
    if (tid == 0) {
      uint32_t old;
      asm volatile("atom.acq_rel.gpu.global.add.u32 %0, [%1], 1;" : "=r"(old) : "l"(hdr) : "memory");
      last_s = old == (uint32_t)G - 1u;
    }
    __syncthreads();
    CSA2_MARK(kTrReindex, 5, tid == 0);
    if (!last_s) return;

    // ---- the last CTA: every score of the pool is visible (thread 0's
    // acquire, then the block barrier).  Thread t owns the kRLastE slots
    // j0 = t kRLastE ..; shared memory holds the scores with slot j0 + u at
    // sc_s[u NT + t] (lanes read consecutive words), then the bucket
    // histogram with one pad word per 32 bins (bin b at b + b / 32), so that
    // the thread owning bins 32 t .. 32 t + 31 reads them without conflicts.
    // Loops stay rolled: this code runs once per pool, from a cold
    // instruction cache.
    int32_t* sc_s = reinterpret_cast<int32_t*>(smem);
    uint32_t* hs = reinterpret_cast<uint32_t*>(smem + kRLastMaxP * 4);
    for (int i = tid; i < kRLastHist; i += NT) hs[i] = 0u;
    const int32_t j0 = tid * kRLastE;
    const int32_t nv = cnt - j0 < 0 ? 0 : (cnt - j0 > kRLastE ? kRLastE : cnt - j0);
    const uint64_t vm = nv >= 64 ? ~0ull : ((1ull << nv) - 1ull);   // bit u: slot j0 + u is in the pool
    if ((reinterpret_cast<uintptr_t>(srow) & 15u) == 0 && (a.P & 3) == 0) {
      int4 v[kRLastE / 4];
#pragma unroll
      for (int u = 0; u < kRLastE / 4; ++u)
        v[u] = j0 + 4 * u < a.P ? __ldcg(reinterpret_cast<const int4*>(srow + j0) + u) : make_int4(0, 0, 0, 0);
#pragma unroll
      for (int u = 0; u < kRLastE / 4; ++u) {
        sc_s[(4 * u + 0) * NT + tid] = v[u].x;
        sc_s[(4 * u + 1) * NT + tid] = v[u].y;
        sc_s[(4 * u + 2) * NT + tid] = v[u].z;
        sc_s[(4 * u + 3) * NT + tid] = v[u].w;
      }
    } else {
      for (int u = 0; u < kRLastE; ++u) sc_s[u * NT + tid] = j0 + u < a.P ? __ldcg(srow + j0 + u) : 0;
    }
    __syncthreads();
#pragma unroll 4
    for (int u = 0; u < kRLastE; ++u) {
      if ((vm >> u) & 1ull) {
        const uint32_t b = score_bucket(sc_s[u * NT + tid]);
        atomicAdd(&hs[b + (b >> 5)], 1u);
      }
    }
    __syncthreads();

    // threshold bucket b*: the bucket holding the K-th best score
    static_assert(kBuckets == 32 * NT, "32 bins per thread");
    const uint32_t* hb = hs + tid * 33;
    uint32_t hsum = 0;
#pragma unroll 8
    for (int b = 0; b < 32; ++b) hsum += hb[b];
    uint64_t total64;
    const uint64_t hex = sel_scan<NT>(hsum, wtmp, &total64);
    const int64_t total = (int64_t)total64;
    const int64_t above_me = total - (int64_t)hex - hsum;
    const int32_t K = a.K;
    if (total > K && above_me < K && above_me + hsum >= K) {
      int64_t acc = above_me;
      for (int b = 31; b >= 0; --b) {
        if (acc + hb[b] >= K) {
          bstar_s = tid * 32 + b;
          above_s = (int32_t)acc;
          break;
        }
        acc += hb[b];
      }
    }
    __syncthreads();
    CSA2_MARK(kTrReindex, 6, tid == 0);
    const int32_t bstar = bstar_s;   // -1: every slot of the pool is a member

    // classify; the ties at b* go to one list in shared memory (over the histogram)
    uint64_t above_m = 0ull, tie_m = 0ull;
    uint64_t* tl = reinterpret_cast<uint64_t*>(hs);
#pragma unroll 4
    for (int u = 0; u < kRLastE; ++u) {
      if ((vm >> u) & 1ull) {
        const int32_t sc = sc_s[u * NT + tid];
        const int32_t bk = (int32_t)score_bucket(sc);
        if (bk > bstar) {
          above_m |= 1ull << u;
        } else if (bk == bstar) {
          tie_m |= 1ull << u;
          const uint32_t t = atomicAdd(&own_cnt, 1u);
          if (t < (uint32_t)kRTieCap) tl[t] = cand_key(sc, j0 + u);
        }
      }
    }
    __syncthreads();
    if (bstar >= 0) {
      const uint32_t nt = own_cnt;
      const int32_t need = K - above_s;
      if (nt <= (uint32_t)kRTieCap) {   // a tie is in when fewer than `need` ties beat it
        for (uint32_t i = warp; i < nt; i += NT / 32) {
          const uint64_t ki = tl[i];
          uint32_t r = 0;
          for (uint32_t j = lane; j < nt; j += 32) r += tl[j] > ki;
#pragma unroll
          for (int o = 16; o > 0; o >>= 1) r += __shfl_xor_sync(0xffffffffu, r, o);
          if (lane == 0 && (int32_t)r < need) atomicMin(&kthr_s, (unsigned long long)ki);
        }
      } else {   // a flat distribution: the need-th key among every tie of the pool
        static_assert(sizeof(ListKthSmem) <= (size_t)kRLastHist * 4, "the select's scratch fits the histogram");
        const uint64_t k0 = tl[0];
        ListKthSmem& lk = *reinterpret_cast<ListKthSmem*>(hs);   // over the tie list: k0 is read first
        const uint64_t kth = block_kth<NT>(
            (uint32_t)cnt, need,
            [&](uint32_t i) -> uint64_t {
              const int32_t v = sc_s[(i % kRLastE) * NT + i / kRLastE];
              return (int32_t)score_bucket(v) == bstar ? cand_key(v, (int32_t)i) : 0ull;
            },
            k0, wtmp, lk);
        if (tid == 0) kthr_s = kth;
      }
      __syncthreads();
    }
    CSA2_MARK(kTrReindex, 8, tid == 0);
    uint64_t mem = above_m;
    if (tie_m) {
      const uint64_t kthr = kthr_s;
      for (int u = 0; u < kRLastE; ++u)
        if (((tie_m >> u) & 1ull) && cand_key(sc_s[u * NT + tid], j0 + u) >= kthr) mem |= 1ull << u;
    }

    // the members' slots in pool order (= position order), then their positions
    uint64_t grand;
    int64_t k = (int64_t)sel_scan<NT>((uint64_t)__popcll(mem), wtmp, &grand);   // ends with a barrier:
    int32_t* out_s = sc_s;                                                      // the scores are done
    for (uint64_t m = mem; m; m &= m - 1ull) {
      if (k < K) out_s[k] = j0 + __ffsll((long long)m) - 1;
      ++k;
    }
    __syncthreads();
    const int32_t n_out = grand < (uint64_t)K ? (int32_t)grand : K;
    int32_t* dst = J.sel_idx + (int64_t)q * K;
#pragma unroll 4
    for (int32_t i = tid; i < K; i += NT) dst[i] = i < n_out ? __ldg(pidx + out_s[i]) : -1;
    if (tid == 0) {
      if (J.sel_cnt) J.sel_cnt[q] = n_out;
      hdr[0] = 0u;   // every CTA has arrived: the count is ready for the next launch
    }
    CSA2_MARK(kTrReindex, 10, tid == 0);
    return;
  }
  if (J.scores && valid) J.scores[(int64_t)q * a.P + slot] = s;

  // ---- the pool's bucket histogram, then the threshold bucket.  The CTA
  // counts its scores in shared memory first (the tiles are free now) and
  // adds each populated bucket to the global histogram once: global atomics
  // on one address serialise, so one add per (CTA, bucket) instead of one per
  // score shortens this phase.
  uint32_t* hist = a.hist + (size_t)prob * kBuckets;
  uint32_t* hdr = a.hdr + (size_t)prob * 4;
  const int32_t bk = (int32_t)score_bucket(s);
  {
    static_assert(kBuckets * 4 <= Lay::region, "the shared histogram fits in the tile region");
    uint32_t* hs = reinterpret_cast<uint32_t*>(smem);
    for (int i = tid; i < kBuckets; i += NT) hs[i] = 0u;
    __syncthreads();
    if (valid) atomicAdd(&hs[bk], 1u);
    __syncthreads();
    // one 64-bit add per populated pair of buckets (no carry: counts stay far below 2^32)
    for (int i = tid; i < kBuckets / 2; i += NT) {
      const uint2 v = reinterpret_cast<const uint2*>(hs)[i];
      if (v.x | v.y)
        atomicAdd(reinterpret_cast<unsigned long long*>(hist) + i,
                  (unsigned long long)v.x | ((unsigned long long)v.y << 32));
    }
  }
  uint32_t phase = 0;
  sel_grid_sync(&hdr[0], ++phase * G, a.status);
  CSA2_MARK(kTrReindex, 5, tid == 0);
  constexpr int kBins = kBuckets / NT;   // bins per thread
  uint4 hv[kBins / 4];
  const uint4* hp = reinterpret_cast<const uint4*>(hist + tid * kBins);
#pragma unroll
  for (int u = 0; u < kBins / 4; ++u) hv[u] = __ldcg(hp + u);
  uint32_t hsum = 0;
#pragma unroll
  for (int u = 0; u < kBins / 4; ++u) hsum += hv[u].x + hv[u].y + hv[u].z + hv[u].w;
  uint64_t total64;
  const uint64_t hex = sel_scan<NT>(hsum, wtmp, &total64);
  const int64_t total = (int64_t)total64;
  const int64_t above_me = total - (int64_t)hex - hsum;
  const int32_t K = a.K;
  if (total > K && above_me < K && above_me + hsum >= K) {
    int64_t acc = above_me;
    bool found = false;
#pragma unroll
    for (int u = kBins / 4 - 1; u >= 0; --u) {
      const uint32_t v4[4] = {hv[u].x, hv[u].y, hv[u].z, hv[u].w};
#pragma unroll
      for (int e = 3; e >= 0; --e) {
        if (!found && acc + v4[e] >= K) {
          bstar_s = tid * kBins + 4 * u + e;
          above_s = (int32_t)acc;
          found = true;
        }
        if (!found) acc += v4[e];
      }
    }
  }
  __syncthreads();
  CSA2_MARK(kTrReindex, 6, tid == 0);
  const int32_t bstar = bstar_s;   // -1: every valid entry is a member

  // ---- ties at b*: ranked against the pool's tie list
  const uint64_t key = cand_key(s, slot);
  const bool above = valid && bk > bstar;
  const bool tie = valid && bk == bstar;
  if (bstar >= 0) {
    if (tie) {
      own[atomicAdd(&own_cnt, 1u)] = key;
      const uint32_t g = atomicAdd(&hdr[1], 1u);
      if (g < (uint32_t)kRTieCap) a.ties[(size_t)prob * kRTieCap + g] = key;
    }
    sel_grid_sync(&hdr[0], ++phase * G, a.status);
    CSA2_MARK(kTrReindex, 7, tid == 0);
    const uint32_t nt = __ldcg(&hdr[1]);
    const int32_t need = K - above_s;
    if (nt <= (uint32_t)kRTieCap) {
      const uint64_t* src = a.ties + (size_t)prob * kRTieCap;
      for (uint32_t i = tid; i < nt; i += NT) rowties[i] = __ldcg(src + i);
      __syncthreads();
      for (uint32_t i = warp; i < own_cnt; i += NT / 32) {
        const uint64_t ki = own[i];
        uint32_t r = 0;
#pragma unroll 4
        for (uint32_t j = lane; j < nt; j += 32) r += rowties[j] > ki;
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) r += __shfl_xor_sync(0xffffffffu, r, o);
        if (lane == 0 && (int32_t)r < need) atomicMin(&kthr_s, (unsigned long long)ki);
      }
    } else {
      const int32_t sv[1] = {s};
      const uint64_t kth = radix_kth<NT, 1>(sv, tie ? 1u : 0u, slot, need, G, x,
                                             a.radix + (size_t)prob * 8 * 256, &hdr[0], phase, a.status, rsm);
      if (tid == 0) kthr_s = kth;
    }
    __syncthreads();
    CSA2_MARK(kTrReindex, 8, tid == 0);
  }
  const bool member = above || (tie && key >= kthr_s);

  // ---- slots: within the CTA by ballot, across CTAs from the published counts
  const uint32_t bal = __ballot_sync(0xffffffffu, member);
  if (lane == 0) wcnt[warp] = __popc(bal);
  __syncthreads();
  uint32_t before = __popc(bal & ((1u << lane) - 1u)), cta_cnt = 0;
#pragma unroll
  for (int w = 0; w < NT / 32; ++w) {
    before += w < warp ? wcnt[w] : 0u;
    cta_cnt += wcnt[w];
  }
  uint32_t* mc = a.mcnt + (size_t)prob * G;
  if (tid == 0) mc[x] = cta_cnt;
  sel_grid_sync(&hdr[0], ++phase * G, a.status);
  CSA2_MARK(kTrReindex, 9, tid == 0);
  uint64_t part = 0ull;   // (members of the CTAs before) | (all members) << 32
  for (int r = tid; r < G; r += NT) {
    const uint64_t v = __ldcg(mc + r);
    part += (r < x ? v : 0ull) | (v << 32);
  }
  uint64_t sums;
  sel_scan<NT>(part, wtmp, &sums);
  const int64_t off = (int64_t)(sums & 0xffffffffu), grand = (int64_t)(sums >> 32);
  int32_t* dst = J.sel_idx + (int64_t)q * K;
  if (member && off + before < K) dst[off + before] = pos;
  if (x == G - 1) {
    const int32_t n_out = grand < K ? (int32_t)grand : K;
    for (int32_t i = n_out + tid; i < K; i += NT) dst[i] = -1;
    if (tid == 0 && J.sel_cnt) J.sel_cnt[q] = n_out;
  }
  CSA2_MARK(kTrReindex, 10, tid == 0);
}

template <int D, int N, int T, bool LAST>
cudaError_t launch_rs_t(const RSelArgs& a_in, int n_jobs, int nq, size_t zero_bytes, cudaStream_t st) {
  using Lay = RSelLayout<D, N, T, LAST>;
  constexpr size_t smem = Lay::smem;
  static SetupMask done{0};
  static std::atomic<int> max_ctas[64];   // co-resident CTAs per device (0: not yet known)
  cudaError_t e = ensure_smem(reindex_select_kernel<D, N, T, LAST>, (int)smem, done);
  if (e != cudaSuccess) return e;
  RSelArgs a = a_in;
  a.G = (a.P + Lay::NT - 1) / Lay::NT;
  if constexpr (!LAST) {   // the CTAs of a pool meet at grid barriers: all must be resident
    int dev = 0;
    e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev >= 64) return cudaErrorNotSupported;
    if (!max_ctas[dev]) {
      int per_sm = 0;
      e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, reindex_select_kernel<D, N, T, LAST>, Lay::NT,
                                                        smem);
      if (e != cudaSuccess) return e;
      max_ctas[dev] = per_sm * sm_count();
    }
    if ((int64_t)a.G * nq * n_jobs > max_ctas[dev]) return cudaErrorNotSupported;
  }
  if (!launch_opts().prezeroed) {
    e = cudaMemsetAsync(a.hist, 0, zero_bytes, st);   // histograms and barrier headers
    if (e != cudaSuccess) return e;
  }
  return launch_k(reindex_select_kernel<D, N, T, LAST>, dim3(a.G, nq, n_jobs), dim3(Lay::NT), smem, st, false,
                  launch_opts().pdl, a);
}

// Co-resident CTAs of two tiles each when they fit the device.  Otherwise
// (a batch of many pools) the last-CTA select for pools of up to kRLastMaxP
// slots, else co-resident CTAs of four tiles.  The grid-barrier path is the
// faster one when it fits: its selection work is spread over every CTA of
// the pool, while the last CTA's runs on one SM.
template <int D, int N>
cudaError_t launch_rs(const RSelArgs& a, int n_jobs, int nq, size_t zero_bytes, cudaStream_t st) {
  cudaError_t e = launch_rs_t<D, N, 2, false>(a, n_jobs, nq, zero_bytes, st);
  if (e != cudaErrorNotSupported) return e;
  if (a.P <= kRLastMaxP && a.K <= kRLastMaxP) return launch_rs_t<D, N, 2, true>(a, n_jobs, nq, zero_bytes, st);
  return launch_rs_t<D, N, 4, false>(a, n_jobs, nq, zero_bytes, st);
}

}  // namespace

cudaError_t launch_reindex_score(const int8_t* q, const int8_t* w, const csa2_rows& keys,
                                 const int32_t* seq_of_query, const int32_t* pool_idx,
                                 const int32_t* pool_cnt, int32_t nq, int32_t H, int32_t D,
                                 int32_t P, int32_t* scores, int32_t* status, cudaStream_t st) {
  ReindexArgs a{q, w, seq_of_query, pool_idx, pool_cnt, static_cast<const uint8_t*>(keys.base),
                keys.row_bytes, to_rowmap(keys), H, P, scores, status};
  const int N = H <= 16 ? 16 : H <= 32 ? 32 : H <= 64 ? 64 : 128;
  if (D == 128) {
    switch (N) {
      case 16: return launch_r<128, 16>(a, nq, st);
      case 32: return launch_r<128, 32>(a, nq, st);
      case 64: return launch_r<128, 64>(a, nq, st);
      default: return launch_r<128, 128>(a, nq, st);
    }
  }
  switch (N) {
    case 16: return launch_r<64, 16>(a, nq, st);
    case 32: return launch_r<64, 32>(a, nq, st);
    case 64: return launch_r<64, 64>(a, nq, st);
    default: return launch_r<64, 128>(a, nq, st);
  }
}

size_t reindex_select_scratch_bytes(int32_t n_probs, int32_t P) {
  Carver c(nullptr);
  ReindexSelScratch r = carve_reindex_select(c, n_probs, P);
  (void)r;
  return c.used + 256;
}

ReindexSelScratch carve_reindex_select(Carver& c, int32_t n_probs, int32_t P) {
  const int32_t G = (P + 255) / 256;   // CTAs per pool: at least 256 slots each
  ReindexSelScratch r;
  r.n_probs = n_probs;
  r.hist = c.take<uint32_t>((size_t)n_probs * kBuckets);
  r.hdr = c.take<uint32_t>((size_t)n_probs * 4);   // directly after hist: one memset zeroes both
  r.ties = c.take<uint64_t>((size_t)n_probs * kRTieCap);
  r.mcnt = c.take<uint32_t>((size_t)n_probs * G);
  r.radix = c.take<uint32_t>((size_t)n_probs * 8 * 256);
  r.sc = c.take<int32_t>((size_t)n_probs * P);
  return r;
}

cudaError_t launch_reindex_select(const ReindexJobDesc* jobs, int32_t n_jobs, const int32_t* seq_of_query,
                                  const int32_t* pool_idx, const int32_t* pool_cnt, int32_t nq, int32_t H,
                                  int32_t D, int32_t P, int32_t K, const ReindexSelScratch& r,
                                  int32_t* status, cudaStream_t st) {
  if (n_jobs < 1 || n_jobs > kMaxReindexJobs || r.n_probs < n_jobs * nq) return cudaErrorInvalidValue;
  RSelArgs a{};
  for (int j = 0; j < n_jobs; ++j) {
    const ReindexJobDesc& d = jobs[j];
    a.job[j] = RSelJob{d.q, d.w, static_cast<const uint8_t*>(d.keys->base), d.keys->row_bytes, to_rowmap(*d.keys),
                       d.scores, d.sel_idx, d.sel_cnt};
  }
  a.seq_of_query = seq_of_query;
  a.pool_idx = pool_idx;
  a.pool_cnt = pool_cnt;
  a.H = H;
  a.P = P;
  a.K = K;
  a.nq = nq;
  a.hist = r.hist;
  a.hdr = r.hdr;
  a.ties = r.ties;
  a.mcnt = r.mcnt;
  a.radix = r.radix;
  a.sc = r.sc;
  a.status = status;
  const int N = H <= 16 ? 16 : H <= 32 ? 32 : H <= 64 ? 64 : 128;
  if (N == 128) return cudaErrorNotSupported;
  const size_t zb = (size_t)n_jobs * nq * (kBuckets + 4) * sizeof(uint32_t);
  if (D == 128) {
    switch (N) {
      case 16: return launch_rs<128, 16>(a, n_jobs, nq, zb, st);
      case 32: return launch_rs<128, 32>(a, n_jobs, nq, zb, st);
      default: return launch_rs<128, 64>(a, n_jobs, nq, zb, st);
    }
  }
  switch (N) {
    case 16: return launch_rs<64, 16>(a, n_jobs, nq, zb, st);
    case 32: return launch_rs<64, 32>(a, n_jobs, nq, zb, st);
    default: return launch_rs<64, 64>(a, n_jobs, nq, zb, st);
  }
}

}  // namespace csa2
