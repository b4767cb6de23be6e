// K1: the full-mode indexer score stream on the 5th-generation tensor cores.
//
// score[s] = sum_h w[h] * max(0, q[h] . key[s]) for every position s <= pos of
// every query ("the first full-mode indexing layer searches the large
// context": "DeepSeek V4.1-Flash: 552B runs like 16B", Act 2).
//
// Design (one persistent CTA per SM, 10 warps):
//   warp 0     TMA producer: streams 128-row key tiles (two 64-row boxes, so
//              64-row pages work unchanged) into an NST-deep ring with evict-
//              first L2 hints.  The key rows are the only O(context) bytes of
//              a decode step; everything else is sized by the pool.
//   warp 1     tcgen05 issuer: D[128 keys x N heads] = keys (K-major, swizzled)
//              x q^T, int8 x int8 -> int32 in TMEM, double-buffered so the
//              epilogue of tile i overlaps the MMA of tile i+1.
//   warps 2-9  epilogue, two groups of four warps on alternate tiles: each
//              thread owns one key row (one TMEM lane), loads its N int32
//              head dots, applies ReLU and the integer head weights in
//              registers, stores the int32 score (coalesced) and adds the
//              score's bucket to a shared-memory radix histogram that is
//              flushed once per query segment (the first pass of the top-k).
// Work is the flat list of (query, 128-row tile) items over all queries,
// split evenly between CTAs, so ragged batches stay balanced.
#include "csa2_device.cuh"
#include "internal.h"

namespace csa2 {

CSA2_TRACE_UNIT(index)

namespace {

struct IndexArgs {
  const int8_t* q;
  const int8_t* w;
  const int32_t* seq_of_query;
  const int32_t* query_pos;
  RowMap rows;
  int32_t nq, H, max_ctx;
  int32_t* scores;
  int64_t ld;
  uint32_t* hist;
  int32_t* status;
};

constexpr int kMaxQueries = 4096;   // per launch (the work list prefix lives in shared memory)
constexpr int kGroupMinQueries = 16;   // from this many queries on, queries of a sequence share key tiles

template <int D>
struct IndexCfg {
  static constexpr int kTile = 128 * D;                       // bytes of one key tile
  static constexpr int kStages = (D == 128) ? 8 : 12;         // >= 96 KiB in flight per SM
};

// Epilogue warps.  One query per segment: 8, two groups of four (one warp per
// TMEM lane quarter) on alternate tiles.  Queries sharing tiles: 16, four per
// lane quarter, warp group m reading query m of every tile, so that four
// warps per scheduler hide the TMEM and arithmetic latencies.
template <int QG>
constexpr int epi_warps() { return QG == 1 ? 8 : 16; }
template <int QG>
__device__ __forceinline__ void named_sync_epi() {
  asm volatile("bar.sync 1, %0;" ::"n"(32 * epi_warps<QG>()) : "memory");
}

__device__ __forceinline__ bool mbar_wait_drain(uint64_t* bar, uint32_t parity) {
  const uint64_t t0 = global_ns();
  while (!mbar_try_wait(bar, parity)) {
    if (global_ns() - t0 > 100000000ull) return false;   // 100 ms
  }
  return true;
}

// QG queries of one sequence share each key tile (QG = 1 for decode; 4 for a
// prefill chunk, where consecutive queries of a sequence form the groups).
template <int D, int N, int QG>
__global__ void __launch_bounds__(64 + 32 * epi_warps<QG>(), 1)
index_score_kernel(const __grid_constant__ CUtensorMap kmap, const IndexArgs a) {
  constexpr int kEpiThreads = 32 * epi_warps<QG>();
  using Cfg = IndexCfg<D>;
  constexpr int NST = Cfg::kStages;
  constexpr int TILE = Cfg::kTile;
  constexpr int NG = N * QG;            // MMA N: the heads of every query of a group
  static_assert(NG <= 256, "one MMA covers the group");
  static_assert(QG == 1 || QG == epi_warps<QG>() / 4, "grouped epilogue: one warp group of four per query of the group");
  // As many TMEM accumulator buffers as fit in the 512 columns (at most 8),
  // so the MMA can run up to NBUF tiles ahead of the epilogue.
  constexpr int NBUF = (512 / NG) < 8 ? (512 / NG) : 8;
  constexpr uint32_t TMEM_COLS = NBUF * NG <= 32 ? 32 : NBUF * NG <= 64 ? 64 : NBUF * NG <= 128 ? 128 : NBUF * NG <= 256 ? 256 : 512;
  constexpr int kHist = QG == 1 ? kBuckets : 0;   // grouped launches leave the histogram to the top-k

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* stages = smem;
  uint8_t* bmat = stages + NST * TILE;
  uint32_t* hist_s = reinterpret_cast<uint32_t*>(bmat + NG * D);
  int32_t* w_s = reinterpret_cast<int32_t*>(hist_s + kHist);     // [NG] (at least 128)
  int32_t* prefix = w_s + (NG > 128 ? NG : 128);                 // [groups + 1] tiles before each group
  int32_t* gq = prefix + ((a.nq + 2) & ~1);                      // [groups + 1] first query of each group
  int32_t* gseq = gq + ((a.nq + 2) & ~1);                        // [groups] sequence of each group
  // bit g: the second 64-row box of group g's last tile is visible (its last
  // position mod 128 is at least 64); with the tile count this is all the
  // producer needs to know of the positions
  uint32_t* ghalf = reinterpret_cast<uint32_t*>(gseq + ((a.nq + 2) & ~1));
  uint64_t* bars = reinterpret_cast<uint64_t*>(ghalf + ((a.nq + 63) / 64) * 2);
  uint64_t* full = bars;
  uint64_t* empty = bars + NST;
  uint64_t* tfull = bars + 2 * NST;
  uint64_t* tempty = tfull + NBUF;
  uint64_t* bready = tempty + NBUF;                              // the segment's B operand is in place
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bready + 2);
  volatile int32_t* abort_flag = reinterpret_cast<volatile int32_t*>(tmem_slot + 1);
  int32_t* ngroups_s = const_cast<int32_t*>(abort_flag) + 1;
  unsigned long long* bound_acc = reinterpret_cast<unsigned long long*>(tmem_slot + 4);   // [QG]
  int32_t* mpos = reinterpret_cast<int32_t*>(bound_acc + QG);                         // [QG] member positions

  const int tid = threadIdx.x;
  const int warp = tid >> 5;
  const int lane = tid & 31;
  // trace points: 1 prologue done, 2 first TMA issued, 3 first stage landed,
  // 4 first epilogue tile done, 5 last epilogue tile done, 6 histogram
  // flushed, 7 producer done, 8 MMA issuer done, 9 exit, 10 producer at its
  // first ring slot (segment set up)
  CSA2_TRACE_BEGIN(kTrIndex, tid == 0);
  if (tid == 0) prefetch_tensormap(&kmap);   // the descriptor's fetch overlaps the prologue

  // ---- prologue: warp 0 builds the work list (groups of queries, their
  // sequences and the tiles before each group), warp 1 allocates TMEM, thread 0 sets up the
  // barriers; one block barrier later the producer streams.  The epilogue
  // warps zero their histogram behind a barrier of their own.
  if (tid == 0) {
    for (int i = 0; i < NST; ++i) {
      mbar_init(&full[i], 1);
      mbar_init(&empty[i], 1);
    }
    for (int i = 0; i < NBUF; ++i) {
      mbar_init(&tfull[i], 1);
      // one arrival per warp that reads the buffer: a group of four, or every epilogue warp
      mbar_init(&tempty[i], QG == 1 ? 4 : epi_warps<QG>());
    }
    mbar_init(bready, kEpiThreads / 32);
    for (int k = 0; k < QG; ++k) bound_acc[k] = 0ull;
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, TMEM_COLS);
    tmem_relinquish();
  }
  if (warp == 0) {
    // groups: runs of consecutive queries of one sequence, cut every QG
    int32_t n_groups = 0;
    if constexpr (QG == 1) {
      for (int i = lane; i <= a.nq; i += 32) gq[i] = i;
      n_groups = a.nq;
      __syncwarp();
    } else {
      int32_t last_start = 0;
      for (int base = 0; base < a.nq; base += 32) {
        const int i = base + lane;
        const bool valid = i < a.nq;
        bool s = false;
        if (valid) {
          const int32_t sq = a.seq_of_query ? __ldg(a.seq_of_query + i) : i;
          const int32_t sp = i == 0 ? -1 : (a.seq_of_query ? __ldg(a.seq_of_query + i - 1) : i - 1);
          s = i == 0 || sq != sp;
        }
        int32_t v = s ? i : -1;   // latest run start at or before i
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
          const int32_t n = __shfl_up_sync(0xffffffffu, v, o);
          if (lane >= o) v = v > n ? v : n;
        }
        v = v > last_start ? v : last_start;
        const bool f = valid && (s || (i - v) % QG == 0);
        const uint32_t bal = __ballot_sync(0xffffffffu, f);
        if (f) gq[n_groups + __popc(bal & ((1u << lane) - 1u))] = i;
        n_groups += __popc(bal);
        last_start = __shfl_sync(0xffffffffu, v, 31);
      }
      if (lane == 0) gq[n_groups] = a.nq;
      __syncwarp();
    }
    // prefix[g+1] = work units up to group g (a group's tiles cover the
    // longest causal prefix of its queries; one unit per tile, or 3 + its
    // queries per tile in a grouped launch)
    int32_t carry = 0;
    if (lane == 0) {
      prefix[0] = 0;
      *ngroups_s = n_groups;
    }
    for (int base = 0; base < n_groups; base += 32) {
      const int g = base + lane;
      int32_t v = 0, last = -1;   // tiles and last visible position of the group
      if (g < n_groups) {
        gseq[g] = a.seq_of_query ? __ldg(a.seq_of_query + gq[g]) : gq[g];   // in flight with the positions
        for (int i = gq[g]; i < gq[g + 1]; ++i) {
          const int32_t pos = __ldg(a.query_pos + i);
          if (pos < 0 || pos >= a.max_ctx) record_error(a.status, CSA2_ERR_INDEX_RANGE);
          else if (pos > last) last = pos;
        }
        v = (last + 128) / 128;
        // grouped launches divide work units, not tiles, among the CTAs: a
        // tile costs about 3 + (its group's queries) units (the epilogue's
        // share grows with the queries, the stream's does not)
        if constexpr (QG != 1) v *= 3 + (gq[g + 1] - gq[g]);
      }
      const uint32_t half = __ballot_sync(0xffffffffu, last >= 0 && (last & 127) >= 64);
      if (lane == 0) ghalf[base >> 5] = half;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int32_t n = __shfl_up_sync(0xffffffffu, v, o);
        if (lane >= o) v += n;
      }
      if (g < n_groups) prefix[g + 1] = v + carry;
      carry += __shfl_sync(0xffffffffu, v, 31);
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  const int ngroups = *ngroups_s;
  CSA2_MARK(kTrIndex, 1, tid == 0);
  pdl_trigger();   // the next grid may be launched (it waits for this one to finish)
  if (warp >= 2) {   // the epilogue's histogram, zeroed before its first use
    for (int i = tid - 64; i < kHist; i += kEpiThreads) hist_s[i] = 0;
    named_sync_epi<QG>();
  }

  const int64_t total = prefix[ngroups];
  const int64_t lo = total * blockIdx.x / gridDim.x;
  const int64_t hi = total * (blockIdx.x + 1) / gridDim.x;
  int g0 = 0;
  {
    int l = 0, r = ngroups > 0 ? ngroups - 1 : 0;   // last group with prefix[g] <= lo
    while (l < r) {
      const int m = (l + r + 1) >> 1;
      if (prefix[m] <= lo) l = m; else r = m - 1;
    }
    g0 = l;
  }

  // The CTA's items are processed one group segment at a time.  Within a
  // segment the producer, the MMA issuer and the epilogue run as a pipeline.
  // Between segments the whole CTA synchronises, so the B operand (the
  // queries) and the histogram can be swapped without any hand-off protocol.
  // `git` numbers the items of the CTA and drives every barrier phase.
  const int et = tid - 64;                 // epilogue thread 0..kEpiThreads-1 (negative for warps 0-1)
  const int group = et >> 7;               // warp group of four: tiles i % 2 (QG 1) or query `group` (QG 4)
  const int quarter = warp & 3;            // TMEM lanes this warp may access
  const int row = quarter * 32 + lane;     // key row of the tile this thread owns
  int64_t git = 0;
  int seg_count = 0;   // segments done by this CTA (bready phase)
  int g = g0;
  for (int64_t s_lo = lo; s_lo < hi;) {
    while (s_lo >= prefix[g + 1]) ++g;
    const int64_t s_hi = hi < (int64_t)prefix[g + 1] ? hi : (int64_t)prefix[g + 1];
    const int q0 = gq[g], nm = gq[g + 1] - gq[g];   // the group's queries
    // the tiles of group g whose first work unit lies in [s_lo, s_hi)
    const int32_t wu = QG == 1 ? 1 : 3 + nm;
    const int32_t tile0 = (int32_t)((s_lo - prefix[g] + wu - 1) / wu);
    const int n_it = (int)((s_hi - prefix[g] + wu - 1) / wu) - tile0;
    if (n_it <= 0) {   // (every thread agrees) no tile starts in this range
      s_lo = s_hi;
      continue;
    }
    // box j of tile t is visible unless it is the second box of the group's
    // last tile and that tile's visible rows end before it
    const int32_t t_last = (prefix[g + 1] - prefix[g]) / wu - 1;
    const bool half = (ghalf[g >> 5] >> (g & 31)) & 1u;

    // ---- segment set-up (epilogue threads): B operand = the group's q rows
    // (query k at rows k N .. k N + H - 1, zero rows elsewhere), K-major with
    // the tile swizzle, and the head weights.  The producer does not wait for
    // it (key tiles do not depend on the queries); the MMA issuer waits on
    // `bready`.  The int32 overflow guard 128 * sum_h |w_h| * sum_d |q_hd| <
    // 2^31 is checked per query off the critical path.
    if (warp >= 2) {
      for (int idx = et; idx < NG * (D / 16); idx += kEpiThreads) {
        const int r = idx / (D / 16), c = idx % (D / 16);
        const int k = r / N, h = r % N;
        int4 v = make_int4(0, 0, 0, 0);
        if (k < nm && h < a.H) v = __ldg(reinterpret_cast<const int4*>(a.q + ((int64_t)(q0 + k) * a.H + h) * D) + c);
        *reinterpret_cast<int4*>(bmat + swizzled_chunk(r, c, D)) = v;
      }
      for (int r = et; r < NG; r += kEpiThreads) {
        const int k = r / N, h = r % N;
        w_s[r] = (k < nm && h < a.H) ? (int32_t)__ldg(a.w + (int64_t)(q0 + k) * a.H + h) : 0;
      }
      if (et < QG) mpos[et] = et < nm ? __ldg(a.query_pos + q0 + et) : -1;
      fence_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive(bready);
      named_sync_epi<QG>();
      for (int r = et; r < nm * a.H; r += kEpiThreads) {
        const int k = r / a.H, h = r % a.H;
        int32_t sq = 0;
        const int4* src = reinterpret_cast<const int4*>(a.q + ((int64_t)(q0 + k) * a.H + h) * D);
        for (int c = 0; c < D / 16; ++c) {
          const int4 v = __ldg(src + c);
          const int32_t wv[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
          for (int j = 0; j < 4; ++j)
#pragma unroll
            for (int b2 = 0; b2 < 4; ++b2) sq += abs((int32_t)(int8_t)(wv[j] >> (8 * b2)));
        }
        const unsigned long long t = (unsigned long long)sq * (unsigned long long)abs(w_s[k * N + h]);
        if (t) atomicAdd(&bound_acc[k], t);
      }
    }

    if (warp == 0) {
      // ---------------------------------------------------------- producer
      // Lane 0 issues the loads.  With a paged view the whole warp reads the
      // page-table entries one chunk of 16 tiles ahead (lane l: box l & 1 of
      // tile l >> 1 of the chunk), so no load waits on a table lookup.
      CSA2_MARK(kTrIndex, 10, tid == 0 && git == 0);
      const uint64_t pol = l2_policy_evict_first();
      const int32_t seq = gseq[g];
      const RowMap& m = a.rows;
      auto page_entry = [&](int i0) -> int32_t {   // raw entry behind this lane's box of the chunk at i0
        const int i = i0 + (lane >> 1);
        const int32_t p0 = (tile0 + i) * 128 + 64 * (lane & 1);
        if (i >= n_it || ((lane & 1) && tile0 + i == t_last && !half)) return -1;
        const int32_t pg = p0 / m.page_rows;
        return pg < m.max_pages ? __ldg(m.page_table + (int64_t)seq * m.max_pages + pg) : -1;
      };
      int32_t ent = -1, ent_next = -1;
      if (m.page_table) {
        ent = page_entry(0);
        ent_next = page_entry(16);
      }
      int i = 0;
      for (; i < n_it; ++i) {
        if (m.page_table && i > 0 && i % 16 == 0) {
          ent = ent_next;
          ent_next = page_entry(i + 16);
        }
        const int32_t tile = tile0 + i;
        int64_t r[2];
#pragma unroll
        for (int j = 0; j < 2; ++j) {
          const int32_t p0 = tile * 128 + 64 * j;
          if (m.page_table) {
            const int32_t e = __shfl_sync(0xffffffffu, ent, 2 * (i % 16) + j);
            const int64_t row = (int64_t)e * m.page_rows + (p0 % m.page_rows);
            r[j] = (e >= 0 && row < m.n_rows) ? row : -1;
          } else {
            r[j] = map_row(m, seq, p0);
          }
          if (j == 1 && tile == t_last && !half) r[j] = -2;   // past the last visible position: no box
        }
        bool ok = true;
        if (lane == 0) {
          const int64_t gi = git + i;
          const int st = (int)(gi % NST);
          const uint32_t ph = (uint32_t)((gi / NST) & 1);
          ok = mbar_wait(&empty[st], ph ^ 1, abort_flag);
          if (ok) {
            uint32_t bytes = 0;
#pragma unroll
            for (int j = 0; j < 2; ++j) {
              if (r[j] == -1) record_error(a.status, CSA2_ERR_INDEX_RANGE);
              else if (r[j] >= 0) bytes += 64 * D;
            }
            mbar_arrive_expect_tx(&full[st], bytes);
#pragma unroll
            for (int j = 0; j < 2; ++j)
              if (r[j] >= 0)
                tma_load_2d(stages + st * TILE + j * 64 * D, &kmap, 0, (int32_t)r[j], &full[st], pol);
            CSA2_MARK(kTrIndex, 2, gi == 0);
          }
        }
        if (!__shfl_sync(0xffffffffu, ok, 0)) break;
      }
      if (lane == 0) {
        if (*abort_flag) {   // let loads already in flight land before moving on
          const int64_t issued = git + i;
          const int64_t n = i < NST ? i : NST;
          for (int64_t k = issued - n; k < issued; ++k)
            mbar_wait_drain(&full[k % NST], (uint32_t)((k / NST) & 1));
        }
        CSA2_MARK(kTrIndex, 7, true);
      }
    } else if (warp == 1) {
      // ---------------------------------------------------------- MMA issuer
      if (lane == 0) {
        constexpr uint32_t idesc = idesc_i8(128, NG);
        const uint32_t b_addr = smem_u32(bmat);
        const bool bok = mbar_wait(bready, (uint32_t)(seg_count & 1), abort_flag);
        tc_fence_after();
        for (int i = 0; i < n_it && bok; ++i) {
          const int64_t gi = git + i;
          const int st = (int)(gi % NST);
          const uint32_t ph = (uint32_t)((gi / NST) & 1);
          const int buf = (int)(gi % NBUF);
          const uint32_t tph = (uint32_t)((gi / NBUF) & 1);
          if (!mbar_wait(&full[st], ph, abort_flag)) break;
          CSA2_MARK(kTrIndex, 3, gi == 0);
          if (!mbar_wait(&tempty[buf], tph ^ 1, abort_flag)) break;
          tc_fence_after();
          const uint32_t a_addr = smem_u32(stages + st * TILE);
#pragma unroll
          for (int k = 0; k < D / 32; ++k)
            mma_i8(tmem_base + buf * NG, smem_desc_kmajor(a_addr + 32 * k, D),
                   smem_desc_kmajor(b_addr + 32 * k, D), idesc, k > 0 ? 1u : 0u);
          mma_commit(&empty[st]);
          mma_commit(&tfull[buf]);
        }
        CSA2_MARK(kTrIndex, 8, true);
      }
    } else {
      // ---------------------------------------------------------- epilogue
      // Two groups of four warps (one warp per TMEM lane quarter each) take
      // alternate tiles, so the groups never wait for each other within a
      // segment.  A thread owns one key row: for each query of the segment's
      // group it loads the row's N head dots, applies ReLU and the head
      // weights in independent partial sums and stores the score (and, with
      // one query per group, adds its bucket to the shared histogram); then
      // it frees the TMEM buffer.  Every epilogue thread walks the same tiles
      // and reaches the same barriers even after a timeout (it then skips the
      // TMEM reads and the stores).
      if (seg_count == 0) pdl_wait();   // scores and histogram: after the grid before (it zeroes them)
      constexpr bool kRegW = QG == 1 && N <= 64;
      int32_t wreg[kRegW ? N : 1];
      if constexpr (kRegW) {
#pragma unroll
        for (int h = 0; h < N; ++h) wreg[h] = w_s[h];
      }
      // Queries sharing tiles: the head weights of this warp group's query,
      // four int8 per register for the whole segment (re-reading them from
      // shared memory for every tile kept the load pipe the busiest unit).
      constexpr bool kPackW = QG != 1;
      uint32_t wpk[kPackW ? N / 4 : 1];
      if constexpr (kPackW) {
#pragma unroll
        for (int h4 = 0; h4 < N / 4; ++h4) {
          const int4 v = *reinterpret_cast<const int4*>(w_s + group * N + 4 * h4);
          wpk[h4] = (uint32_t)(v.x & 0xFF) | ((uint32_t)(v.y & 0xFF) << 8) | ((uint32_t)(v.z & 0xFF) << 16) |
                    ((uint32_t)v.w << 24);
        }
      }
      for (int i = QG == 1 ? group : 0; i < n_it; i += QG == 1 ? 2 : 1) {
        const int64_t gi = git + i;
        const bool ok = __all_sync(0xffffffffu, mbar_wait(&tfull[gi % NBUF], (uint32_t)((gi / NBUF) & 1), abort_flag));
        const int32_t pos = (tile0 + i) * 128 + row;
        if (ok) tc_fence_after();
        const uint32_t tbase = tmem_base + ((uint32_t)(quarter * 32) << 16) + (uint32_t)((gi % NBUF) * NG);
        if constexpr (QG == 1) {
          uint32_t r[N];
          if (ok) {
            if constexpr (N == 16) {
              tmem_ld16(tbase, r);
            } else {
#pragma unroll
              for (int c = 0; c < N / 32; ++c)
                tmem_ld32(tbase + 32 * c, *reinterpret_cast<uint32_t(*)[32]>(&r[32 * c]));
            }
            tmem_wait_ld();
          }
          tc_fence_before();   // the buffer has been read: free it for the MMA
          __syncwarp();
          if (lane == 0) mbar_arrive(&tempty[gi % NBUF]);
          if (ok) {
            int32_t part[8] = {0, 0, 0, 0, 0, 0, 0, 0};   // independent chains, no long serial sum
#pragma unroll
            for (int h = 0; h < N; ++h) part[h & 7] += (kRegW ? wreg[h] : w_s[h]) * max((int32_t)r[h], 0);
            const int32_t sc = ((part[0] + part[1]) + (part[2] + part[3])) + ((part[4] + part[5]) + (part[6] + part[7]));
            if (pos <= mpos[0]) {
              a.scores[(int64_t)q0 * a.ld + pos] = sc;
              atomicAdd(&hist_s[score_bucket(sc)], 1u);
            }
          }
        } else {
          // Warp group m reads query m of the tile: its N head dots 16 columns
          // at a time (with four partial sums this leaves room for the packed
          // weights in the 96 registers of an 18-warp CTA); every warp frees
          // the buffer once, after its last TMEM read.
          constexpr int CH = 16;
          const int k = group;
          int32_t sc = 0;
          if (ok && k < nm) {
            int32_t part[4] = {0, 0, 0, 0};
#pragma unroll
            for (int c = 0; c < N / CH; ++c) {
              uint32_t rb[CH];
              tmem_ld16(tbase + (uint32_t)(k * N + c * CH), rb);
              tmem_wait_ld();
#pragma unroll
              for (int j = 0; j < CH; ++j) {
                const int h = c * CH + j;
                const int32_t wv = (int32_t)(int8_t)(wpk[h >> 2] >> (8 * (h & 3)));
                part[j & 3] += wv * max((int32_t)rb[j], 0);
              }
            }
            sc = (part[0] + part[1]) + (part[2] + part[3]);
          }
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(&tempty[gi % NBUF]);
          if (ok && k < nm && pos <= mpos[k]) a.scores[(int64_t)(q0 + k) * a.ld + pos] = sc;
        }
        if (QG == 1 && nm == 0) {   // no query (cannot happen for a segment with tiles): still free the buffer
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(&tempty[gi % NBUF]);
        }
        CSA2_MARK(kTrIndex, 4, tid == 64 && gi == 0);
      }
      CSA2_MARK(kTrIndex, 5, tid == 64);
      // this query's histogram goes to global memory
      named_sync_epi<QG>();
      if constexpr (QG == 1) {
        if (a.hist) {
          // Four bins per 16-byte read; each populated pair of bins costs one
          // 64-bit add (a count never reaches 2^32, so the low bin cannot
          // carry into the high one, and the pair is the two 32-bit bins in
          // memory order).  The adds of every CTA meet in a few L2 slices at
          // the end of the launch, and the next grid waits for all of them:
          // their number, not their size, sets that wait.
          unsigned long long* gh = reinterpret_cast<unsigned long long*>(a.hist + (int64_t)q0 * kBuckets);
          for (int b4 = et; b4 < kBuckets / 4; b4 += kEpiThreads) {
            uint4* hp = reinterpret_cast<uint4*>(hist_s) + b4;
            const uint4 v = *hp;
            if (v.x | v.y | v.z | v.w) {
              if (v.x | v.y) atomicAdd(gh + 2 * b4, (unsigned long long)v.x | ((unsigned long long)v.y << 32));
              if (v.z | v.w) atomicAdd(gh + 2 * b4 + 1, (unsigned long long)v.z | ((unsigned long long)v.w << 32));
              *hp = make_uint4(0, 0, 0, 0);
            }
          }
        }
      }
      CSA2_MARK(kTrIndex, 6, tid == 64);
    }
    tc_fence_before();
    __syncthreads();   // the segment is done everywhere: B and the histogram may be reused
    tc_fence_after();
    if (tid == 64) {
      for (int k = 0; k < nm; ++k) {
        if (bound_acc[k] * 128ull >= (1ull << 31)) record_error(a.status, CSA2_ERR_SCORE_RANGE);
        bound_acc[k] = 0ull;
      }
    }
    __syncthreads();
    git += n_it;
    ++seg_count;
    s_lo = s_hi;
  }

  CSA2_MARK(kTrIndex, 9, tid == 0);
  if (warp == 1) tmem_dealloc(tmem_base, TMEM_COLS);
  if (tid == 0 && *abort_flag) record_error(a.status, CSA2_ERR_TIMEOUT);
}

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static std::atomic<EncodeTiledFn> cached{nullptr};   // looked up again until found
  EncodeTiledFn fn = cached.load(std::memory_order_acquire);
  if (!fn) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult qr;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &qr) == cudaSuccess &&
        qr == cudaDriverEntryPointSuccess) {
      fn = reinterpret_cast<EncodeTiledFn>(p);
      cached.store(fn, std::memory_order_release);
    }
  }
  return fn;
}

template <int D>
size_t index_smem_bytes(int N, int QG, int nq) {
  using Cfg = IndexCfg<D>;
  const int NG = N * QG;
  return 1024 + (size_t)Cfg::kStages * Cfg::kTile + (size_t)NG * D + (QG == 1 ? kBuckets * 4 : 0) +
         (size_t)(NG > 128 ? NG : 128) * 4 + 3 * (size_t)((nq + 2) & ~1) * 4 + (size_t)((nq + 63) / 64) * 8 + (2 * Cfg::kStages + 2 * 8) * 8 +
         32 + 8 * (size_t)QG + 4 * (size_t)QG + 16;
}

template <int D, int N, int QG>
cudaError_t launch_one(const CUtensorMap& map, const IndexArgs& a, int grid, cudaStream_t st) {
  const size_t smem = index_smem_bytes<D>(N, QG, a.nq);
  static SetupMask done{0};
  cudaError_t e = ensure_smem(index_score_kernel<D, N, QG>, (int)index_smem_bytes<D>(N, QG, kMaxQueries), done);
  if (e != cudaSuccess) return e;
  return launch_k(index_score_kernel<D, N, QG>, dim3(grid), dim3(64 + 32 * epi_warps<QG>()), smem, st, false,
                  launch_opts().pdl, map, a);
}

}  // namespace

int sm_count() {
  int dev = 0, n = 148;
  if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
  return n;
}

cudaError_t launch_index_score(const int8_t* q, const int8_t* w, const csa2_rows& keys,
                               const int32_t* seq_of_query, const int32_t* query_pos,
                               int32_t nq, int32_t H, int32_t D, int32_t max_ctx,
                               int32_t* scores, int64_t ld, uint32_t* hist, int32_t* status,
                               cudaStream_t st, bool* hist_built) {
  if (nq > kMaxQueries) return cudaErrorInvalidValue;
  EncodeTiledFn enc = encode_fn();
  if (!enc) return cudaErrorNotSupported;
  CUtensorMap map;
  cuuint64_t gdim[2] = {(cuuint64_t)D, (cuuint64_t)keys.n_rows};
  cuuint64_t gstride[1] = {(cuuint64_t)keys.row_bytes};
  cuuint32_t box[2] = {(cuuint32_t)D, 64};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = enc(&map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(keys.base), gdim, gstride,
                   box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                   D == 128 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_64B,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return cudaErrorInvalidValue;

  const int N = H <= 16 ? 16 : H <= 32 ? 32 : H <= 64 ? 64 : 128;
  // Many queries (a prefill chunk) share key tiles in groups of four, with the
  // histogram left to the top-k; decode keeps one query per segment.  A plan
  // call groups only when it says its queries come in same-sequence blocks (a
  // verify block), and then from two queries on; a plan's batch of distinct
  // sequences keeps one query per segment whatever its size.
  const LaunchOpts& lo = launch_opts();
  const bool grouped = N <= 64 && (lo.group ? nq >= 2 : (!lo.plan && nq >= kGroupMinQueries));
  if (hist_built) *hist_built = !grouped && hist;
  IndexArgs a{q, w, seq_of_query, query_pos, to_rowmap(keys), nq, H, max_ctx, scores, ld,
              grouped ? nullptr : hist, status};
  const int64_t upper = (int64_t)nq * ((max_ctx + 127) / 128);
  const int grid = (int)(upper < sm_count() ? (upper > 0 ? upper : 1) : sm_count());
  if (D == 128) {
    switch (N) {
      case 16: return grouped ? launch_one<128, 16, 4>(map, a, grid, st) : launch_one<128, 16, 1>(map, a, grid, st);
      case 32: return grouped ? launch_one<128, 32, 4>(map, a, grid, st) : launch_one<128, 32, 1>(map, a, grid, st);
      case 64: return grouped ? launch_one<128, 64, 4>(map, a, grid, st) : launch_one<128, 64, 1>(map, a, grid, st);
      default: return launch_one<128, 128, 1>(map, a, grid, st);
    }
  }
  switch (N) {
    case 16: return grouped ? launch_one<64, 16, 4>(map, a, grid, st) : launch_one<64, 16, 1>(map, a, grid, st);
    case 32: return grouped ? launch_one<64, 32, 4>(map, a, grid, st) : launch_one<64, 32, 1>(map, a, grid, st);
    case 64: return grouped ? launch_one<64, 64, 4>(map, a, grid, st) : launch_one<64, 64, 1>(map, a, grid, st);
    default: return launch_one<64, 128, 1>(map, a, grid, st);
  }
}

}  // namespace csa2
