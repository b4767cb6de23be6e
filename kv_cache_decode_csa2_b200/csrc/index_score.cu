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

template <int D>
struct IndexCfg {
  static constexpr int kTile = 128 * D;                       // bytes of one key tile
  static constexpr int kStages = (D == 128) ? 8 : 12;         // >= 96 KiB in flight per SM
};

constexpr int kEpiThreads = 256;   // 8 epilogue warps: two groups, one warp per TMEM lane quarter each
__device__ __forceinline__ void named_sync_epi() { asm volatile("bar.sync 1, 256;" ::: "memory"); }

__device__ __forceinline__ bool mbar_wait_drain(uint64_t* bar, uint32_t parity) {
  const uint64_t t0 = global_ns();
  while (!mbar_try_wait(bar, parity)) {
    if (global_ns() - t0 > 100000000ull) return false;   // 100 ms
  }
  return true;
}

template <int D, int N>
__global__ void __launch_bounds__(64 + kEpiThreads, 1)
index_score_kernel(const __grid_constant__ CUtensorMap kmap, const IndexArgs a) {
  using Cfg = IndexCfg<D>;
  constexpr int NST = Cfg::kStages;
  constexpr int TILE = Cfg::kTile;
  // As many TMEM accumulator buffers as fit in the 512 columns (at most 8),
  // so the MMA can run up to NBUF tiles ahead of the epilogue.
  constexpr int NBUF = (512 / N) < 8 ? (512 / N) : 8;
  constexpr uint32_t TMEM_COLS = NBUF * N <= 32 ? 32 : NBUF * N <= 64 ? 64 : NBUF * N <= 128 ? 128 : NBUF * N <= 256 ? 256 : 512;

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* stages = smem;
  uint8_t* bmat = stages + NST * TILE;
  uint32_t* hist_s = reinterpret_cast<uint32_t*>(bmat + N * D);
  int32_t* w_s = reinterpret_cast<int32_t*>(hist_s + kBuckets);
  int32_t* prefix = w_s + 128;                                   // [nq + 1]
  uint64_t* bars = reinterpret_cast<uint64_t*>(prefix + ((a.nq + 2) & ~1));
  uint64_t* full = bars;
  uint64_t* empty = bars + NST;
  uint64_t* tfull = bars + 2 * NST;
  uint64_t* tempty = tfull + NBUF;
  uint64_t* bready = tempty + NBUF;                              // the segment's B operand is in place
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bready + 2);
  volatile int32_t* abort_flag = reinterpret_cast<volatile int32_t*>(tmem_slot + 1);
  unsigned long long* bound_acc = reinterpret_cast<unsigned long long*>(tmem_slot + 2);

  const int tid = threadIdx.x;
  const int warp = tid >> 5;
  const int lane = tid & 31;

  // ---- work list: prefix[q+1] = tiles of query q (0 for an invalid position)
  for (int i = tid; i < a.nq; i += blockDim.x) {
    const int32_t pos = __ldg(a.query_pos + i);
    int32_t t = 0;
    if (pos < 0 || pos >= a.max_ctx) {
      record_error(a.status, CSA2_ERR_INDEX_RANGE);
    } else {
      t = (pos + 128) / 128;
    }
    prefix[i + 1] = t;
  }
  for (int i = tid; i < kBuckets; i += blockDim.x) hist_s[i] = 0;
  if (tid == 0) {
    prefix[0] = 0;
    for (int i = 0; i < NST; ++i) {
      mbar_init(&full[i], 1);
      mbar_init(&empty[i], 1);
    }
    for (int i = 0; i < NBUF; ++i) {
      mbar_init(&tfull[i], 1);
      mbar_init(&tempty[i], kEpiThreads / 64);   // one arrival per warp of the group that reads it
    }
    mbar_init(bready, kEpiThreads / 32);
    *bound_acc = 0ull;
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, TMEM_COLS);
    tmem_relinquish();
  }
  __syncthreads();
  if (warp == 0) {   // inclusive scan of tile counts, 32 at a time
    int32_t carry = 0;
    for (int base = 0; base < a.nq; base += 32) {
      const int i = base + lane;
      int32_t v = (i < a.nq) ? prefix[i + 1] : 0;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int32_t n = __shfl_up_sync(0xffffffffu, v, o);
        if (lane >= o) v += n;
      }
      if (i < a.nq) prefix[i + 1] = v + carry;
      carry += __shfl_sync(0xffffffffu, v, 31);
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  pdl_trigger();   // the next grid may be launched (it waits for this one to finish)

  const int64_t total = prefix[a.nq];
  const int64_t lo = total * blockIdx.x / gridDim.x;
  const int64_t hi = total * (blockIdx.x + 1) / gridDim.x;
  int q0 = 0;
  {
    int l = 0, r = a.nq - 1;   // last q with prefix[q] <= lo
    while (l < r) {
      const int m = (l + r + 1) >> 1;
      if (prefix[m] <= lo) l = m; else r = m - 1;
    }
    q0 = l;
  }

  // The CTA's items are processed one query segment at a time.  Within a
  // segment the producer, the MMA issuer and the epilogue run as a pipeline.
  // Between segments the whole CTA synchronises, so the B operand (the
  // query) and the histogram can be swapped without any hand-off protocol.
  // `git` numbers the items of the CTA and drives every barrier phase.
  const int et = tid - 64;                 // epilogue thread 0..255 (negative for warps 0-1)
  const int group = et >> 7;               // epilogue group: tiles i with i % 2 == group
  const int quarter = warp & 3;            // TMEM lanes this warp may access
  const int row = quarter * 32 + lane;     // key row of the tile this thread owns
  int64_t git = 0;
  int seg_count = 0;   // segments done by this CTA (bready phase)
  int q = q0;
  for (int64_t s_lo = lo; s_lo < hi;) {
    while (s_lo >= prefix[q + 1]) ++q;
    const int64_t s_hi = hi < (int64_t)prefix[q + 1] ? hi : (int64_t)prefix[q + 1];
    const int n_it = (int)(s_hi - s_lo);
    const int32_t tile0 = (int32_t)(s_lo - prefix[q]);
    const int32_t pos_q = __ldg(a.query_pos + q);

    // ---- segment set-up (epilogue threads): B operand = q rows 0..H-1, zero
    // rows up to N, K-major with the tile swizzle, and the head weights.  The
    // producer does not wait for it (key tiles do not depend on the query);
    // the MMA issuer waits on `bready`.  The int32 overflow guard
    // 128 * sum_h |w_h| * sum_d |q_hd| < 2^31 is checked off the critical path.
    const int8_t* qsrc = a.q + (int64_t)q * a.H * D;
    if (warp >= 2) {
      for (int idx = et; idx < N * (D / 16); idx += kEpiThreads) {
        const int r = idx / (D / 16), c = idx % (D / 16);
        int4 v = make_int4(0, 0, 0, 0);
        if (r < a.H) v = __ldg(reinterpret_cast<const int4*>(qsrc + r * D) + c);
        *reinterpret_cast<int4*>(bmat + swizzled_chunk(r, c, D)) = v;
      }
      if (et < N) w_s[et] = et < a.H ? (int32_t)__ldg(a.w + (int64_t)q * a.H + et) : 0;
      fence_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive(bready);
      named_sync_epi();
      if (et < a.H) {
        int32_t sq = 0;
        const int4* src = reinterpret_cast<const int4*>(qsrc + et * D);
        for (int c = 0; c < D / 16; ++c) {
          const int4 v = __ldg(src + c);
          const int32_t wv[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
          for (int j = 0; j < 4; ++j)
#pragma unroll
            for (int b = 0; b < 4; ++b) sq += abs((int32_t)(int8_t)(wv[j] >> (8 * b)));
        }
        const unsigned long long t = (unsigned long long)sq * (unsigned long long)abs(w_s[et]);
        if (t) atomicAdd(bound_acc, t);
      }
    }

    if (warp == 0) {
      // ---------------------------------------------------------- producer
      if (lane == 0) {
        prefetch_tensormap(&kmap);
        const uint64_t pol = l2_policy_evict_first();
        const int32_t seq = a.seq_of_query ? __ldg(a.seq_of_query + q) : q;
        int i = 0;
        for (; i < n_it; ++i) {
          const int64_t g = git + i;
          const int st = (int)(g % NST);
          const uint32_t ph = (uint32_t)((g / NST) & 1);
          if (!mbar_wait(&empty[st], ph ^ 1, abort_flag)) break;
          const int32_t tile = tile0 + i;
          int64_t r[2];
          uint32_t bytes = 0;
#pragma unroll
          for (int j = 0; j < 2; ++j) {
            const int32_t p0 = tile * 128 + 64 * j;
            r[j] = -1;
            if (p0 <= pos_q) {
              r[j] = map_row(a.rows, seq, p0);
              if (r[j] < 0) record_error(a.status, CSA2_ERR_INDEX_RANGE);
              else bytes += 64 * D;
            }
          }
          mbar_arrive_expect_tx(&full[st], bytes);
#pragma unroll
          for (int j = 0; j < 2; ++j)
            if (r[j] >= 0)
              tma_load_2d(stages + st * TILE + j * 64 * D, &kmap, 0, (int32_t)r[j], &full[st], pol);
        }
        if (*abort_flag) {   // let loads already in flight land before moving on
          const int64_t issued = git + i;
          const int64_t n = i < NST ? i : NST;
          for (int64_t k = issued - n; k < issued; ++k)
            mbar_wait_drain(&full[k % NST], (uint32_t)((k / NST) & 1));
        }
      }
    } else if (warp == 1) {
      // ---------------------------------------------------------- MMA issuer
      if (lane == 0) {
        constexpr uint32_t idesc = idesc_i8(128, N);
        const uint32_t b_addr = smem_u32(bmat);
        const bool bok = mbar_wait(bready, (uint32_t)(seg_count & 1), abort_flag);
        tc_fence_after();
        for (int i = 0; i < n_it && bok; ++i) {
          const int64_t g = git + i;
          const int st = (int)(g % NST);
          const uint32_t ph = (uint32_t)((g / NST) & 1);
          const int buf = (int)(g % NBUF);
          const uint32_t tph = (uint32_t)((g / NBUF) & 1);
          if (!mbar_wait(&full[st], ph, abort_flag)) break;
          if (!mbar_wait(&tempty[buf], tph ^ 1, abort_flag)) break;
          tc_fence_after();
          const uint32_t a_addr = smem_u32(stages + st * TILE);
#pragma unroll
          for (int k = 0; k < D / 32; ++k)
            mma_i8(tmem_base + buf * N, smem_desc_kmajor(a_addr + 32 * k, D),
                   smem_desc_kmajor(b_addr + 32 * k, D), idesc, k > 0 ? 1u : 0u);
          mma_commit(&empty[st]);
          mma_commit(&tfull[buf]);
        }
      }
    } else {
      // ---------------------------------------------------------- epilogue
      // Two groups of four warps (one warp per TMEM lane quarter each) take
      // alternate tiles, so the groups never wait for each other within a
      // segment.  A thread owns one key row: it loads the row's N head dots,
      // frees the TMEM buffer, applies ReLU and the head weights (kept in
      // registers) in independent partial sums, stores the score and adds
      // its bucket to the shared histogram.  Every epilogue thread walks the
      // same tiles and reaches the same barriers even after a timeout (it
      // then skips the TMEM reads and the stores).
      if (seg_count == 0) pdl_wait();   // scores and histogram: after the grid before (it zeroes them)
      constexpr bool kRegW = N <= 64;
      int32_t wreg[kRegW ? N : 1];
      if constexpr (kRegW) {
#pragma unroll
        for (int h = 0; h < N; ++h) wreg[h] = w_s[h];
      }
      for (int i = group; i < n_it; i += 2) {
        const int64_t g = git + i;
        const bool ok = __all_sync(0xffffffffu, mbar_wait(&tfull[g % NBUF], (uint32_t)((g / NBUF) & 1), abort_flag));
        uint32_t r[N];
        if (ok) {
          tc_fence_after();
          const uint32_t taddr = tmem_base + ((uint32_t)(quarter * 32) << 16) + (uint32_t)((g % NBUF) * N);
          if constexpr (N == 16) {
            tmem_ld16(taddr, r);
          } else {
#pragma unroll
            for (int c = 0; c < N / 32; ++c)
              tmem_ld32(taddr + 32 * c, *reinterpret_cast<uint32_t(*)[32]>(&r[32 * c]));
          }
          tmem_wait_ld();
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&tempty[g % NBUF]);
        if (ok) {
          int32_t part[8] = {0, 0, 0, 0, 0, 0, 0, 0};   // independent chains, no long serial sum
#pragma unroll
          for (int h = 0; h < N; ++h) part[h & 7] += (kRegW ? wreg[h] : w_s[h]) * max((int32_t)r[h], 0);
          const int32_t sc = ((part[0] + part[1]) + (part[2] + part[3])) + ((part[4] + part[5]) + (part[6] + part[7]));
          const int32_t pos = (tile0 + i) * 128 + row;
          if (pos <= pos_q) {
            a.scores[(int64_t)q * a.ld + pos] = sc;
            atomicAdd(&hist_s[score_bucket(sc)], 1u);
          }
        }
      }
      // this query's histogram goes to global memory
      named_sync_epi();
      if (a.hist) {
        for (int b = et; b < kBuckets; b += kEpiThreads) {
          const uint32_t v = hist_s[b];
          if (v) {
            atomicAdd(a.hist + (int64_t)q * kBuckets + b, v);
            hist_s[b] = 0;
          }
        }
      }
    }
    tc_fence_before();
    __syncthreads();   // the segment is done everywhere: B and the histogram may be reused
    tc_fence_after();
    if (tid == 64) {
      if ((*bound_acc) * 128ull >= (1ull << 31)) record_error(a.status, CSA2_ERR_SCORE_RANGE);
      *bound_acc = 0ull;
    }
    __syncthreads();
    git += n_it;
    ++seg_count;
    s_lo = s_hi;
  }

  if (warp == 1) tmem_dealloc(tmem_base, TMEM_COLS);
  if (tid == 0 && *abort_flag) record_error(a.status, CSA2_ERR_TIMEOUT);
}

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  if (!fn) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult qr;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &qr) == cudaSuccess &&
        qr == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  }
  return fn;
}

template <int D>
size_t index_smem_bytes(int N, int nq) {
  using Cfg = IndexCfg<D>;
  return 1024 + (size_t)Cfg::kStages * Cfg::kTile + (size_t)N * D + kBuckets * 4 + 128 * 4 +
         (size_t)((nq + 2) & ~1) * 4 + (2 * Cfg::kStages + 2 * 8) * 8 + 32;
}

template <int D, int N>
cudaError_t launch_one(const CUtensorMap& map, const IndexArgs& a, int grid, cudaStream_t st) {
  const size_t smem = index_smem_bytes<D>(N, a.nq);
  static unsigned long long done = 0;
  cudaError_t e = ensure_smem(index_score_kernel<D, N>, (int)index_smem_bytes<D>(N, kMaxQueries), done);
  if (e != cudaSuccess) return e;
  return launch_k(index_score_kernel<D, N>, dim3(grid), dim3(64 + kEpiThreads), smem, st, false, launch_opts().pdl,
                  map, a);
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
                               cudaStream_t st) {
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

  IndexArgs a{q, w, seq_of_query, query_pos, to_rowmap(keys), nq, H, max_ctx, scores, ld, hist, status};
  const int64_t upper = (int64_t)nq * ((max_ctx + 127) / 128);
  const int grid = (int)(upper < sm_count() ? (upper > 0 ? upper : 1) : sm_count());
  const int N = H <= 16 ? 16 : H <= 32 ? 32 : H <= 64 ? 64 : 128;
  if (D == 128) {
    switch (N) {
      case 16: return launch_one<128, 16>(map, a, grid, st);
      case 32: return launch_one<128, 32>(map, a, grid, st);
      case 64: return launch_one<128, 64>(map, a, grid, st);
      default: return launch_one<128, 128>(map, a, grid, st);
    }
  }
  switch (N) {
    case 16: return launch_one<64, 16>(map, a, grid, st);
    case 32: return launch_one<64, 32>(map, a, grid, st);
    case 64: return launch_one<64, 64>(map, a, grid, st);
    default: return launch_one<64, 128>(map, a, grid, st);
  }
}

}  // namespace csa2
