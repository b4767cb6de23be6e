// K2: exact top-k over int32 scores, ties to the lower position, results in
// ascending position order (the candidate pool of up to 16,384 positions and
// the 512-position selections: "How DeepSeek V4.1 Flash Actually Works",
// three KV-cache optimizations, item 2).
//
// Every candidate j gets the 64-bit key (score ^ sign bit) << 32 | ~j.  Keys
// are distinct, and a larger key is a better candidate: higher score, then
// lower index.  The index order equals the position order because candidate
// positions ascend.  The top-k is therefore {j : key_j >= kth}, where kth
// is the k-th largest key.
//
// Every candidate also gets a 13-bit bucket, monotone in its score.  Counting
// buckets gives the threshold bucket b*: everything above b* is in, and
// the k-th key is among the b* candidates ("ties").  A radix select on the
// ties finds it, and a stable compaction writes the members in position
// order.  No sort is needed.
//
// Passes:
//   hist    bucket histogram (fused into the index-score kernel when the scores
//           come from there)
//   select  (topk_select.cu) when the rows fit on the device at once: the
//           whole selection in one launch of co-resident CTAs; it is also the
//           small-n path (n <= kSmallMax, one CTA per query)
//   rows    (topk_rows.cu) many rows of up to kRowSelMax candidates: one CTA
//           per row, with its own histogram
// Otherwise, the multi-pass path:
//   thresh  one CTA per query finds b* from the histogram
//   gather  one CTA per 4096-candidate chunk counts the chunk's candidates
//           with bucket >= b*, publishes the count, adds up the counts of the
//           chunks before it (bounded wait), and writes those candidates' keys
//           in position order
//   finish  one CTA per (query, k): radix select of the k-th key among the
//           ties of its ordered candidate list, then the ordered compaction
//           (a list that overflowed its capacity is redone from the score row)
// Bucket histograms use plain shared atomics (scores spread over many buckets);
// the digit histograms of the radix select, where lanes collide, are warp-aggregated.
#include "csa2_device.cuh"
#include "internal.h"

namespace csa2 {

size_t topk_scratch_bytes(int32_t nq, int32_t n_max) {
  Carver c(nullptr);
  carve_topk(c, nq, n_max);
  return c.used + 256;
}

TopkScratch carve_topk(Carver& c, int32_t nq, int32_t n_max) {
  TopkScratch s;
  s.n_chunks = (int32_t)(((int64_t)n_max + kChunk - 1) / kChunk);
  if (s.n_chunks < 1) s.n_chunks = 1;
  s.cand_cap = kCandCap;
  s.hist = c.take<uint32_t>((size_t)nq * kBuckets);
  s.sel_hdr = c.take<uint32_t>((size_t)nq * 4);   // directly after hist: one memset zeroes both
  s.chunk_cnt = c.take<uint32_t>((size_t)nq * 2 * s.n_chunks * 2);   // published (flag, count) pairs
  s.cand = c.take<uint64_t>((size_t)nq * 2 * s.cand_cap);
  s.cand_cnt = c.take<uint32_t>((size_t)nq * 2);
  s.kth = c.take<uint64_t>((size_t)nq * 2);
  s.thresh = c.take<int32_t>((size_t)nq * 4);
  s.sel_ties = c.take<uint64_t>((size_t)nq * 2 * kSelTieCap);
  s.sel_mcnt = c.take<uint32_t>((size_t)nq * 2 * kSelMaxG);
  s.sel_radix = c.take<uint32_t>((size_t)nq * 2 * 8 * 256);
  return s;
}

namespace {

struct CandView {
  const int32_t* scores;
  int64_t ld;
  const int32_t* n_valid;
  const int32_t* query_pos;
  const int32_t* cand_pos;
  int32_t n_max;
};

// Number of valid candidates of query q.
__device__ __forceinline__ int32_t n_of(const CandView& v, int q) {
  if (v.n_valid) {
    const int32_t n = __ldg(v.n_valid + q);
    return n < 0 ? 0 : (n > v.n_max ? v.n_max : n);
  }
  if (v.query_pos) {
    const int32_t p = __ldg(v.query_pos + q);
    return (p < 0 || p >= v.n_max) ? 0 : p + 1;
  }
  return v.n_max;
}

__device__ __forceinline__ int32_t pos_of(const CandView& v, int q, int32_t j) {
  return v.cand_pos ? __ldg(v.cand_pos + (int64_t)q * v.ld + j) : j;
}

__device__ __forceinline__ uint64_t key_of(int32_t score, int32_t j) { return cand_key(score, j); }
__device__ __forceinline__ int32_t key_index(uint64_t key) { return key_pos(key); }
__device__ __forceinline__ int32_t key_bucket(uint64_t key) { return (int32_t)score_bucket(key_score(key)); }

// One increment of hist[bin] per active lane, aggregated over lanes that hit
// the same bin.  All 32 lanes of the warp must call it.
__device__ __forceinline__ void agg_inc(uint32_t* hist, uint32_t bin, bool active) {
  const uint32_t v = active ? bin : 0xFFFFFFFFu;
  const uint32_t peers = __match_any_sync(0xffffffffu, v);
  if (active && (threadIdx.x & 31) == (uint32_t)(__ffs(peers) - 1)) atomicAdd(hist + bin, (uint32_t)__popc(peers));
}

// Block-wide exclusive scan of one int per thread (blockDim.x <= 1024).
__device__ __forceinline__ int32_t block_excl_scan(int32_t v, int32_t* tmp, int32_t* total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = (blockDim.x + 31) >> 5;
  int32_t x = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int32_t n = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += n;
  }
  if (lane == 31) tmp[warp] = x;
  __syncthreads();
  if (warp == 0) {
    int32_t y = lane < nw ? tmp[lane] : 0;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int32_t n = __shfl_up_sync(0xffffffffu, y, o);
      if (lane >= o) y += n;
    }
    if (lane < nw) tmp[lane] = y;   // inclusive warp totals
  }
  __syncthreads();
  const int32_t base = warp > 0 ? tmp[warp - 1] : 0;
  if (total) *total = tmp[nw - 1];
  __syncthreads();
  return base + x - v;
}

// Threshold bucket for k: the largest b with count(>= b) >= k, or -1 when
// there are at most k candidates (all are members).  Also returns the count
// strictly above b*.  All NT threads of the block call it.  Each thread reads
// its kBuckets/NT contiguous bins with 16-byte loads, all issued before any
// is used (the histogram may be in global or shared memory).
template <int NT>
__device__ void find_threshold(const uint32_t* hist, int32_t k, int32_t* out_b, int32_t* out_above,
                               int32_t* tmp) {
  constexpr int PER = kBuckets / NT;
  static_assert(PER % 4 == 0, "bins per thread must be a multiple of 4");
  const int t = threadIdx.x;
  // thread t owns bins [kBuckets - (t+1)*PER, kBuckets - t*PER): the highest first
  const uint4* src = reinterpret_cast<const uint4*>(hist + kBuckets - (t + 1) * PER);
  uint4 v[PER / 4];
#pragma unroll
  for (int i = 0; i < PER / 4; ++i) v[i] = src[i];
  uint32_t bins[PER];
#pragma unroll
  for (int i = 0; i < PER / 4; ++i) {
    bins[4 * i] = v[i].x;
    bins[4 * i + 1] = v[i].y;
    bins[4 * i + 2] = v[i].z;
    bins[4 * i + 3] = v[i].w;
  }
  int32_t sum = 0;
#pragma unroll
  for (int i = 0; i < PER; ++i) sum += (int32_t)bins[i];
  int32_t total;
  const int32_t before = block_excl_scan(sum, tmp, &total);   // count in higher segments
  if (t == 0 && total <= k) {
    *out_b = -1;
    *out_above = total;
  }
  if (total > k && before < k && before + sum >= k) {
    int32_t acc = before;
#pragma unroll
    for (int i = PER - 1; i >= 0; --i) {     // from this thread's highest bin down
      const int32_t c = (int32_t)bins[i];
      if (acc + c >= k) {
        *out_b = kBuckets - (t + 1) * PER + i;
        *out_above = acc;
        break;
      }
      acc += c;
    }
  }
  __syncthreads();
}

// Returns, to every thread of the block, the need-th largest (1-based) of the
// non-zero keys among get(0..m-1) (zero marks "not a candidate"; need is at
// most the number of non-zero keys).  The bits above the highest bit where the
// candidates differ are common; digits of at most 8 bits are fixed from there
// downwards, and the select stops early once every key under the fixed prefix
// is a member (kth is then the smallest of them).
template <class Get>
__device__ uint64_t radix_select(Get get, int64_t m, int64_t need, uint32_t* hist256,
                                 unsigned long long* red) {
  __shared__ int32_t dsel;
  __shared__ long long rnew;
  __shared__ uint32_t dcnt;
  if (threadIdx.x == 0) {
    red[0] = ~0ull;
    red[1] = 0ull;
  }
  __syncthreads();
  unsigned long long kand = ~0ull, kor = 0ull;
  for (int64_t i = threadIdx.x; i < m; i += blockDim.x) {
    const uint64_t k = get(i);
    if (k) {
      kand &= k;
      kor |= k;
    }
  }
  atomicAnd(&red[0], kand);
  atomicOr(&red[1], kor);
  __syncthreads();
  const uint64_t kand_all = red[0], diff = red[0] ^ red[1];
  __syncthreads();
  if (diff == 0) return kand_all;
  int top = 63 - __clzll((long long)diff);
  uint64_t fixed = (top == 63) ? 0ull : ~((2ull << top) - 1ull);   // bits above `top`
  uint64_t prefix = kand_all & fixed;
  int64_t r = need;
  const int64_t m_pad = (m + 31) & ~int64_t(31);
  while (true) {
    const int lo = top >= 7 ? top - 7 : 0;
    const uint32_t dmask = (uint32_t)((2ull << (top - lo)) - 1ull);
    for (int i = threadIdx.x; i < 256; i += blockDim.x) hist256[i] = 0;
    __syncthreads();
    for (int64_t i = threadIdx.x; i < m_pad; i += blockDim.x) {
      const uint64_t k = i < m ? get(i) : 0ull;
      const bool in = k && (k & fixed) == prefix;
      agg_inc(hist256, (uint32_t)(k >> lo) & dmask, in);
    }
    __syncthreads();
    if (threadIdx.x < 32) {   // walk digits from the top, 8 per lane
      const int lane = threadIdx.x;
      uint32_t seg = 0;
      for (int i = 0; i < 8; ++i) seg += hist256[255 - (lane * 8 + i)];
      uint32_t incl = seg;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const uint32_t nn = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += nn;
      }
      const uint32_t before = incl - seg;
      if ((int64_t)before < r && (int64_t)incl >= r) {
        uint32_t acc = before;
        for (int i = 0; i < 8; ++i) {
          const int d = 255 - (lane * 8 + i);
          const uint32_t cnt = hist256[d];
          if ((int64_t)(acc + cnt) >= r) {
            dsel = d;
            rnew = r - acc;
            dcnt = cnt;
            break;
          }
          acc += cnt;
        }
      }
    }
    __syncthreads();
    prefix |= (uint64_t)dsel << lo;
    fixed = (lo == 0) ? ~0ull : ~((1ull << lo) - 1ull);
    r = rnew;
    const uint32_t cnt = dcnt;
    __syncthreads();
    if (lo == 0) return prefix;
    if ((int64_t)cnt == r) {   // all keys under the prefix are in: kth is their minimum
      if (threadIdx.x == 0) red[0] = ~0ull;
      __syncthreads();
      for (int64_t i = threadIdx.x; i < m; i += blockDim.x) {
        const uint64_t k = get(i);
        if (k && (k & fixed) == prefix) atomicMin(&red[0], (unsigned long long)k);
      }
      __syncthreads();
      const uint64_t res = red[0];
      __syncthreads();
      return res;
    }
    top = lo - 1;
  }
}

// ------------------------------------------------------------------ hist
__global__ void __launch_bounds__(256) topk_hist_kernel(CandView v, uint32_t* hist) {
  pdl_wait();      // the scores come from the grid before
  pdl_trigger();
  __shared__ uint32_t h[kBuckets];
  const int q = blockIdx.y;
  const int32_t n = n_of(v, q);
  const int32_t j0 = blockIdx.x * kChunk;
  if (j0 >= n) return;
  for (int i = threadIdx.x; i < kBuckets; i += blockDim.x) h[i] = 0;
  __syncthreads();
  const int32_t* sc = v.scores + (int64_t)q * v.ld;
  constexpr int kPerT = kChunk / 256;
  int32_t sr[kPerT];
#pragma unroll
  for (int i = 0; i < kPerT; ++i) {            // all loads in flight before any use
    const int32_t j = j0 + i * 256 + threadIdx.x;
    sr[i] = j < n ? __ldg(sc + j) : 0;
  }
#pragma unroll
  for (int i = 0; i < kPerT; ++i) {
    const int32_t j = j0 + i * 256 + threadIdx.x;
    if (j < n) atomicAdd(&h[score_bucket(sr[i])], 1u);
  }
  __syncthreads();
  // one 64-bit add per populated pair of buckets (no carry: a count stays below 2^32)
  unsigned long long* gh = reinterpret_cast<unsigned long long*>(hist + (int64_t)q * kBuckets);
  for (int i = threadIdx.x; i < kBuckets / 2; i += blockDim.x) {
    const uint32_t lo = h[2 * i], hi = h[2 * i + 1];
    if (lo | hi) atomicAdd(gh + i, (unsigned long long)lo | ((unsigned long long)hi << 32));
  }
}

// ------------------------------------------------------------------ thresholds
struct ThreshArgs {
  TopkScratch s;
  int32_t k[2];
  int32_t n_k;
};

// One CTA per query: the threshold bucket and the count above it, per k.
__global__ void __launch_bounds__(256) topk_thresh_kernel(ThreshArgs a) {
  __shared__ int32_t tmp[32];
  __shared__ int32_t b_s, above_s;
  const int q = blockIdx.x;
  pdl_wait();      // the histogram comes from the grids before
  pdl_trigger();
  // the gather's published chunk counts start at zero (the gather runs after
  // this grid has completed)
  unsigned long long* pub = reinterpret_cast<unsigned long long*>(a.s.chunk_cnt) + (int64_t)q * 2 * a.s.n_chunks;
  for (int i = threadIdx.x; i < 2 * a.s.n_chunks; i += blockDim.x) pub[i] = 0ull;
  const uint32_t* hist = a.s.hist + (int64_t)q * kBuckets;
  for (int t = 0; t < a.n_k; ++t) {
    find_threshold<256>(hist, a.k[t], &b_s, &above_s, tmp);
    if (threadIdx.x == 0) {
      a.s.thresh[(q * 2 + t) * 2 + 0] = b_s;
      a.s.thresh[(q * 2 + t) * 2 + 1] = above_s;
    }
    __syncthreads();
  }
}

// ------------------------------------------------------------------ gather
struct GatherArgs {
  CandView v;
  TopkScratch s;
  int32_t n_k;
  int32_t* status;
};

constexpr int kPer = kChunk / 256;   // candidates per thread in the chunk kernel

__device__ __forceinline__ unsigned long long ld_relaxed_u64(const unsigned long long* p) {
  unsigned long long v;
  asm volatile("ld.relaxed.gpu.global.u64 %0, [%1];" : "=l"(v) : "l"(p) : "memory");
  return v;
}

__global__ void __launch_bounds__(256) topk_gather_kernel(GatherArgs a) {
  pdl_wait();      // scores, thresholds and zeroed counts come from the grids before
  pdl_trigger();
  __shared__ int32_t tmp[32];
  __shared__ int32_t base_s;
  const int q = blockIdx.y, c = blockIdx.x;
  const int32_t n = n_of(a.v, q);
  const int32_t j0 = c * kChunk + threadIdx.x * kPer;
  const int32_t* sc = a.v.scores + (int64_t)q * a.v.ld;
  int32_t s[kPer];
  int32_t bk[kPer];
#pragma unroll
  for (int i = 0; i < kPer; ++i) {
    const int32_t j = j0 + i;
    s[i] = j < n ? __ldg(sc + j) : 0;
  }
  int32_t bst[2];
  bst[0] = a.s.thresh[(q * 2 + 0) * 2];
  bst[1] = a.n_k > 1 ? a.s.thresh[(q * 2 + 1) * 2] : 0;
#pragma unroll
  for (int i = 0; i < kPer; ++i) bk[i] = j0 + i < n ? (int32_t)score_bucket(s[i]) : -2;
  if (a.v.cand_pos) {
    int32_t p[kPer + 1];
#pragma unroll
    for (int i = 0; i <= kPer; ++i) {
      const int32_t j = j0 + i - 1;
      p[i] = (j >= 0 && j < n) ? pos_of(a.v, q, j) : 0;
    }
#pragma unroll
    for (int i = 1; i <= kPer; ++i) {
      const int32_t j = j0 + i - 1;
      if (j > 0 && j < n && p[i] <= p[i - 1]) record_error(a.status, CSA2_ERR_ORDER);
    }
  }
  for (int t = 0; t < a.n_k; ++t) {
    const int32_t bstar = bst[t];
    int32_t cnt = 0;
#pragma unroll
    for (int i = 0; i < kPer; ++i) cnt += bk[i] >= bstar && bk[i] > -2;
    int32_t chunk_total;
    const int32_t off = block_excl_scan(cnt, tmp, &chunk_total);
    // publish this chunk's count, then add up the counts of the chunks before it
    unsigned long long* pub =
        reinterpret_cast<unsigned long long*>(a.s.chunk_cnt) + ((int64_t)q * 2 + t) * a.s.n_chunks;
    if (threadIdx.x == 0) atomicExch(pub + c, (1ull << 32) | (uint32_t)chunk_total);
    int32_t part = 0;
    bool ok = true;
    for (int i = threadIdx.x; i < c; i += blockDim.x) {
      unsigned long long v = ld_relaxed_u64(pub + i);
      if (!(v >> 32)) {
        const uint64_t t0 = global_ns();
        while (!((v = ld_relaxed_u64(pub + i)) >> 32)) {
          if (global_ns() - t0 > kWaitLimitNs) {
            ok = false;
            break;
          }
        }
      }
      part += (int32_t)(uint32_t)v;
    }
    if (!ok) record_error(a.status, CSA2_ERR_TIMEOUT);
    int32_t before;
    block_excl_scan(part, tmp, &before);
    if (threadIdx.x == 0) {
      base_s = before;
      const int32_t last = n > 0 ? (n - 1) / kChunk : 0;   // the chunk holding the last candidate
      if (c == last) a.s.cand_cnt[q * 2 + t] = (uint32_t)(before + chunk_total);
    }
    __syncthreads();
    int32_t w = base_s + off;
    uint64_t* dst = a.s.cand + ((int64_t)q * 2 + t) * a.s.cand_cap;
#pragma unroll
    for (int i = 0; i < kPer; ++i) {
      if (bk[i] >= bstar && bk[i] > -2) {
        if (w < a.s.cand_cap) dst[w] = key_of(s[i], j0 + i);
        ++w;
      }
    }
    __syncthreads();
  }
}

// ------------------------------------------------------------------ finish
struct FinishArgs {
  CandView v;
  TopkScratch s;
  TopkOut out[2];
};

constexpr int kTieCap = 2048;
constexpr int kFinishPer = (kCandCap + 1023) / 1024;   // list keys per thread: i*1024 + thread

// One CTA per (query, k).  The candidate list (position order) is loaded once
// with all loads in flight, then every pass over it is a fully unrolled loop
// over shared memory.  The ordered write uses per-(pass, warp) member counts,
// as in the one-CTA kernel.
__global__ void __launch_bounds__(1024, 1) topk_finish_kernel(FinishArgs a) {
  pdl_wait();      // the candidate lists come from the grid before
  pdl_trigger();
  extern __shared__ uint64_t keys_s[];            // [cand_cap] then [kTieCap] ties
  uint64_t* ties = keys_s + kCandCap;
  __shared__ int32_t cmat[kFinishPer * 32];
  __shared__ uint32_t hist256[256];
  __shared__ unsigned long long red[2];
  __shared__ int32_t tmp[32];
  __shared__ unsigned long long found;
  const int q = blockIdx.x, t = blockIdx.y, tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const TopkOut o = a.out[t];
  const int32_t n = n_of(a.v, q);
  const int32_t k = o.k;
  const int32_t bstar = a.s.thresh[(q * 2 + t) * 2 + 0];
  const int32_t above = a.s.thresh[(q * 2 + t) * 2 + 1];
  const int32_t m = n > 0 ? (int32_t)a.s.cand_cnt[q * 2 + t] : 0;
  int32_t* dst = o.idx + (int64_t)q * k;
  const int32_t total = n < k ? n : k;
  uint64_t kth = 0ull;
  const int32_t* sc = a.v.scores + (int64_t)q * a.v.ld;
  if (m <= kCandCap) {
    const unsigned long long* src =
        reinterpret_cast<const unsigned long long*>(a.s.cand + ((int64_t)q * 2 + t) * a.s.cand_cap);
    {
      uint64_t r[kFinishPer];
#pragma unroll
      for (int i = 0; i < kFinishPer; ++i) {
        const int32_t j = i * 1024 + tid;
        r[i] = j < m ? __ldcg(src + j) : 0ull;
      }
#pragma unroll
      for (int i = 0; i < kFinishPer; ++i) keys_s[i * 1024 + tid] = r[i];
    }
    __syncthreads();
    if (bstar >= 0 && n > k) {
      const int64_t need = (int64_t)k - above;
      int32_t cnt = 0;
#pragma unroll
      for (int i = 0; i < kFinishPer; ++i) {
        const int32_t j = i * 1024 + tid;
        cnt += j < m && key_bucket(keys_s[j]) == bstar;
      }
      int32_t nt;
      int32_t w = block_excl_scan(cnt, tmp, &nt);
      if (nt <= kTieCap) {
#pragma unroll
        for (int i = 0; i < kFinishPer; ++i) {
          const int32_t j = i * 1024 + tid;
          if (j < m && key_bucket(keys_s[j]) == bstar) ties[w++] = keys_s[j];
        }
      }
      if (tid == 0) found = 0ull;
      __syncthreads();
      if (nt <= 1024) {   // exact rank among the ties
        if (tid < nt) {
          const uint64_t ki = ties[tid];
          int32_t above_i = 0;
          for (int32_t j = 0; j < nt; ++j) above_i += ties[j] > ki;
          if (above_i == need - 1) found = ki;
        }
        __syncthreads();
        kth = found;
      } else if (nt <= kTieCap) {
        kth = radix_select([&](int64_t i) { return ties[i]; }, nt, need, hist256, red);
      } else {
        kth = radix_select([&](int64_t i) { return key_bucket(keys_s[i]) == bstar ? keys_s[i] : 0ull; }, m,
                           need, hist256, red);
      }
    }
    uint32_t mem = 0;
#pragma unroll
    for (int i = 0; i < kFinishPer; ++i) {
      const int32_t j = i * 1024 + tid;
      const bool in = j < m && keys_s[j] >= kth;
      mem |= (uint32_t)in << i;
      const uint32_t bal = __ballot_sync(0xffffffffu, in);
      if (lane == 0) cmat[i * 32 + warp] = __popc(bal);
    }
    __syncthreads();
    const int32_t cval = tid < kFinishPer * 32 ? cmat[tid] : 0;
    const int32_t cbase = block_excl_scan(cval, tmp, nullptr);
    if (tid < kFinishPer * 32) cmat[tid] = cbase;
    __syncthreads();
#pragma unroll
    for (int i = 0; i < kFinishPer; ++i) {
      const int32_t j = i * 1024 + tid;
      const bool in = (mem >> i) & 1u;
      const uint32_t bal = __ballot_sync(0xffffffffu, in);
      const int32_t slot = cmat[i * 32 + warp] + __popc(bal & ((1u << lane) - 1u));
      if (in && slot < k) dst[slot] = pos_of(a.v, q, key_index(keys_s[j]));
    }
  } else {
    // The list overflowed (a very flat score distribution): select and compact
    // over the whole score row instead.
    auto get = [&](int64_t j) -> uint64_t {
      const int32_t s = __ldg(sc + j);
      return (int32_t)score_bucket(s) == bstar ? key_of(s, (int32_t)j) : 0ull;
    };
    if (bstar >= 0 && n > k) kth = radix_select(get, n, (int64_t)k - above, hist256, red);
    __shared__ int32_t run;
    if (tid == 0) run = 0;
    __syncthreads();
    for (int32_t base = 0; base < n; base += 1024 * 8) {
      const int32_t j0 = base + tid * 8;
      int32_t cnt = 0;
      for (int i = 0; i < 8; ++i) cnt += (j0 + i < n) && key_of(__ldg(sc + j0 + i), j0 + i) >= kth;
      int32_t tot;
      int32_t w = run + block_excl_scan(cnt, tmp, &tot);
      for (int i = 0; i < 8; ++i) {
        const int32_t j = j0 + i;
        if (j < n && key_of(__ldg(sc + j), j) >= kth) {
          if (w < k) dst[w] = pos_of(a.v, q, j);
          ++w;
        }
      }
      __syncthreads();
      if (tid == 0) run += tot;
      __syncthreads();
    }
  }
  for (int32_t i = total + tid; i < k; i += 1024) dst[i] = -1;
  if (tid == 0) {
    if (o.cnt) o.cnt[q] = total;
    a.s.kth[q * 2 + t] = kth;
  }
}

}  // namespace

cudaError_t launch_topk_large(const int32_t* scores, int64_t ld, const int32_t* n_valid,
                              const int32_t* query_pos, const int32_t* cand_pos, int32_t nq,
                              int32_t n_max, const TopkOut* outs, int32_t n_k,
                              const TopkScratch& s, bool hist_ready, int32_t* status,
                              cudaStream_t st) {
  CandView v{scores, ld, n_valid, query_pos, cand_pos, n_max};
  const dim3 grid(s.n_chunks, nq);
  cudaError_t e;
  // Many rows that do not fit on the device at once: one CTA per row, which
  // builds its own histogram.  Fewer rows than half the SMs (a decode batch of
  // long sequences) would leave most SMs idle that way: they take the chunked
  // passes below, which spread every row over many CTAs.
  if (!select_fits(nq, n_max) && n_max <= kRowSelMax && 2 * nq >= sm_count())
    return launch_row_select(scores, ld, n_valid, query_pos, cand_pos, nq, n_max, outs, n_k, status, st);
  const bool pdl = launch_opts().pdl;
  if (!hist_ready) {
    e = cudaMemsetAsync(s.hist, 0, topk_zero_bytes(nq), st);
    if (e != cudaSuccess) return e;
    e = launch_k(topk_hist_kernel, grid, dim3(256), 0, st, false, false, v, s.hist);
    if (e != cudaSuccess) return e;
  }
  // One pass of co-resident select CTAs when the rows fit on the device.
  e = launch_select(scores, ld, n_valid, query_pos, cand_pos, nq, n_max, outs, n_k, s.hist, &s, status, st);
  if (e != cudaErrorNotSupported) return e;
  (void)cudaGetLastError();
  // thresholds (which also zero the gather's chunk counts), gather, finish:
  // programmatic dependents of one another within a plan step
  ThreshArgs ta{s, {outs[0].k, n_k > 1 ? outs[1].k : 0}, n_k};
  e = launch_k(topk_thresh_kernel, dim3(nq), dim3(256), 0, st, false, pdl, ta);
  if (e != cudaSuccess) return e;
  GatherArgs ga{v, s, n_k, status};
  e = launch_k(topk_gather_kernel, grid, dim3(256), 0, st, false, pdl, ga);
  if (e != cudaSuccess) return e;
  const int smem = (kCandCap + kTieCap) * 8;
  static SetupMask done{0};
  e = ensure_smem(topk_finish_kernel, smem, done);
  if (e != cudaSuccess) return e;
  FinishArgs fa{v, s, {outs[0], n_k > 1 ? outs[1] : outs[0]}};
  return launch_k(topk_finish_kernel, dim3(nq, n_k), dim3(1024), smem, st, false, pdl, fa);
}

cudaError_t launch_topk_small(const int32_t* scores, int64_t ld, const int32_t* n_valid,
                              const int32_t* cand_pos, int32_t nq, int32_t n_max, int32_t k,
                              int32_t* out_idx, int32_t* out_cnt, int32_t* status,
                              cudaStream_t st) {
  const TopkOut o{out_idx, out_cnt, k};
  return launch_select(scores, ld, n_valid, nullptr, cand_pos, nq, n_max, &o, 1, nullptr, nullptr, status, st);
}

}  // namespace csa2
