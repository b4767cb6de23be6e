// K2: exact top-k over int32 scores, ties to the lower position, results in
// ascending position order (the candidate pool of up to 16,384 positions and
// the 512-position selections: "How DeepSeek V4.1 Flash Actually Works",
// three KV-cache optimizations, item 2).
//
// Every candidate j gets the 64-bit key (score ^ sign bit) << 32 | ~j.  Keys
// are distinct, and a larger key is a better candidate: higher score, then
// lower index.  The index order equals the position order because candidate
// positions ascend.  The top-k is therefore {j : key_j >= kth}, where kth
// is the k-th largest key.  Finding kth is a radix select; writing the
// members in index order is a stable stream compaction, so no sort is needed.
//
// Large n (multi-CTA, one chunk of kChunk candidates per CTA):
//   hist    12-bit monotone score buckets -> per-query histogram (fused into
//           the index-score kernel when the scores come from there)
//   select  each CTA finds the threshold bucket b* from the histogram, counts
//           its members above b*, and appends threshold-bucket keys to a
//           candidate list
//   resolve one CTA per (query, k): radix select of the k-th key among the
//           threshold-bucket keys (in shared memory; a global-memory fallback
//           covers lists that overflow), then per-chunk member counts
//   write   each CTA writes its chunk's members at the prefix of the counts
//           of the chunks before it
// Small n (<= kSmallMax): one CTA per query does all of this in shared memory.
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
  s.chunk_cnt = c.take<uint32_t>((size_t)nq * 2 * s.n_chunks);
  s.cand = c.take<uint64_t>((size_t)nq * 2 * s.cand_cap);
  s.cand_cnt = c.take<uint32_t>((size_t)nq * 2);
  s.kth = c.take<uint64_t>((size_t)nq * 2);
  s.thresh = c.take<int32_t>((size_t)nq * 4);
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

// Threshold bucket for k from a 4096-bucket histogram: the largest b with
// count(>= b) >= k.  Returns b* (or -1 when every candidate is a member) and
// the count strictly above it.  Called by all threads of a 256-thread block.
__device__ void find_threshold(const uint32_t* hist, int32_t k, int32_t* out_b, int32_t* out_above,
                               int32_t* tmp) {
  const int t = threadIdx.x;              // 256 threads x 16 buckets, from the top
  int32_t seg[16];
  int32_t sum = 0;
#pragma unroll
  for (int i = 0; i < 16; ++i) {
    seg[i] = (int32_t)hist[kBuckets - 1 - (t * 16 + i)];
    sum += seg[i];
  }
  int32_t total;
  const int32_t before = block_excl_scan(sum, tmp, &total);   // count in higher segments
  if (t == 0 && total <= k) {
    *out_b = -1;
    *out_above = total;
  }
  if (total > k && before < k && before + sum >= k) {
    int32_t acc = before;
#pragma unroll
    for (int i = 0; i < 16; ++i) {
      if (acc + seg[i] >= k) {
        *out_b = kBuckets - 1 - (t * 16 + i);
        *out_above = acc;
        break;
      }
      acc += seg[i];
    }
  }
  __syncthreads();
}

// ------------------------------------------------------------------ hist
__global__ void __launch_bounds__(256) topk_hist_kernel(CandView v, uint32_t* hist) {
  __shared__ uint32_t h[kBuckets];
  const int q = blockIdx.y;
  const int32_t n = n_of(v, q);
  const int64_t j0 = (int64_t)blockIdx.x * kChunk;
  if (j0 >= n) return;
  for (int i = threadIdx.x; i < kBuckets; i += blockDim.x) h[i] = 0;
  __syncthreads();
  const int32_t j1 = (int32_t)(j0 + kChunk < (int64_t)n ? j0 + kChunk : (int64_t)n);
  const int32_t* sc = v.scores + (int64_t)q * v.ld;
  for (int32_t j = (int32_t)j0 + threadIdx.x; j < j1; j += blockDim.x)
    atomicAdd(&h[score_bucket(__ldg(sc + j))], 1u);
  __syncthreads();
  for (int i = threadIdx.x; i < kBuckets; i += blockDim.x)
    if (h[i]) atomicAdd(hist + (int64_t)q * kBuckets + i, h[i]);
}

// ------------------------------------------------------------------ select
struct SelectArgs {
  CandView v;
  TopkScratch s;
  int32_t k[2];
  int32_t n_k;
  int32_t* status;
};

__global__ void __launch_bounds__(256) topk_select_kernel(SelectArgs a) {
  __shared__ int32_t tmp[32];
  __shared__ int32_t b_s[2], above_s[2];
  __shared__ uint32_t cnt_s[2];
  const int q = blockIdx.y, c = blockIdx.x;
  const int32_t n = n_of(a.v, q);
  const uint32_t* hist = a.s.hist + (int64_t)q * kBuckets;
  for (int t = 0; t < a.n_k; ++t) find_threshold(hist, a.k[t], &b_s[t], &above_s[t], tmp);
  if (threadIdx.x < 2) cnt_s[threadIdx.x] = 0;
  if (c == 0 && threadIdx.x < a.n_k) {
    a.s.thresh[(q * 2 + threadIdx.x) * 2 + 0] = b_s[threadIdx.x];
    a.s.thresh[(q * 2 + threadIdx.x) * 2 + 1] = above_s[threadIdx.x];
  }
  __syncthreads();
  const int64_t j0 = (int64_t)c * kChunk;
  const int32_t j1 = (int32_t)(j0 + kChunk < (int64_t)n ? j0 + kChunk : (int64_t)n);
  const int32_t* sc = a.v.scores + (int64_t)q * a.v.ld;
  const int lane = threadIdx.x & 31;
  uint32_t mine[2] = {0, 0};
  for (int64_t base = j0; base < j1; base += blockDim.x) {
    const int32_t j = (int32_t)base + threadIdx.x;
    const bool in = j < j1;
    int32_t s = 0;
    if (in) {
      s = __ldg(sc + j);
      if (a.v.cand_pos && j > 0 && j < n) {
        if (pos_of(a.v, q, j) <= pos_of(a.v, q, j - 1)) record_error(a.status, CSA2_ERR_ORDER);
      }
    }
    const int32_t b = in ? (int32_t)score_bucket(s) : -2;
    for (int t = 0; t < a.n_k; ++t) {
      if (b > b_s[t]) mine[t]++;
      const bool tie = in && b == b_s[t];
      const uint32_t m = __ballot_sync(0xffffffffu, tie);
      if (m) {
        uint32_t slot0 = 0;
        const int leader = __ffs(m) - 1;
        if (lane == leader) slot0 = atomicAdd(a.s.cand_cnt + q * 2 + t, (uint32_t)__popc(m));
        slot0 = __shfl_sync(0xffffffffu, slot0, leader);
        if (tie) {
          const uint32_t slot = slot0 + __popc(m & ((1u << lane) - 1u));
          if (slot < (uint32_t)a.s.cand_cap)
            a.s.cand[((int64_t)q * 2 + t) * a.s.cand_cap + slot] = key_of(s, j);
        }
      }
    }
  }
  for (int t = 0; t < a.n_k; ++t) {
    uint32_t x = mine[t];
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
    if (lane == 0 && x) atomicAdd(&cnt_s[t], x);
  }
  __syncthreads();
  if (threadIdx.x < a.n_k)
    a.s.chunk_cnt[((int64_t)q * 2 + threadIdx.x) * a.s.n_chunks + c] = cnt_s[threadIdx.x];
}

// ------------------------------------------------------------------ radix select
// Returns, to every thread of the block, the need-th largest (1-based) of the
// m distinct keys get(0..m-1).  The bits above the highest bit where the keys
// differ are common (AND == OR there).  Digits of at most 8 bits are fixed
// from there downwards.  The select stops early once every key under the fixed
// prefix is a member: kth is then the smallest of those keys.
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
    kand &= k;
    kor |= k;
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
  while (true) {
    const int lo = top >= 7 ? top - 7 : 0;
    const uint32_t dmask = (uint32_t)((2ull << (top - lo)) - 1ull);
    for (int i = threadIdx.x; i < 256; i += blockDim.x) hist256[i] = 0;
    __syncthreads();
    for (int64_t i = threadIdx.x; i < m; i += blockDim.x) {
      const uint64_t k = get(i);
      if ((k & fixed) == prefix) atomicAdd(&hist256[(uint32_t)(k >> lo) & dmask], 1u);
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
        if ((k & fixed) == prefix) atomicMin(&red[0], (unsigned long long)k);
      }
      __syncthreads();
      const uint64_t res = red[0];
      __syncthreads();
      return res;
    }
    top = lo - 1;
  }
}

// ------------------------------------------------------------------ resolve
struct ResolveArgs {
  CandView v;
  TopkScratch s;
  int32_t k[2];
};

constexpr int kResolveSmemKeys = kCandCap;

__global__ void __launch_bounds__(1024) topk_resolve_kernel(ResolveArgs a) {
  extern __shared__ uint64_t keys_s[];
  __shared__ uint32_t hist256[256];
  __shared__ unsigned long long red[2];
  const int q = blockIdx.x, t = blockIdx.y;
  const int32_t n = n_of(a.v, q);
  const int32_t k = a.k[t];
  const int32_t bstar = a.s.thresh[(q * 2 + t) * 2 + 0];
  const int32_t above = a.s.thresh[(q * 2 + t) * 2 + 1];
  uint32_t* ccnt = a.s.chunk_cnt + ((int64_t)q * 2 + t) * a.s.n_chunks;
  if (bstar < 0 || n <= k) {   // every candidate is a member
    if (threadIdx.x == 0) a.s.kth[q * 2 + t] = 0ull;
    return;
  }
  const int64_t need = (int64_t)k - above;
  const uint32_t m = a.s.cand_cnt[q * 2 + t];
  uint64_t kth;
  if (m <= (uint32_t)kResolveSmemKeys) {
    const uint64_t* src = a.s.cand + ((int64_t)q * 2 + t) * a.s.cand_cap;
    for (uint32_t i = threadIdx.x; i < m; i += blockDim.x) keys_s[i] = src[i];
    __syncthreads();
    kth = radix_select([&](int64_t i) { return keys_s[i]; }, m, need, hist256, red);
    for (uint32_t i = threadIdx.x; i < m; i += blockDim.x) {
      const uint64_t key = keys_s[i];
      if (key >= kth) atomicAdd(ccnt + (0xFFFFFFFFu - (uint32_t)key) / kChunk, 1u);
    }
  } else {
    // Overflowed candidate list (a very flat score distribution): select over
    // the whole score row, restricted to the threshold bucket.
    const int32_t* sc = a.v.scores + (int64_t)q * a.v.ld;
    auto get = [&](int64_t j) -> uint64_t {
      const int32_t s = __ldg(sc + j);
      return (int32_t)score_bucket(s) == bstar ? key_of(s, (int32_t)j) : 0ull;
    };
    // Keys outside the bucket map to 0, below every real key (a real key has
    // an index < 2^31 in its low half, so it is never 0).  need is at most the
    // bucket's count, so the need-th largest is always a real key.
    kth = radix_select(get, n, need, hist256, red);
    for (int64_t j = threadIdx.x; j < n; j += blockDim.x) {
      const uint64_t key = get(j);
      if (key != 0ull && key >= kth) atomicAdd(ccnt + j / kChunk, 1u);
    }
  }
  if (threadIdx.x == 0) a.s.kth[q * 2 + t] = kth;
}

// ------------------------------------------------------------------ write
struct WriteArgs {
  CandView v;
  TopkScratch s;
  TopkOut out[2];
  int32_t n_k;
};

__global__ void __launch_bounds__(256) topk_write_kernel(WriteArgs a) {
  __shared__ int32_t tmp[32];
  __shared__ int32_t base_s;
  const int q = blockIdx.y, c = blockIdx.x;
  const int32_t n = n_of(a.v, q);
  const int32_t chunks_q = (int32_t)(((int64_t)n + kChunk - 1) / kChunk);
  for (int t = 0; t < a.n_k; ++t) {
    const TopkOut o = a.out[t];
    const uint32_t* ccnt = a.s.chunk_cnt + ((int64_t)q * 2 + t) * a.s.n_chunks;
    const uint64_t kth = a.s.kth[q * 2 + t];
    int32_t* dst = o.idx + (int64_t)q * o.k;
    const int32_t total = n < o.k ? n : o.k;
    if (c == (chunks_q > 0 ? chunks_q - 1 : 0)) {
      for (int32_t i = total + threadIdx.x; i < o.k; i += blockDim.x) dst[i] = -1;
      if (threadIdx.x == 0 && o.cnt) o.cnt[q] = total;
    }
    if (c >= chunks_q) continue;
    // members in earlier chunks
    int32_t part = 0;
    for (int i = threadIdx.x; i < c; i += blockDim.x) part += (int32_t)ccnt[i];
    int32_t sum;
    block_excl_scan(part, tmp, &sum);
    if (threadIdx.x == 0) base_s = sum;
    __syncthreads();
    const int32_t base = base_s;
    // this chunk: 16 consecutive candidates per thread, in index order
    const int32_t j0 = c * kChunk + threadIdx.x * (kChunk / 256);
    const int32_t* sc = a.v.scores + (int64_t)q * a.v.ld;
    uint32_t flags = 0;
    int32_t cnt = 0;
#pragma unroll
    for (int i = 0; i < kChunk / 256; ++i) {
      const int32_t j = j0 + i;
      if (j < n && key_of(__ldg(sc + j), j) >= kth) {
        flags |= 1u << i;
        ++cnt;
      }
    }
    const int32_t off = block_excl_scan(cnt, tmp, nullptr);
    int32_t w = base + off;
#pragma unroll
    for (int i = 0; i < kChunk / 256; ++i) {
      if (flags & (1u << i)) {
        if (w < o.k) dst[w] = pos_of(a.v, q, j0 + i);
        ++w;
      }
    }
    __syncthreads();
  }
}

// ------------------------------------------------------------------ small: one CTA per query
struct SmallArgs {
  CandView v;
  int32_t k;
  int32_t* out_idx;
  int32_t* out_cnt;
  int32_t* status;
};

__global__ void __launch_bounds__(1024) topk_small_kernel(SmallArgs a) {
  extern __shared__ uint64_t keys_s[];   // [n]
  __shared__ uint32_t hist256[256];
  __shared__ unsigned long long red[2];
  __shared__ int32_t tmp[32];
  const int q = blockIdx.x;
  const int32_t n = n_of(a.v, q);
  const int32_t k = a.k;
  int32_t* dst = a.out_idx + (int64_t)q * k;
  const int32_t total = n < k ? n : k;
  const int32_t* sc = a.v.scores + (int64_t)q * a.v.ld;
  for (int32_t j = threadIdx.x; j < n; j += blockDim.x) {
    keys_s[j] = key_of(__ldg(sc + j), j);
    if (a.v.cand_pos && j > 0 && pos_of(a.v, q, j) <= pos_of(a.v, q, j - 1))
      record_error(a.status, CSA2_ERR_ORDER);
  }
  __syncthreads();
  uint64_t kth = 0ull;
  if (n > k) kth = radix_select([&](int64_t i) { return keys_s[i]; }, n, k, hist256, red);
  // stable compaction: ceil(n / 1024) consecutive candidates per thread
  const int32_t per = (n + blockDim.x - 1) / blockDim.x;
  const int32_t j0 = threadIdx.x * per;
  int32_t cnt = 0;
  for (int32_t i = 0; i < per; ++i) {
    const int32_t j = j0 + i;
    if (j < n && keys_s[j] >= kth) ++cnt;
  }
  int32_t w = block_excl_scan(cnt, tmp, nullptr);
  for (int32_t i = 0; i < per; ++i) {
    const int32_t j = j0 + i;
    if (j < n && keys_s[j] >= kth) {
      if (w < k) dst[w] = pos_of(a.v, q, j);
      ++w;
    }
  }
  for (int32_t i = total + threadIdx.x; i < k; i += blockDim.x) dst[i] = -1;
  if (threadIdx.x == 0 && a.out_cnt) a.out_cnt[q] = total;
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
  if (!hist_ready) {
    e = cudaMemsetAsync(s.hist, 0, (size_t)nq * kBuckets * sizeof(uint32_t), st);
    if (e != cudaSuccess) return e;
    topk_hist_kernel<<<grid, 256, 0, st>>>(v, s.hist);
  }
  e = cudaMemsetAsync(s.cand_cnt, 0, (size_t)nq * 2 * sizeof(uint32_t), st);
  if (e != cudaSuccess) return e;
  SelectArgs sa{v, s, {outs[0].k, n_k > 1 ? outs[1].k : 0}, n_k, status};
  topk_select_kernel<<<grid, 256, 0, st>>>(sa);
  static unsigned long long done = 0;
  e = ensure_smem(topk_resolve_kernel, kResolveSmemKeys * 8, done);
  if (e != cudaSuccess) return e;
  ResolveArgs ra{v, s, {outs[0].k, n_k > 1 ? outs[1].k : 0}};
  topk_resolve_kernel<<<dim3(nq, n_k), 1024, kResolveSmemKeys * 8, st>>>(ra);
  WriteArgs wa{v, s, {outs[0], n_k > 1 ? outs[1] : outs[0]}, n_k};
  topk_write_kernel<<<grid, 256, 0, st>>>(wa);
  return cudaGetLastError();
}

cudaError_t launch_topk_small(const int32_t* scores, int64_t ld, const int32_t* n_valid,
                              const int32_t* cand_pos, int32_t nq, int32_t n_max, int32_t k,
                              int32_t* out_idx, int32_t* out_cnt, int32_t* status,
                              cudaStream_t st) {
  static unsigned long long done = 0;
  cudaError_t e = ensure_smem(topk_small_kernel, kSmallMax * 8, done);
  if (e != cudaSuccess) return e;
  CandView v{scores, ld, n_valid, nullptr, cand_pos, n_max};
  SmallArgs sa{v, k, out_idx, out_cnt, status};
  const size_t smem = (size_t)(n_max > 0 ? n_max : 1) * 8;
  topk_small_kernel<<<nq, 1024, smem, st>>>(sa);
  return cudaGetLastError();
}

}  // namespace csa2
