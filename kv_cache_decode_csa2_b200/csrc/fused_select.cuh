// The pool select fused into the tail of the full-mode index-score kernel
// (K1) for one query: after the key stream, the kernel's own persistent CTAs
// (one per SM, all resident) find the top-P pool and the layer's top-K
// selection of the scores they have just written, with no further launch.
//
// The pool is the P best positions of the full-mode scores and the full
// layer's selection the K best ("DeepSeek V4.1-Flash: 552B runs like 16B",
// Act 2: a candidate pool of about 16K, then 512 of it).  Ties go to the
// lower position; outputs ascend.
//
// Same-address global atomics serialise (tens of ns each), so every exchange
// here goes through per-CTA slots and a bounded grid barrier instead:
//   1. every CTA stores its 13-bit bucket histogram (built in shared memory
//      during the stream) as one row; barrier;
//   2. CTA b sums bucket slice b over all rows; barrier;
//   3. every CTA finds, for each target, the slice and then the bucket b*
//      that holds the k-th best score, classifies its own scores (above b*,
//      tie at b*) and publishes its counts and tie keys; barrier;
//   4. when a target's ties must be split, every CTA gathers the tie keys of
//      all CTAs and ranks its own against them (or, when one CTA holds more
//      tie keys than its slot, the grid runs a radix select of the need-th
//      tie key), publishes its tie-member count; barrier;
//   5. the counts of the CTAs before it give every CTA its output offset; it
//      writes its members in position order (a CTA owns one contiguous range
//      of positions).
#pragma once

#include "csa2_device.cuh"
#include "select_common.cuh"

namespace csa2 {

constexpr int kFsOwnCap = 256;    // tie keys one CTA publishes per target
constexpr int kFsGather = 4096;   // tie keys gathered into every CTA for the exact rank
constexpr int kFsMaxG = 256;      // CTAs the scratch is sized for
constexpr unsigned long long kNoTie = ~0ull;   // "no tie of this CTA is a member" (no key is ~0 here)

struct FusedSel {
  int32_t on;           // 1: select after the stream (one query, one CTA per SM)
  int32_t n_k;          // targets: 1 or 2 (k[0] >= k[1])
  int32_t k[2];
  int32_t* out_idx[2];  // [k[t]] ascending, -1 padded
  int32_t* out_cnt[2];  // [1] or nullptr
  uint32_t* hrows;      // [kFsMaxG][kBuckets]   per-CTA histograms
  uint32_t* red;        // [kBuckets]            the summed histogram
  uint32_t* stot;       // [kFsMaxG]             slice totals
  uint32_t* cnts;       // [kFsMaxG][2][4]       above, ties, tie members per target
  uint64_t* tkeys;      // [kFsMaxG][2][kFsOwnCap]
  uint32_t* radix;      // [2][8][256]           zero before the launch
  uint32_t* bar;        // grid barrier count:   zero before the launch
};

// Global scratch of the fused select inside the index workspace.
inline size_t fused_sel_bytes() {
  return (size_t)kFsMaxG * kBuckets * 4 + (size_t)kBuckets * 4 + (size_t)kFsMaxG * 4 +
         (size_t)kFsMaxG * 2 * 4 * 4 + (size_t)kFsMaxG * 2 * kFsOwnCap * 8 + 2 * 8 * 256 * 4 + 6 * 256;
}

// Runs in every thread of every CTA of the index-score launch after its
// stream.  NT threads per CTA; `hist_s` is the CTA's bucket histogram in
// shared memory; `ring` is free shared memory of MAXP * 4 + kFsGather * 8
// bytes; positions [p_lo, p_hi) are this CTA's (scores already in
// a_scores).
// `mark(p)` records trace point p (a no-op outside the traced build).
template <int NT, int MAXP, class Mark>
__device__ __forceinline__ void fused_select(const FusedSel& f, const int32_t* a_scores, uint32_t* hist_s,
                                             uint8_t* ring, int32_t p_lo, int32_t p_hi, int32_t* status,
                                             Mark mark) {
  static_assert(NT % 32 == 0 && NT >= kFsMaxG, "one thread per CTA slot in the scans");
  __shared__ uint64_t fwtmp[NT / 32];
  __shared__ int32_t bstar_s[2], above_s[2], slice_s[2], sabove_s[2];
  __shared__ uint32_t own_n[2], tm_s[2];
  __shared__ unsigned long long kmin_s[2], rprefix_s;
  __shared__ int32_t rneed_s;
  __shared__ uint32_t pre_s[kFsMaxG];
  __shared__ uint64_t off_s;
  const int G = gridDim.x, b = blockIdx.x, tid = threadIdx.x;
  const int lane = tid & 31, warp = tid >> 5;
  const int32_t n = p_hi > p_lo ? p_hi - p_lo : 0;
  int32_t* sc_s = reinterpret_cast<int32_t*>(ring);                        // [MAXP] this CTA's scores
  uint64_t* gath = reinterpret_cast<uint64_t*>(ring + (size_t)MAXP * 4);   // [kFsGather]
  uint32_t* part_s = hist_s;                                               // after its row is stored
  uint64_t* own = reinterpret_cast<uint64_t*>(hist_s + 4096);              // [2][kFsOwnCap]
  uint32_t* dh = hist_s + 4096 + 4 * kFsOwnCap;                            // [256] digit counts
  uint32_t phase = 0;

  pdl_wait();   // the zeroed counts come from the grid before (complete long ago)
  if (tid < 2) {
    bstar_s[tid] = -1;
    above_s[tid] = 0;
    own_n[tid] = 0;
    tm_s[tid] = 0;
    kmin_s[tid] = ~0ull;
  }
  // ---- 1. this CTA's histogram row, and its scores into shared memory
  {
    const uint4* src = reinterpret_cast<const uint4*>(hist_s);
    uint4* dst = reinterpret_cast<uint4*>(f.hrows + (size_t)b * kBuckets);
    for (int i = tid; i < kBuckets / 4; i += NT) dst[i] = src[i];
    // the scores, 8 independent loads in flight per thread (an L2 round trip
    // costs about half a microsecond, so loads must not wait on each other)
    for (int base = 0; base < n; base += 8 * NT) {
      int32_t v[8];
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        const int i = base + u * NT + tid;
        v[u] = i < n ? __ldcg(a_scores + p_lo + i) : 0;
      }
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        const int i = base + u * NT + tid;
        if (i < n) sc_s[i] = v[u];
      }
    }
  }
  sel_grid_sync(f.bar, ++phase * G, status);
  mark(11);

  // ---- 2. slice b of the summed histogram
  const int BS = (kBuckets + G - 1) / G;
  {
    // every (row, bucket) pair of the slice is one load; 8 independent loads
    // per thread per round, added into the slice's counts in shared memory
    for (int j = tid; j < BS; j += NT) part_s[j] = 0u;
    __syncthreads();
    const int items = G * BS;
    for (int base = 0; base < items; base += 8 * NT) {
      uint32_t v[8];
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        const int it = base + u * NT + tid;
        const int c = it / BS, j = it - c * BS, bk = b * BS + j;
        v[u] = (it < items && bk < kBuckets) ? __ldcg(f.hrows + (size_t)c * kBuckets + bk) : 0u;
      }
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        const int it = base + u * NT + tid;
        if (v[u]) atomicAdd(&part_s[it - (it / BS) * BS], v[u]);
      }
    }
    __syncthreads();
    uint32_t local = 0;
    for (int j = tid; j < BS; j += NT) {
      const uint32_t v = part_s[j];
      if (b * BS + j < kBuckets) {
        f.red[b * BS + j] = v;
        local += v;
      }
    }
    uint64_t tot;
    sel_scan<NT>(local, fwtmp, &tot);
    if (tid == 0) f.stot[b] = (uint32_t)tot;
  }
  sel_grid_sync(f.bar, ++phase * G, status);
  mark(12);

  // ---- 3. thresholds: the slice holding the k-th best score, then the bucket
  {
    const uint32_t v = tid < G ? __ldcg(f.stot + (G - 1 - tid)) : 0u;   // thread 0: the top slice
    uint64_t total64;
    const uint64_t ex = sel_scan<NT>(v, fwtmp, &total64);
#pragma unroll
    for (int t = 0; t < 2; ++t) {
      if (tid == 0) slice_s[t] = -1;
      __syncthreads();
      const int64_t k = f.k[t];
      if (t < f.n_k && (int64_t)total64 > k && (int64_t)ex < k && (int64_t)(ex + v) >= k) {
        slice_s[t] = G - 1 - tid;
        sabove_s[t] = (int32_t)ex;
      }
      __syncthreads();
      const int sl = slice_s[t];
      if (sl >= 0) {   // block-uniform
        const int per = (BS + NT - 1) / NT;   // buckets per thread, thread 0 the highest
        uint32_t hs = 0;
        for (int i = 0; i < per; ++i) {
          const int j = BS - 1 - (tid * per + i);
          const int bk = sl * BS + j;
          if (j >= 0 && bk < kBuckets) hs += __ldcg(f.red + bk);
        }
        uint64_t st;
        const uint64_t sx = sel_scan<NT>(hs, fwtmp, &st);
        const int64_t kk = k - sabove_s[t];
        if ((int64_t)sx < kk && (int64_t)(sx + hs) >= kk) {
          int64_t run = (int64_t)sx;
          for (int i = 0; i < per; ++i) {
            const int j = BS - 1 - (tid * per + i);
            const int bk = sl * BS + j;
            if (j < 0 || bk >= kBuckets) continue;
            const uint32_t c = __ldcg(f.red + bk);
            if (run + c >= kk) {
              bstar_s[t] = bk;
              above_s[t] = sabove_s[t] + (int32_t)run;
              break;
            }
            run += c;
          }
        }
      }
      __syncthreads();
    }
  }

  mark(13);
  // ---- classify this CTA's scores; publish counts and tie keys
  {
    uint32_t ab[2] = {0u, 0u};
    const int32_t b0 = bstar_s[0], b1 = f.n_k > 1 ? bstar_s[1] : INT32_MIN;
    for (int i = tid; i < n; i += NT) {
      const int32_t s = sc_s[i];
      const int32_t bk = (int32_t)score_bucket(s);
#pragma unroll
      for (int t = 0; t < 2; ++t) {
        const int32_t bs = t ? b1 : b0;
        if (bk > bs) ++ab[t];
        else if (bk == bs) {
          const uint32_t slot = atomicAdd(&own_n[t], 1u);
          if (slot < (uint32_t)kFsOwnCap) own[t * kFsOwnCap + slot] = cand_key(s, p_lo + i);
        }
      }
    }
    uint64_t tot;
    sel_scan<NT>((uint64_t)ab[0] | ((uint64_t)ab[1] << 32), fwtmp, &tot);
    uint32_t* mine = f.cnts + (size_t)b * 8;
#pragma unroll
    for (int t = 0; t < 2; ++t) {
      const uint32_t m = own_n[t] < (uint32_t)kFsOwnCap ? own_n[t] : (uint32_t)kFsOwnCap;
      for (uint32_t i = tid; i < m; i += NT)
        f.tkeys[((size_t)b * 2 + t) * kFsOwnCap + i] = own[t * kFsOwnCap + i];
      if (tid == 0) {
        mine[t * 4 + 0] = (uint32_t)(tot >> (32 * t));
        mine[t * 4 + 1] = own_n[t];
      }
    }
  }
  sel_grid_sync(f.bar, ++phase * G, status);
  mark(14);

  // ---- 4. ties: split where needed
  bool any_split = false;
  bool split[2] = {false, false};
  // kthr[t]: own ties with keys >= kthr[t] are members (0: every tie; kNoTie: none)
  uint64_t kthr[2] = {0ull, 0ull};
#pragma unroll
  for (int t = 0; t < 2; ++t) {
    if (t >= f.n_k || bstar_s[t] < 0) continue;
    // every CTA's tie count (thread c reads CTA c's)
    const uint32_t tc = tid < G ? __ldcg(f.cnts + (size_t)tid * 8 + t * 4 + 1) : 0u;
    uint64_t T64;
    sel_scan<NT>(tc, fwtmp, &T64);
    const bool over = __syncthreads_or(tc > (uint32_t)kFsOwnCap) != 0;
    const int32_t need = f.k[t] - above_s[t];
    if ((int64_t)T64 <= need) continue;   // every tie is a member
    split[t] = any_split = true;
    if (!over && T64 <= (uint64_t)kFsGather) {
      // gather the tie keys of all CTAs (CTA c's at [its prefix, + count))
      uint64_t dummy;
      const uint64_t px = sel_scan<NT>(tc, fwtmp, &dummy);
      if (tid < G) pre_s[tid] = (uint32_t)px;
      __syncthreads();
      // key g of the list comes from the CTA c with pre_s[c] <= g < pre_s[c + 1];
      // all loads of a round are independent
      const uint32_t T = (uint32_t)T64;
      for (uint32_t base = 0; base < T; base += 8 * NT) {
        uint64_t v[8];
#pragma unroll
        for (int u = 0; u < 8; ++u) {
          const uint32_t g = base + u * NT + tid;
          v[u] = 0ull;
          if (g < T) {
            int lo_c = 0, hi_c = G - 1;   // last CTA whose prefix is <= g
            while (lo_c < hi_c) {
              const int mid = (lo_c + hi_c + 1) >> 1;
              if (pre_s[mid] <= g) lo_c = mid;
              else hi_c = mid - 1;
            }
            v[u] = __ldcg(f.tkeys + ((size_t)lo_c * 2 + t) * kFsOwnCap + (g - pre_s[lo_c]));
          }
        }
#pragma unroll
        for (int u = 0; u < 8; ++u) {
          const uint32_t g = base + u * NT + tid;
          if (g < T) gath[g] = v[u];
        }
      }
      __syncthreads();   // the whole list is in place before any rank is taken
      const uint32_t mine = own_n[t];
      for (uint32_t i = warp; i < mine; i += NT / 32) {
        const uint64_t ki = own[t * kFsOwnCap + i];
        uint32_t r = 0;
        for (uint32_t j = lane; j < T; j += 32) r += gath[j] > ki;
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) r += __shfl_xor_sync(0xffffffffu, r, o);
        if (lane == 0 && (int32_t)r < need) {
          atomicAdd(&tm_s[t], 1u);
          atomicMin(&kmin_s[t], (unsigned long long)ki);
        }
      }
      __syncthreads();
      kthr[t] = tm_s[t] ? kmin_s[t] : kNoTie;
    } else {
      // radix select of the need-th tie key over the grid: one 8-bit digit of
      // the 64-bit key per pass, digit counts summed in global memory
      const int32_t bs = bstar_s[t];
      if (tid == 0) {
        rprefix_s = 0ull;
        rneed_s = need;
      }
      unsigned long long mask = 0ull;
#pragma unroll 1
      for (int pass = 0; pass < 8; ++pass) {
        const int shift = 56 - 8 * pass;
        for (int d = tid; d < 256; d += NT) dh[d] = 0u;
        __syncthreads();
        const unsigned long long prefix = rprefix_s;
        for (int i = tid; i < n; i += NT) {
          const int32_t s = sc_s[i];
          if ((int32_t)score_bucket(s) != bs) continue;
          const uint64_t key = cand_key(s, p_lo + i);
          if ((key & mask) == prefix) atomicAdd(&dh[(key >> shift) & 255u], 1u);
        }
        __syncthreads();
        uint32_t* gd = f.radix + ((size_t)t * 8 + pass) * 256;
        for (int d = tid; d < 256; d += NT)
          if (dh[d]) atomicAdd(gd + d, dh[d]);
        const int32_t nd = rneed_s;
        sel_grid_sync(f.bar, ++phase * G, status);
        const uint32_t v = tid < 256 ? __ldcg(gd + 255 - tid) : 0u;   // thread 0: the highest digit
        uint64_t dt;
        const uint64_t dx = sel_scan<NT>(v, fwtmp, &dt);
        if (tid < 256 && (int64_t)dx < nd && (int64_t)(dx + v) >= nd) {
          rprefix_s = prefix | ((unsigned long long)(255 - tid) << shift);
          rneed_s = nd - (int32_t)dx;
        }
        __syncthreads();
        mask |= 0xFFull << shift;
      }
      kthr[t] = rprefix_s;   // the need-th best tie key, exactly
      uint32_t m = 0;
      for (int i = tid; i < n; i += NT) {
        const int32_t s = sc_s[i];
        if ((int32_t)score_bucket(s) == bs && cand_key(s, p_lo + i) >= kthr[t]) ++m;
      }
      uint64_t mt;
      sel_scan<NT>(m, fwtmp, &mt);
      if (tid == 0) tm_s[t] = (uint32_t)mt;
      __syncthreads();
    }
    if (tid == 0) f.cnts[(size_t)b * 8 + t * 4 + 2] = tm_s[t];
  }
  if (any_split) sel_grid_sync(f.bar, ++phase * G, status);   // grid-uniform
  mark(15);

  // ---- 5. offsets from the CTAs before, then the members in position order
  uint64_t off = 0, grand = 0;   // packed: target 0 low, target 1 high
  {
    uint64_t mine_cnt = 0;
    if (tid < G) {
      const uint32_t* cc = f.cnts + (size_t)tid * 8;
#pragma unroll
      for (int t = 0; t < 2; ++t) {
        if (t >= f.n_k) break;
        uint32_t m = __ldcg(cc + t * 4 + 0);
        if (bstar_s[t] >= 0) m += split[t] ? __ldcg(cc + t * 4 + 2) : __ldcg(cc + t * 4 + 1);
        mine_cnt |= (uint64_t)m << (32 * t);
      }
    }
    const uint64_t ex = sel_scan<NT>(mine_cnt, fwtmp, &grand);
    if (tid == b) off_s = ex;
    __syncthreads();
    off = off_s;
  }
  {
    const int32_t b0 = bstar_s[0], b1 = f.n_k > 1 ? bstar_s[1] : INT32_MIN;
    const int R = (n + NT - 1) / NT;   // positions per thread, contiguous
    const int i0 = tid * R, i1 = i0 + R < n ? i0 + R : n;
    uint64_t cnt = 0;
    for (int i = i0; i < i1; ++i) {
      const int32_t s = sc_s[i];
      const int32_t bk = (int32_t)score_bucket(s);
      const uint64_t key = cand_key(s, p_lo + i);
      const bool m0 = bk > b0 || (bk == b0 && kthr[0] != kNoTie && key >= kthr[0]);
      const bool m1 = f.n_k > 1 && (bk > b1 || (bk == b1 && kthr[1] != kNoTie && key >= kthr[1]));
      cnt += (uint64_t)m0 | ((uint64_t)m1 << 32);
    }
    uint64_t dummy;
    const uint64_t ex = sel_scan<NT>(cnt, fwtmp, &dummy) + off;
    int64_t at[2] = {(int64_t)(ex & 0xffffffffu), (int64_t)(ex >> 32)};
    for (int i = i0; i < i1; ++i) {
      const int32_t s = sc_s[i];
      const int32_t bk = (int32_t)score_bucket(s);
      const uint64_t key = cand_key(s, p_lo + i);
#pragma unroll
      for (int t = 0; t < 2; ++t) {
        if (t >= f.n_k) break;
        const int32_t bs = t ? b1 : b0;
        if (bk > bs || (bk == bs && kthr[t] != kNoTie && key >= kthr[t])) {
          if (at[t] < f.k[t]) f.out_idx[t][at[t]] = p_lo + i;
          ++at[t];
        }
      }
    }
    if (b == G - 1) {
#pragma unroll
      for (int t = 0; t < 2; ++t) {
        if (t >= f.n_k) break;
        const int64_t g = (int64_t)((grand >> (32 * t)) & 0xffffffffu);
        const int32_t c = g < f.k[t] ? (int32_t)g : f.k[t];
        for (int32_t i = c + tid; i < f.k[t]; i += NT) f.out_idx[t][i] = -1;
        if (tid == 0 && f.out_cnt[t]) f.out_cnt[t][0] = c;
      }
    }
  }
}

}  // namespace csa2
