// Row select: exact top-k of many long score rows, one CTA per row.
//
// The top-k of every query of a prefill chunk is taken over its whole causal
// prefix (there is no pool), so a chunk of 2048 queries at a 262,144-row
// context has 2048 rows of up to 262,144 candidates: far more rows than the
// select kernel can hold co-resident.  Here one CTA of kRowNT threads takes a
// row, and thread t owns the candidates [t R, t R + R), R <= kRowPer:
//   pass 1  bucket histogram of the row in shared memory, counting only
//           candidates at or above a cut that a small sample of the row
//           picks (with a full-histogram redo should too few clear it); one
//           block scan finds the threshold bucket b* of each target.  Each
//           thread also keeps its first kRowKeep candidates at or above the
//           cut (score and offset) in shared memory;
//   pass 2  when no thread kept more than kRowKeep, every member is among
//           the kept candidates (b* is at or above the cut), and the ties at
//           b* come from them; otherwise the row is read again into
//           per-thread bitmasks of the members above b* and of the ties.
//           The ties go to a shared list, each warp ranks some of them
//           against it, and this gives the smallest member tie key;
//   write   one packed block scan of the member counts gives every thread
//           its first output slot; the members are written in position
//           order from the kept list or the bitmasks.
// A row reads its scores once when the cut is selective (about 2.5
// candidates per thread clear it for a top-512 of 262,144), else twice.  A
// tie list longer than kRowTieCap (a very flat score distribution) is
// resolved by a radix select of the k-th tie key, one 8-bit digit per pass
// over the row.
#include "csa2_device.cuh"
#include "internal.h"
#include "select_common.cuh"

namespace csa2 {

CSA2_TRACE_UNIT(rows)

namespace {

constexpr int kRowNT = 1024;
constexpr int kRowWords = kRowPer / 32;   // bitmask words per thread and target
constexpr int kRowTieCap = 4096;
constexpr int kRowKeep = 16;               // kept candidates per thread
static_assert(kRowPer % 32 == 0 && kBuckets / kRowNT == 8, "shapes");
static_assert(kRowPer <= 256, "a kept candidate's offset is one byte");

struct RowArgs {
  const int32_t* scores;
  int64_t ld;
  const int32_t* n_valid;
  const int32_t* query_pos;
  const int32_t* cand_pos;
  int32_t n_max;
  int32_t n_k;
  int32_t k[2];
  int32_t* out_idx[2];
  int32_t* out_cnt[2];
  int32_t* status;
};

__device__ __forceinline__ int32_t row_n(const RowArgs& a, int q) {
  if (a.n_valid) {
    const int32_t n = __ldg(a.n_valid + q);
    return n < 0 ? 0 : (n > a.n_max ? a.n_max : n);
  }
  if (a.query_pos) {
    const int32_t p = __ldg(a.query_pos + q);
    return (p < 0 || p >= a.n_max) ? 0 : p + 1;
  }
  return a.n_max;
}

template <int NK>   // targets: 1, or 2 (a pool and a selection)
__global__ void __launch_bounds__(kRowNT, 1) row_select_kernel(const __grid_constant__ RowArgs a) {
  extern __shared__ __align__(16) unsigned char row_dyn[];
  uint32_t* hist = reinterpret_cast<uint32_t*>(row_dyn);                      // [kBuckets]
  uint64_t* ties = reinterpret_cast<uint64_t*>(row_dyn + kBuckets * 4);       // [2][kRowTieCap]
  int32_t* keep_s = reinterpret_cast<int32_t*>(ties + 2 * kRowTieCap);        // [kRowKeep][kRowNT]
  uint8_t* keep_o = reinterpret_cast<uint8_t*>(keep_s + kRowKeep * kRowNT);   // [kRowKeep][kRowNT]
  __shared__ uint64_t wtmp[32];
  __shared__ int32_t bstar_s[2], above_s[2];
  __shared__ uint32_t nt_s[2];
  __shared__ unsigned long long kthr_s[2];
  __shared__ uint32_t dig[256];
  __shared__ unsigned long long prefix_s;
  __shared__ int32_t rem_s;

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int q = blockIdx.x;
  constexpr int n_k = NK;
  // trace points: 1 threshold buckets, 2 score bounds, 3 classified, 4 ties
  // resolved, 5 written
  CSA2_TRACE_BEGIN(kTrRowSel, tid == 0);
  const int32_t n = row_n(a, q);
  const int32_t R = (((n + kRowNT - 1) / kRowNT) + 3) & ~3;   // candidates per thread, a multiple of 4
  const int32_t j0 = tid * R;
  const int32_t j1 = j0 + R < n ? j0 + R : n;
  const int32_t* row = a.scores + (int64_t)q * a.ld;
  const bool vec = (reinterpret_cast<uintptr_t>(row) & 15) == 0;
  if (tid < 2) {
    bstar_s[tid] = -1;
    above_s[tid] = 0;
    nt_s[tid] = 0;
    kthr_s[tid] = ~0ull;
  }
  // Calls f(j, score) for this thread's candidates, four at a time where aligned.
  auto for_own = [&](auto&& f) {
    int32_t j = j0;
    if (vec) {
      for (; j + 4 <= j1; j += 4) {
        const int4 v = __ldcg(reinterpret_cast<const int4*>(row + j));
        f(j, v.x);
        f(j + 1, v.y);
        f(j + 2, v.z);
        f(j + 3, v.w);
      }
    }
    for (; j < j1; ++j) f(j, __ldcg(row + j));
  };

  // ---- pass 1: histogram, threshold buckets.  A sample (each thread's first
  // 8 candidates) picks a lower cut that about four times the wanted count
  // clears; the exact histogram then counts only candidates at or above it,
  // which spares most shared-memory atomics.  Should fewer than k candidates
  // clear the cut, the full histogram is built instead.
  __shared__ int32_t cut_s;
  const int32_t kmax = n_k > 1 && a.k[1] > a.k[0] ? a.k[1] : a.k[0];
  auto zero_hist = [&]() {
    uint4* h4 = reinterpret_cast<uint4*>(hist + tid * 8);
    h4[0] = make_uint4(0, 0, 0, 0);
    h4[1] = make_uint4(0, 0, 0, 0);
  };
  // walks this thread's 8 bins for the bucket where the count above crosses
  // `want`; returns the block total
  auto scan_bins = [&](auto&& on_cross) -> int64_t {
    const uint4* h4 = reinterpret_cast<const uint4*>(hist + tid * 8);
    const uint4 h0 = h4[0], h1 = h4[1];
    const uint32_t hb[8] = {h0.x, h0.y, h0.z, h0.w, h1.x, h1.y, h1.z, h1.w};
    uint32_t hsum = 0;
#pragma unroll
    for (int b = 0; b < 8; ++b) hsum += hb[b];
    uint64_t total64;
    const uint64_t excl = sel_scan<kRowNT>(hsum, wtmp, &total64);
    const int64_t above_me = (int64_t)total64 - (int64_t)excl - hsum;
    on_cross(hb, above_me, hsum, (int64_t)total64);
    return (int64_t)total64;
  };
  zero_hist();
  if (tid == 0) cut_s = -1;
  __syncthreads();
  if (n > kmax) {   // the sample
    const int32_t m = j1 - j0 < 8 ? j1 - j0 : 8;
    int32_t v[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) v[e] = e < m ? __ldcg(row + j0 + e) : 0;
#pragma unroll
    for (int e = 0; e < 8; ++e)
      if (e < m) atomicAdd(&hist[score_bucket(v[e])], 1u);
  }
  __syncthreads();
  if (n > kmax) {
    scan_bins([&](const uint32_t (&hb)[8], int64_t above_me, uint32_t hsum, int64_t S) {
      const int64_t want = 4 * (int64_t)kmax * S / n + 16;   // S samples of n candidates
      if (above_me < want && above_me + hsum >= want) {
        int64_t acc = above_me;
#pragma unroll
        for (int b = 7; b >= 0; --b) {
          if (acc + hb[b] >= want) {
            cut_s = tid * 8 + b;
            break;
          }
          acc += hb[b];
        }
      }
    });
  }
  zero_hist();
  __shared__ int32_t cut_score_s;
  if (tid == 0) cut_score_s = bucket_min_score(cut_s);
  __syncthreads();
  const int32_t cut_score = cut_score_s;
  // candidates of this thread at or above the cut; the first kRowKeep are kept
  int32_t n_kept = 0;
  bool kept_all = true;   // the kept list holds every candidate at or above the cut
#pragma unroll 1
  for (int attempt = 0; attempt < 2; ++attempt) {
    const int32_t lo_s = attempt == 0 ? cut_score : INT32_MIN;   // count scores >= lo_s
    const bool keep = attempt == 0;
    auto count = [&](int32_t off, int32_t sv) {
      if (sv >= lo_s) {   // about one candidate in a hundred above a sampled cut
        atomicAdd(&hist[score_bucket(sv)], 1u);
        if (keep) {
          if (n_kept < kRowKeep) {
            keep_s[n_kept * kRowNT + tid] = sv;
            keep_o[n_kept * kRowNT + tid] = (uint8_t)off;
          }
          ++n_kept;
        }
      }
    };
    // words of 32 candidates; a word's eight loads are all issued before any is used
#pragma unroll 1
    for (int x = 0; x < kRowWords; ++x) {
      const int32_t base = j0 + 32 * x;
      if (base >= j1) break;
      if (vec && base + 32 <= j1) {
        int4 v[8];
#pragma unroll
        for (int u = 0; u < 8; ++u) v[u] = __ldcg(reinterpret_cast<const int4*>(row + base) + u);
#pragma unroll
        for (int u = 0; u < 8; ++u) {
          count(32 * x + 4 * u, v[u].x);
          count(32 * x + 4 * u + 1, v[u].y);
          count(32 * x + 4 * u + 2, v[u].z);
          count(32 * x + 4 * u + 3, v[u].w);
        }
      } else {
#pragma unroll 1
        for (int e = 0; e < 32 && base + e < j1; ++e) count(32 * x + e, __ldcg(row + base + e));
      }
    }
    if (attempt == 1) kept_all = false;   // the redo counted below the cut: the list is partial
    if (attempt == 0 && a.cand_pos) {   // candidate positions must ascend
      const int32_t* cp = a.cand_pos + (int64_t)q * a.ld;
      bool bad = false;
      for (int32_t j = j0 > 0 ? j0 : 1; j < j1; ++j) bad |= __ldg(cp + j) <= __ldg(cp + j - 1);
      if (bad) record_error(a.status, CSA2_ERR_ORDER);
    }
    __syncthreads();
    const int64_t total = scan_bins([&](const uint32_t (&hb)[8], int64_t above_me, uint32_t hsum, int64_t) {
#pragma unroll
      for (int t = 0; t < 2; ++t) {
        const int32_t k = a.k[t];
        if (t < n_k && n > k && above_me < k && above_me + hsum >= k) {
          int64_t acc = above_me;
#pragma unroll
          for (int b = 7; b >= 0; --b) {
            if (acc + hb[b] >= k) {
              bstar_s[t] = tid * 8 + b;
              above_s[t] = (int32_t)acc;
              break;
            }
            acc += hb[b];
          }
        }
      }
    });
    // the counted candidates must cover every target that is not "take all"
    bool short_of = false;
#pragma unroll
    for (int t = 0; t < 2; ++t)
      if (t < n_k && n > a.k[t] && total < a.k[t]) short_of = true;
    if (!short_of) break;
    zero_hist();
    if (tid < 2) {
      bstar_s[tid] = -1;
      above_s[tid] = 0;
    }
    __syncthreads();
  }
  // every member is kept when every thread kept all it counted above the cut
  const bool fast = __syncthreads_and(kept_all && n_kept <= kRowKeep) != 0;
  CSA2_MARK(kTrRowSel, 1, tid == 0);

  // ---- pass 2: members above b* and ties at b*, from the kept list or as bitmasks
  const int32_t b0 = bstar_s[0], b1 = n_k > 1 ? bstar_s[1] : INT32_MIN;
  // score ranges: above b* means s >= hi_t, at b* means lo_t <= s < hi_t
  // (64-bit: the bucket above the top one starts past every int32 score)
  __shared__ long long bound_s[4];
  if (tid < 4) {
    const int t = tid >> 1;
    const int32_t bs = bstar_s[t];
    const int32_t b = (tid & 1) ? bs + 1 : bs;
    bound_s[tid] = (t >= n_k || bs < 0) ? 0ll : b >= kBuckets ? (long long)INT32_MAX + 1 : bucket_min_score(b);
  }
  __syncthreads();
  CSA2_MARK(kTrRowSel, 2, tid == 0);
  const long long lo0 = bound_s[0], hi0 = bound_s[1], lo1 = bound_s[2], hi1 = bound_s[3];
  const bool all0 = b0 < 0, all1 = n_k > 1 && b1 < 0;
  // Word x of the bitmasks covers candidates j0 + 32 x .. j0 + 32 x + 31.  The
  // word loop stays rolled (this code runs once per row, from a cold
  // instruction cache): each word's masks come from branch-free comparisons
  // and are shifted into the register arrays, so that word x ends at index
  // kRowWords - 1 - x with every index a constant.
  uint32_t above_m[NK][kRowWords], tie_m[NK][kRowWords];
#pragma unroll
  for (int t = 0; t < NK; ++t)
#pragma unroll
    for (int w = 0; w < kRowWords; ++w) above_m[t][w] = tie_m[t][w] = 0u;
  auto add_tie = [&](int t, int32_t sv, int32_t j) {
    const uint32_t slot = atomicAdd(&nt_s[t], 1u);
    if (slot < (uint32_t)kRowTieCap) ties[t * kRowTieCap + slot] = cand_key(sv, j);
  };
  if (fast) {   // the kept candidates: offsets ascend with the slot
#pragma unroll 1
    for (int c = 0; c < n_kept; ++c) {
      const int32_t sv = keep_s[c * kRowNT + tid];
      const int32_t j = j0 + keep_o[c * kRowNT + tid];
      const long long sl = sv;
      if (!all0 && sl >= lo0 && sl < hi0) add_tie(0, sv, j);
      if constexpr (NK > 1)
        if (!all1 && sl >= lo1 && sl < hi1) add_tie(1, sv, j);
    }
  }
#pragma unroll 1
  for (int x = 0; x < (fast ? 0 : kRowWords); ++x) {
    const int32_t base = j0 + 32 * x;
    uint32_t am[NK], tm[NK];
#pragma unroll
    for (int t = 0; t < NK; ++t) am[t] = tm[t] = 0u;
    auto take = [&](int e, int32_t sv) {
      const long long s = sv;
      am[0] |= (uint32_t)(all0 || s >= hi0) << e;   // b* = -1 takes every candidate
      tm[0] |= (uint32_t)(!all0 && s >= lo0 && s < hi0) << e;
      if constexpr (NK > 1) {
        am[NK - 1] |= (uint32_t)(all1 || s >= hi1) << e;
        tm[NK - 1] |= (uint32_t)(!all1 && s >= lo1 && s < hi1) << e;
      }
    };
    if (base < j1) {
      if (vec && base + 32 <= j1) {
        int4 v[8];
#pragma unroll
        for (int u = 0; u < 8; ++u) v[u] = __ldcg(reinterpret_cast<const int4*>(row + base) + u);
#pragma unroll
        for (int u = 0; u < 8; ++u) {
          take(4 * u, v[u].x);
          take(4 * u + 1, v[u].y);
          take(4 * u + 2, v[u].z);
          take(4 * u + 3, v[u].w);
        }
      } else {
#pragma unroll 1
        for (int e = 0; e < 32 && base + e < j1; ++e) take(e, __ldcg(row + base + e));
      }
    }
#pragma unroll
    for (int t = 0; t < NK; ++t) {
#pragma unroll
      for (int w = kRowWords - 1; w > 0; --w) {
        above_m[t][w] = above_m[t][w - 1];
        tie_m[t][w] = tie_m[t][w - 1];
      }
      above_m[t][0] = am[t];
      tie_m[t][0] = tm[t];
    }
  }
  // the ties (few) go to the row's list; their scores are read again
  // (the masks are all zero on the kept-list path)
#pragma unroll
  for (int t = 0; t < NK; ++t) {
#pragma unroll
    for (int x = 0; x < kRowWords; ++x) {
      uint32_t tmk = tie_m[t][kRowWords - 1 - x];
      while (tmk) {
        const int b = __ffs(tmk) - 1;
        tmk &= tmk - 1u;
        const int32_t j = j0 + 32 * x + b;
        add_tie(t, __ldcg(row + j), j);
      }
    }
  }
  __syncthreads();
  CSA2_MARK(kTrRowSel, 3, tid == 0);
  // rank the ties: the members among them are those with fewer than need
  // better ties; the smallest such key is the threshold key
#pragma unroll
  for (int t = 0; t < 2; ++t) {
    const uint32_t nt = nt_s[t];
    if (bstar_s[t] < 0 || nt > (uint32_t)kRowTieCap) continue;
    const int32_t need = a.k[t] - above_s[t];
    const uint64_t* L = ties + t * kRowTieCap;
    for (uint32_t i = warp; i < nt; i += kRowNT / 32) {
      const uint64_t ki = L[i];
      uint32_t r = 0;
      for (uint32_t jj = lane; jj < nt; jj += 32) r += L[jj] > ki;
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) r += __shfl_xor_sync(0xffffffffu, r, o);
      if (lane == 0 && (int32_t)r < need) atomicMin(&kthr_s[t], (unsigned long long)ki);
    }
  }
  // very many ties: radix select of the need-th tie key, one digit per pass over the row
#pragma unroll 1
  for (int t = 0; t < 2; ++t) {
    if (bstar_s[t] < 0 || nt_s[t] <= (uint32_t)kRowTieCap) continue;
    const int32_t bst = bstar_s[t];
    uint64_t prefix = 0ull, fixed = 0ull;
    int32_t rem = a.k[t] - above_s[t];
    for (int pass = 0; pass < 8; ++pass) {
      const int shift = 56 - 8 * pass;
      if (tid < 256) dig[tid] = 0u;
      __syncthreads();
      for_own([&](int32_t j, int32_t s) {
        if ((int32_t)score_bucket(s) == bst) {
          const uint64_t key = cand_key(s, j);
          if ((key & fixed) == prefix) atomicAdd(&dig[(key >> shift) & 255u], 1u);
        }
      });
      __syncthreads();
      if (warp == 0) {   // lane l holds digits 255-8l .. 248-8l (lane 0: the highest)
        uint32_t d8[8], sum = 0;
#pragma unroll
        for (int u = 0; u < 8; ++u) {
          d8[u] = dig[255 - 8 * lane - u];
          sum += d8[u];
        }
        uint32_t incl = sum;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
          const uint32_t y = __shfl_up_sync(0xffffffffu, incl, o);
          if (lane >= o) incl += y;
        }
        const uint32_t before = incl - sum;
        if ((int64_t)before < rem && (int64_t)incl >= rem) {
          uint32_t acc = before;
#pragma unroll
          for (int u = 0; u < 8; ++u) {
            if ((int64_t)acc + d8[u] >= rem) {
              prefix_s = prefix | ((uint64_t)(255 - 8 * lane - u) << shift);
              rem_s = rem - (int32_t)acc;
              break;
            }
            acc += d8[u];
          }
        }
      }
      __syncthreads();
      prefix = prefix_s;
      rem = rem_s;
      fixed |= 255ull << shift;
      __syncthreads();
    }
    if (tid == 0) kthr_s[t] = prefix;
  }
  __syncthreads();
  CSA2_MARK(kTrRowSel, 4, tid == 0);

  // ---- members: ties at or above the threshold key join the bitmasks
  const uint64_t kthr[2] = {kthr_s[0], kthr_s[1]};
  uint32_t cnt[2] = {0u, 0u};
  // kept-list path: a member is above b*, or a tie whose key is at least the
  // threshold key (a target that takes every candidate kept them all)
  auto member = [&](int t, int32_t sv, int32_t j) -> bool {
    const long long sl = sv;
    if (t == 0) return all0 || sl >= hi0 || (sl >= lo0 && cand_key(sv, j) >= kthr[0]);
    return all1 || sl >= hi1 || (sl >= lo1 && cand_key(sv, j) >= kthr[1]);
  };
  if (fast) {
#pragma unroll 1
    for (int c = 0; c < n_kept; ++c) {
      const int32_t sv = keep_s[c * kRowNT + tid];
      const int32_t j = j0 + keep_o[c * kRowNT + tid];
#pragma unroll
      for (int t = 0; t < NK; ++t) cnt[t] += member(t, sv, j) ? 1u : 0u;
    }
  }
#pragma unroll
  for (int t = 0; t < NK; ++t) {
#pragma unroll
    for (int x = 0; x < kRowWords; ++x) {
      uint32_t tm = tie_m[t][kRowWords - 1 - x];
      while (tm) {   // ties are few: read their scores again
        const int b = __ffs(tm) - 1;
        tm &= tm - 1u;
        const int32_t j = j0 + x * 32 + b;
        if (cand_key(__ldcg(row + j), j) >= kthr[t]) above_m[t][kRowWords - 1 - x] |= 1u << b;
      }
      cnt[t] += __popc(above_m[t][kRowWords - 1 - x]);
    }
  }
  uint64_t tot;
  const uint64_t ex = sel_scan<kRowNT>((uint64_t)cnt[0] | ((uint64_t)cnt[1] << 32), wtmp, &tot);
  const int32_t* cp = a.cand_pos ? a.cand_pos + (int64_t)q * a.ld : nullptr;
#pragma unroll
  for (int t = 0; t < NK; ++t) {
    const int32_t k = a.k[t];
    int32_t* dst = a.out_idx[t] + (int64_t)q * k;
    int64_t slot = (int64_t)((ex >> (32 * t)) & 0xffffffffu);
    if (fast) {
#pragma unroll 1
      for (int c = 0; c < n_kept; ++c) {
        const int32_t sv = keep_s[c * kRowNT + tid];
        const int32_t j = j0 + keep_o[c * kRowNT + tid];
        if (member(t, sv, j)) {
          if (slot < k) dst[slot] = cp ? __ldg(cp + j) : j;
          ++slot;
        }
      }
    }
#pragma unroll
    for (int x = 0; x < kRowWords; ++x) {
      uint32_t m = above_m[t][kRowWords - 1 - x];
      while (m) {
        const int b = __ffs(m) - 1;
        m &= m - 1u;
        const int32_t j = j0 + x * 32 + b;
        if (slot < k) dst[slot] = cp ? __ldg(cp + j) : j;
        ++slot;
      }
    }
    const int64_t g = (int64_t)((tot >> (32 * t)) & 0xffffffffu);
    const int32_t c = g < k ? (int32_t)g : k;
    for (int32_t i = c + tid; i < k; i += kRowNT) dst[i] = -1;
    if (tid == 0 && a.out_cnt[t]) a.out_cnt[t][q] = c;
  }
  CSA2_MARK(kTrRowSel, 5, tid == 0);
}

constexpr int kRowSmem = kBuckets * 4 + 2 * kRowTieCap * 8 + kRowKeep * kRowNT * 5;

}  // namespace

cudaError_t launch_row_select(const int32_t* scores, int64_t ld, const int32_t* n_valid,
                              const int32_t* query_pos, const int32_t* cand_pos, int32_t nq, int32_t n_max,
                              const TopkOut* outs, int32_t n_k, int32_t* status, cudaStream_t st) {
  if (n_max > kRowSelMax || n_k < 1 || n_k > 2) return cudaErrorNotSupported;
  static SetupMask done1{0}, done2{0};
  cudaError_t e = n_k == 1 ? ensure_smem(row_select_kernel<1>, kRowSmem, done1)
                           : ensure_smem(row_select_kernel<2>, kRowSmem, done2);
  if (e != cudaSuccess) return e;
  RowArgs a{};
  a.scores = scores;
  a.ld = ld;
  a.n_valid = n_valid;
  a.query_pos = query_pos;
  a.cand_pos = cand_pos;
  a.n_max = n_max;
  a.n_k = n_k;
  for (int t = 0; t < 2; ++t) {
    const TopkOut& o = outs[t < n_k ? t : 0];
    a.k[t] = o.k;
    a.out_idx[t] = o.idx;
    a.out_cnt[t] = o.cnt;
  }
  a.status = status;
  if (n_k == 1) row_select_kernel<1><<<nq, kRowNT, kRowSmem, st>>>(a);
  else row_select_kernel<2><<<nq, kRowNT, kRowSmem, st>>>(a);
  return cudaGetLastError();
}

}  // namespace csa2
