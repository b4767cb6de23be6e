// Exact top-k of a score row, written in position order ("select").
//
// The pool of a decode step is the top-P positions of the full-mode index
// scores and the attended set is the top-K ("DeepSeek V4.1-Flash: 552B runs
// like 16B", Act 2: the indexer keeps a pool of about 16K candidates, later
// layers pick 512 from it).  Ties go to the lower position, so the result is
// unique: the candidates with the k largest keys (score, then ~position).
//
// One CTA of kSelNT threads covers kSelSpan consecutive candidates, kSelPer
// per thread, held in registers.  A row of n candidates takes G =
// ceil(n / kSelSpan) CTAs; for G > 1 they are co-resident (checked at
// launch) and meet at two grid barriers.
//   1. threshold bucket b* from the 13-bit bucket histogram of the row (given,
//      or built here when G == 1): every thread owns 8 bins, one block scan
//      gives the count above each thread's bins, and the thread whose bins
//      hold the k-th candidate walks them;
//   2. the ties (bucket == b*) of all CTAs form one list per row; each warp
//      ranks one of this CTA's ties against the whole list at a time.  A tie
//      is a member when fewer than need = k - (count above b*) ties beat it,
//      so this CTA's tie members are those at or above the smallest such key;
//   3. members are counted per thread; one block scan, plus for G > 1 the
//      counts of the CTAs before (published at the second barrier), gives
//      every member its output slot.
// A tie list longer than kSelTieCap (a very flat score distribution) is
// resolved instead by a radix select of the need-th tie key, one 8-bit digit
// of the 64-bit key per pass.
#include "csa2_device.cuh"
#include "internal.h"
#include "select_common.cuh"

namespace csa2 {

CSA2_TRACE_UNIT(select)

namespace {

constexpr int kBinsPer = kBuckets / kSelNT;
static_assert(kBinsPer == 8, "each thread owns 8 histogram bins");
static_assert(kSelNT == 1024, "the block scan assumes 32 warps");
constexpr int kSmemTies = 2 * kSelTieCap * 8;
static_assert(kBuckets * 4 <= kSmemTies, "the histogram shares room with the row's ties");
// this CTA's ties, then the row's ties (several CTAs) or the histogram (one CTA)
constexpr int kSelSmem = 2 * kSmemTies;

struct SelArgs {
  const int32_t* scores;
  int64_t ld;
  const int32_t* n_valid;
  const int32_t* query_pos;
  const int32_t* cand_pos;
  int32_t n_max;
  const uint32_t* hist;   // [nq][kBuckets] complete histograms, or nullptr (G == 1: built here)
  uint32_t* hdr;          // [nq][4]: barrier count, tie counts (zeroed before the launch; G > 1)
  uint64_t* ties;         // [nq][2][kSelTieCap]                                         (G > 1)
  uint32_t* mcnt;         // [nq][2][kSelMaxG] member counts per CTA                     (G > 1)
  uint32_t* radix;        // [nq][2][8][256] digit counts of the flat-distribution path  (G > 1)
  int32_t G;
  int32_t n_k;
  int32_t vec;            // rows start 16-byte aligned
  int32_t k[2];
  int32_t* out_idx[2];
  int32_t* out_cnt[2];
  int32_t* status;
};

__device__ __forceinline__ int32_t sel_n(const SelArgs& a, int q) {
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

// E candidates per thread (contiguous), kSelNT * E per CTA.
template <int E>
__global__ void __launch_bounds__(kSelNT, 1) select_kernel(const __grid_constant__ SelArgs a) {
  static_assert(E % 4 == 0 && E <= 32, "E: whole int4 loads, one bit per candidate in a word");
  constexpr int kSpan = kSelNT * E;
  extern __shared__ __align__(16) unsigned char sel_dyn[];
  uint64_t* own = reinterpret_cast<uint64_t*>(sel_dyn);   // [2][kSelTieCap]
  uint64_t* rowties = own + 2 * kSelTieCap;                // [2][kSelTieCap]
  uint32_t* hist = reinterpret_cast<uint32_t*>(rowties);
  __shared__ uint64_t wtmp[32];
  __shared__ int32_t bstar_s[2], above_s[2];
  __shared__ uint32_t own_cnt[2], gbase_s[2], nt_s[2];
  __shared__ unsigned long long kthr_s[2];
  __shared__ RadixSmem rsm;
  __shared__ uint64_t off_s, grand_s;

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int q = blockIdx.y, c = blockIdx.x, G = a.G, n_k = a.n_k;
  const int32_t j0 = c * kSpan + tid * E;
  // trace points: 1 grid before done, 2 threshold buckets, 3 classified,
  // 4 first grid barrier, 5 row ties staged, 6 ties ranked, 7 second grid
  // barrier, 8 written
  CSA2_TRACE_BEGIN(kTrSelect, tid == 0);
  const int32_t* row = a.scores + (int64_t)q * a.ld;
  uint32_t phase = 0;   // grid barriers passed
  uint32_t* hdr = a.hdr ? a.hdr + q * 4 : nullptr;
  if (tid < 2) {
    bstar_s[tid] = -1;
    above_s[tid] = 0;
    own_cnt[tid] = 0;
    kthr_s[tid] = ~0ull;
  }
  pdl_wait();      // the scores, the histogram and the counts come from the grid before
  pdl_trigger();
  CSA2_MARK(kTrSelect, 1, tid == 0);
  const int32_t n = sel_n(a, q);

  // ---- 1. loads: scores (up to n_max, which the row always holds; masked by
  // n below), this thread's histogram bins when given, the order check
  int32_t s[E];
  if (a.vec && j0 + E <= a.n_max) {
    const int4* p = reinterpret_cast<const int4*>(row + j0);
#pragma unroll
    for (int u = 0; u < E / 4; ++u) {
      const int4 v = __ldcg(p + u);
      s[4 * u + 0] = v.x;
      s[4 * u + 1] = v.y;
      s[4 * u + 2] = v.z;
      s[4 * u + 3] = v.w;
    }
  } else {
#pragma unroll
    for (int i = 0; i < E; ++i) s[i] = j0 + i < a.n_max ? __ldcg(row + j0 + i) : 0;
  }
  uint32_t hb[kBinsPer];
  if (a.hist) {
    const uint4* hp = reinterpret_cast<const uint4*>(a.hist + (size_t)q * kBuckets + tid * kBinsPer);
    const uint4 h0 = __ldcg(hp), h1 = __ldcg(hp + 1);
    hb[0] = h0.x; hb[1] = h0.y; hb[2] = h0.z; hb[3] = h0.w;
    hb[4] = h1.x; hb[5] = h1.y; hb[6] = h1.z; hb[7] = h1.w;
  }
  if (a.cand_pos) {   // candidate positions must ascend (coalesced: stride kSelNT)
    const int32_t* cp = a.cand_pos + (int64_t)q * a.ld;
    bool bad = false;
#pragma unroll
    for (int i = 0; i < E; ++i) {
      const int32_t j = c * kSpan + i * kSelNT + tid;
      if (j > 0 && j < a.n_max) {
        const int32_t p = __ldg(cp + j), pp = __ldg(cp + j - 1);
        bad |= j < n && p <= pp;
      }
    }
    if (bad) record_error(a.status, CSA2_ERR_ORDER);
  }
  uint32_t valid = 0u;   // bit i: candidate j0 + i exists
#pragma unroll
  for (int i = 0; i < E; ++i) valid |= (uint32_t)(j0 + i < n) << i;
  if (!a.hist) {   // one CTA per row: the histogram is built here
    uint4* h4 = reinterpret_cast<uint4*>(hist + tid * kBinsPer);
    h4[0] = make_uint4(0, 0, 0, 0);
    h4[1] = make_uint4(0, 0, 0, 0);
    __syncthreads();
#pragma unroll
    for (int i = 0; i < E; ++i)
      if ((valid >> i) & 1u) atomicAdd(&hist[score_bucket(s[i])], 1u);
    __syncthreads();
    const uint4 h0 = h4[0], h1 = h4[1];
    hb[0] = h0.x; hb[1] = h0.y; hb[2] = h0.z; hb[3] = h0.w;
    hb[4] = h1.x; hb[5] = h1.y; hb[6] = h1.z; hb[7] = h1.w;
  }

  // ---- 2. threshold bucket of each target
  uint32_t hsum = 0;
#pragma unroll
  for (int b = 0; b < kBinsPer; ++b) hsum += hb[b];
  uint64_t total64;
  const uint64_t excl = sel_scan<kSelNT>(hsum, wtmp, &total64);
  const int64_t total = (int64_t)total64;
  const int64_t above_me = total - (int64_t)excl - hsum;   // candidates in the bins above this thread's
#pragma unroll
  for (int t = 0; t < 2; ++t) {
    const int32_t k = a.k[t];
    if (t < n_k && total > k && above_me < k && above_me + hsum >= k) {
      int64_t acc = above_me;
#pragma unroll
      for (int b = kBinsPer - 1; b >= 0; --b) {
        if (acc + hb[b] >= k) {
          bstar_s[t] = tid * kBinsPer + b;
          above_s[t] = (int32_t)acc;
          break;
        }
        acc += hb[b];
      }
    }
  }
  __syncthreads();
  CSA2_MARK(kTrSelect, 2, tid == 0);

  // ---- 3. classify: above b* (members), at b* (ties: this CTA's list)
  const int32_t b0 = bstar_s[0], b1 = n_k > 1 ? bstar_s[1] : INT32_MIN;
  uint32_t above_m[2] = {0u, 0u}, tie_m[2] = {0u, 0u};
#pragma unroll
  for (int i = 0; i < E; ++i) {
    if ((valid >> i) & 1u) {
      const int32_t bk = (int32_t)score_bucket(s[i]);
      if (bk > b0) above_m[0] |= 1u << i;   // b* = -1 takes every candidate
      if (bk > b1) above_m[1] |= 1u << i;
      if (bk == b0 || bk == b1) {
        const uint64_t key = cand_key(s[i], j0 + i);
#pragma unroll
        for (int t = 0; t < 2; ++t) {
          if (bk == (t ? b1 : b0)) {
            tie_m[t] |= 1u << i;
            const uint32_t slot = atomicAdd(&own_cnt[t], 1u);
            if (slot < (uint32_t)kSelTieCap) own[t * kSelTieCap + slot] = key;
          }
        }
      }
    }
  }
  __syncthreads();
  CSA2_MARK(kTrSelect, 3, tid == 0);
  const uint32_t* nt = own_cnt;   // ties in the row
  const uint64_t* list = own;     // the row's ties, [2][kSelTieCap]
  if (G > 1) {
    if (tid < 2) gbase_s[tid] = own_cnt[tid] ? atomicAdd(&hdr[1 + tid], own_cnt[tid]) : 0u;
    __syncthreads();
#pragma unroll
    for (int t = 0; t < 2; ++t) {
      const uint32_t m = nt[t] < (uint32_t)kSelTieCap ? nt[t] : (uint32_t)kSelTieCap;
      uint64_t* dst = a.ties + ((size_t)q * 2 + t) * kSelTieCap;
      for (uint32_t i = tid; i < m; i += kSelNT)
        if (gbase_s[t] + i < (uint32_t)kSelTieCap) dst[gbase_s[t] + i] = own[t * kSelTieCap + i];
    }
    sel_grid_sync(&hdr[0], ++phase * G, a.status);
    CSA2_MARK(kTrSelect, 4, tid == 0);
    if (tid < 2) nt_s[tid] = __ldcg(&hdr[1 + tid]);
    __syncthreads();
#pragma unroll
    for (int t = 0; t < 2; ++t) {
      const uint32_t m = nt_s[t];
      if (m <= (uint32_t)kSelTieCap) {
        const uint64_t* src = a.ties + ((size_t)q * 2 + t) * kSelTieCap;
        for (uint32_t i = tid; i < m; i += kSelNT) rowties[t * kSelTieCap + i] = __ldcg(src + i);
      }
    }
    nt = nt_s;
    list = rowties;
    __syncthreads();
    CSA2_MARK(kTrSelect, 5, tid == 0);
  }
  // rank this CTA's ties against the row's ties
#pragma unroll
  for (int t = 0; t < 2; ++t) {
    if (bstar_s[t] < 0 || nt[t] > (uint32_t)kSelTieCap) continue;
    const int32_t need = a.k[t] - above_s[t];
    const uint32_t mine = own_cnt[t], ntt = nt[t];
    const uint64_t* L = list + t * kSelTieCap;
    for (uint32_t i = warp; i < mine; i += kSelNT / 32) {
      const uint64_t ki = own[t * kSelTieCap + i];
      uint32_t r = 0;
#pragma unroll 4
      for (uint32_t j = lane; j < ntt; j += 32) r += L[j] > ki;
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) r += __shfl_xor_sync(0xffffffffu, r, o);
      if (lane == 0 && (int32_t)r < need) atomicMin(&kthr_s[t], (unsigned long long)ki);
    }
  }
  // very many ties: radix select of the need-th tie key
#pragma unroll 1
  for (int t = 0; t < 2; ++t) {
    if (bstar_s[t] < 0 || nt[t] <= (uint32_t)kSelTieCap) continue;
    uint32_t* gbins = G > 1 ? a.radix + ((size_t)q * 2 + t) * 8 * 256 : nullptr;
    const uint64_t kth = radix_kth<kSelNT, E>(s, t ? tie_m[1] : tie_m[0], j0, a.k[t] - above_s[t], G, c, gbins,
                                              hdr ? &hdr[0] : nullptr, phase, a.status, rsm);
    if (tid == 0) kthr_s[t] = kth;
  }
  __syncthreads();
  CSA2_MARK(kTrSelect, 6, tid == 0);

  // ---- 4. members, their slots and the ordered write
  uint32_t mem[2] = {above_m[0], above_m[1]};
#pragma unroll
  for (int t = 0; t < 2; ++t) {
    if (tie_m[t]) {
      const uint64_t kthr = kthr_s[t];
#pragma unroll
      for (int i = 0; i < E; ++i)
        if (((tie_m[t] >> i) & 1u) && cand_key(s[i], j0 + i) >= kthr) mem[t] |= 1u << i;
    }
  }
  if (n_k < 2) mem[1] = 0u;
  const uint64_t pack = (uint64_t)__popc(mem[0]) | ((uint64_t)__popc(mem[1]) << 32);
  uint64_t cta_tot;
  const uint64_t mexcl = sel_scan<kSelNT>(pack, wtmp, &cta_tot);
  uint64_t off = 0ull, grand = cta_tot;
  if (G > 1) {
    uint32_t* mc = a.mcnt + (size_t)q * 2 * kSelMaxG;
    if (tid == 0) {
      mc[c] = (uint32_t)cta_tot;
      mc[kSelMaxG + c] = (uint32_t)(cta_tot >> 32);
    }
    sel_grid_sync(&hdr[0], ++phase * G, a.status);
    CSA2_MARK(kTrSelect, 7, tid == 0);
    if (warp == 0) {
      uint64_t o = 0ull, g = 0ull;
      for (int r = lane; r < G; r += 32) {
        const uint64_t v = (uint64_t)__ldcg(mc + r) | ((uint64_t)__ldcg(mc + kSelMaxG + r) << 32);
        g += v;
        if (r < c) o += v;
      }
#pragma unroll
      for (int x = 16; x > 0; x >>= 1) {
        o += __shfl_xor_sync(0xffffffffu, o, x);
        g += __shfl_xor_sync(0xffffffffu, g, x);
      }
      if (lane == 0) {
        off_s = o;
        grand_s = g;
      }
    }
    __syncthreads();
    off = off_s;
    grand = grand_s;
  }
  const int32_t* cp = a.cand_pos ? a.cand_pos + (int64_t)q * a.ld : nullptr;
#pragma unroll
  for (int t = 0; t < 2; ++t) {
    if (t >= n_k) break;
    const int32_t k = a.k[t];
    int32_t* dst = a.out_idx[t] + (int64_t)q * k;
    int64_t slot = (int64_t)((off >> (32 * t)) & 0xffffffffu) + (int64_t)((mexcl >> (32 * t)) & 0xffffffffu);
#pragma unroll
    for (int i = 0; i < E; ++i) {
      if ((mem[t] >> i) & 1u) {
        if (slot < k) dst[slot] = cp ? __ldg(cp + j0 + i) : j0 + i;
        ++slot;
      }
    }
    if (c == G - 1) {
      const int64_t g = (int64_t)((grand >> (32 * t)) & 0xffffffffu);
      const int32_t cnt = g < k ? (int32_t)g : k;
      for (int32_t i = cnt + tid; i < k; i += kSelNT) dst[i] = -1;
      if (tid == 0 && a.out_cnt[t]) a.out_cnt[t][q] = cnt;
    }
  }
  CSA2_MARK(kTrSelect, 8, tid == 0);
}

struct SelDev {
  std::atomic<int> max_ctas{0};   // co-resident CTAs of select_kernel<8> (0: not yet known)
};
SelDev g_sel_dev[64];

}  // namespace

bool select_fits(int32_t nq, int32_t n_max) {
  if (n_max <= kSelSpan) return true;
  const int64_t G = ((int64_t)n_max + kSelNT * 8 - 1) / (kSelNT * 8);
  if (G > kSelMaxG) return false;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev >= 64) return false;
  SelDev& d = g_sel_dev[dev];
  if (!d.max_ctas) {
    static SetupMask done{0};
    int per_sm = 0;
    if (ensure_smem(select_kernel<8>, kSelSmem, done) != cudaSuccess ||
        cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, select_kernel<8>, kSelNT, kSelSmem) != cudaSuccess)
      return false;
    d.max_ctas = per_sm * sm_count();
  }
  return G * nq <= d.max_ctas;
}

cudaError_t launch_select(const int32_t* scores, int64_t ld, const int32_t* n_valid,
                          const int32_t* query_pos, const int32_t* cand_pos, int32_t nq, int32_t n_max,
                          const TopkOut* outs, int32_t n_k, const uint32_t* hist, const TopkScratch* s,
                          int32_t* status, cudaStream_t st) {
  // One CTA of 16 candidates per thread up to kSelSpan; beyond, 8 per thread
  // over co-resident CTAs (shorter passes per CTA, more SMs).
  const bool one = n_max <= kSelSpan;
  const int span = one ? kSelSpan : kSelNT * 8;
  const int64_t G64 = one ? 1 : ((int64_t)n_max + span - 1) / span;
  if (G64 > 1 && (!hist || !s)) return cudaErrorNotSupported;
  if (G64 > kSelMaxG) return cudaErrorNotSupported;
  const int G = (int)G64;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  static SetupMask done16{0}, done8{0};
  e = one ? ensure_smem(select_kernel<16>, kSelSmem, done16) : ensure_smem(select_kernel<8>, kSelSmem, done8);
  if (e != cudaSuccess) return e;
  if (G > 1) {
    if (dev >= 64) return cudaErrorNotSupported;
    SelDev& d = g_sel_dev[dev];
    if (!d.max_ctas) {
      int per_sm = 0;
      e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, select_kernel<8>, kSelNT, kSelSmem);
      if (e != cudaSuccess) return e;
      d.max_ctas = per_sm * sm_count();
    }
    if ((int64_t)G * nq > d.max_ctas) return cudaErrorNotSupported;
  }
  SelArgs a{};
  a.scores = scores;
  a.ld = ld;
  a.n_valid = n_valid;
  a.query_pos = query_pos;
  a.cand_pos = cand_pos;
  a.n_max = n_max;
  a.hist = hist;
  if (s) {
    a.hdr = s->sel_hdr;
    a.ties = s->sel_ties;
    a.mcnt = s->sel_mcnt;
    a.radix = s->sel_radix;
  }
  a.G = G;
  a.n_k = n_k;
  a.vec = (reinterpret_cast<uintptr_t>(scores) % 16 == 0) && (ld % 4 == 0);
  for (int t = 0; t < 2; ++t) {
    const TopkOut& o = outs[t < n_k ? t : 0];
    a.k[t] = o.k;
    a.out_idx[t] = o.idx;
    a.out_cnt[t] = o.cnt;
  }
  a.status = status;
  const bool pdl = launch_opts().pdl;
  return one ? launch_k(select_kernel<16>, dim3(G, nq, 1), dim3(kSelNT), kSelSmem, st, false, pdl, a)
             : launch_k(select_kernel<8>, dim3(G, nq, 1), dim3(kSelNT), kSelSmem, st, false, pdl, a);
}

}  // namespace csa2
