// Building blocks of the exact top-k selections (topk_select.cu, reindex.cu).
//
// A selection keeps the k candidates with the largest keys cand_key(score,
// index): higher score first, then the lower index.  Its steps share these
// pieces: a block scan, a bounded barrier across the co-resident CTAs of one
// row, and the radix select that finds the k-th key when a score
// distribution is too flat for the tie ranking.
#pragma once

#include "csa2_device.cuh"

namespace csa2 {

// Exclusive scan over the NT threads of a block (pairs of 32-bit counts
// packed in 64 bits add without carries); *total gets the sum.  Ends with a
// barrier, so wtmp (NT / 32 entries) can be reused at once.
template <int NT>
__device__ __forceinline__ uint64_t sel_scan(uint64_t v, uint64_t* wtmp, uint64_t* total) {
  static_assert(NT % 32 == 0 && NT <= 1024, "whole warps");
  constexpr int NW = NT / 32;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  uint64_t x = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const uint64_t y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += y;
  }
  if (lane == 31) wtmp[warp] = x;
  __syncthreads();
  if (warp == 0) {
    uint64_t y = lane < NW ? wtmp[lane] : 0ull;
#pragma unroll
    for (int o = 1; o < NW; o <<= 1) {
      const uint64_t z = __shfl_up_sync(0xffffffffu, y, o);
      if (lane >= o) y += z;
    }
    if (lane < NW) wtmp[lane] = y;
  }
  __syncthreads();
  const uint64_t base = warp > 0 ? wtmp[warp - 1] : 0ull;
  *total = wtmp[NW - 1];
  __syncthreads();
  return base + x - v;
}

// Barrier of the G co-resident CTAs of one row: waits until `bar` (zeroed
// before the launch) reaches `target`, a multiple of G.  The block barrier
// orders the CTA's writes before thread 0's release-add; thread 0's acquire
// load, then the block barrier, order the other CTAs' writes before every
// later read.  Bounded: after limit_ns it records CSA2_ERR_TIMEOUT and goes
// on.
__device__ __forceinline__ void sel_grid_sync(uint32_t* bar, uint32_t target, int32_t* status,
                                              uint64_t limit_ns = kWaitLimitNs) {
  __syncthreads();
  if (threadIdx.x == 0) {
    asm volatile("red.release.gpu.global.add.u32 [%0], 1;" ::"l"(bar) : "memory");
    uint32_t v;
    asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(bar) : "memory");
    if (v < target) {
      const uint64_t t0 = global_ns();
      do {
        if (global_ns() - t0 > limit_ns) {
          record_error(status, CSA2_ERR_TIMEOUT);
          break;
        }
        asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(bar) : "memory");
      } while (v < target);
    }
  }
  __syncthreads();
}

struct RadixSmem {
  uint32_t dig[256];
  unsigned long long prefix;
  int32_t rem;
};

// The rem-th largest key (rem >= 1) among the marked candidates of a row:
// thread-held candidates s[i] (E <= 64) with index j0 + i where bit i of
// `mark` is set.
// One 8-bit digit of the 64-bit key per pass, from the top.  With G > 1 CTAs
// per row, gbins ([8][256], any contents) collects the digit counts of the
// row; CTA c == 0 clears it, and every pass meets at a grid barrier.
template <int NT, int E>
__device__ uint64_t radix_kth(const int32_t (&s)[E], uint64_t mark, int32_t j0, int32_t rem, int G, int c,
                              uint32_t* gbins, uint32_t* bar, uint32_t& phase, int32_t* status, RadixSmem& sm) {
  static_assert(E <= 64, "one mark bit per candidate");
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  if (G > 1) {
    if (c == 0)
      for (int i = tid; i < 8 * 256; i += NT) gbins[i] = 0u;
    sel_grid_sync(bar, ++phase * G, status);
  }
  uint64_t prefix = 0ull, fixed = 0ull;
  for (int pass = 0; pass < 8; ++pass) {
    const int shift = 56 - 8 * pass;
    for (int i = tid; i < 256; i += NT) sm.dig[i] = 0u;
    __syncthreads();
#pragma unroll
    for (int i = 0; i < E; ++i) {
      if ((mark >> i) & 1ull) {
        const uint64_t key = cand_key(s[i], j0 + i);
        if ((key & fixed) == prefix) atomicAdd(&sm.dig[(key >> shift) & 255u], 1u);
      }
    }
    __syncthreads();
    if (G > 1) {
      for (int i = tid; i < 256; i += NT)
        if (sm.dig[i]) atomicAdd(&gbins[pass * 256 + i], sm.dig[i]);
      sel_grid_sync(bar, ++phase * G, status);
      for (int i = tid; i < 256; i += NT) sm.dig[i] = __ldcg(&gbins[pass * 256 + i]);
      __syncthreads();
    }
    if (warp == 0) {   // lane l holds digits 255-8l .. 248-8l (lane 0: the highest)
      uint32_t d8[8], sum = 0;
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        d8[u] = sm.dig[255 - 8 * lane - u];
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
            sm.prefix = prefix | ((uint64_t)(255 - 8 * lane - u) << shift);
            sm.rem = rem - (int32_t)acc;
            break;
          }
          acc += d8[u];
        }
      }
    }
    __syncthreads();
    prefix = sm.prefix;
    rem = sm.rem;
    fixed |= 255ull << shift;
    __syncthreads();
  }
  return prefix;
}

// The rem-th largest (rem >= 1) of the keys key_at(0 .. n-1), found by the
// whole block; every thread returns it.  key_at(i) is the key of item i, or
// 0 when item i takes no part (no candidate key is 0); k0 is the key of any
// item that takes part, and the keys that take part are distinct.  One 11-bit
// digit per pass from the highest bit at which the keys differ; the passes
// stop as soon as the chosen digit holds exactly the keys still wanted (the
// answer is then its smallest key, a single key included).
struct ListKthSmem {
  uint32_t bins[2048];
  unsigned long long orv, res;
  uint64_t prefix;
  int32_t rem;
  uint32_t cnt;
};

template <int NT, class KeyAt>
__device__ uint64_t block_kth(uint32_t n, int32_t rem, KeyAt key_at, uint64_t k0, uint64_t* wtmp, ListKthSmem& sm) {
  static_assert(2048 % NT == 0, "whole bins per thread");
  constexpr int BPT = 2048 / NT;
  const int tid = threadIdx.x, lane = tid & 31;
  __syncthreads();   // earlier readers of sm are done
  if (tid == 0) {
    sm.orv = 0ull;
    sm.res = ~0ull;
  }
  __syncthreads();
  uint64_t d = 0ull;
  for (uint32_t i = tid; i < n; i += NT) {
    const uint64_t k = key_at(i);
    if (k) d |= k ^ k0;
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) d |= __shfl_xor_sync(0xffffffffu, d, o);
  if (lane == 0 && d) atomicOr(&sm.orv, (unsigned long long)d);
  __syncthreads();
  const uint64_t diff = sm.orv;
  if (diff == 0ull) return k0;   // one key
  const int hb = 63 - __clzll((long long)diff);
  uint64_t fixed = hb == 63 ? 0ull : ~((2ull << hb) - 1ull);   // the bits above hb are common
  uint64_t prefix = k0 & fixed;
  int lo = hb + 1;   // bits lo..63 are decided
  for (;;) {
    const int nb = lo < 11 ? lo : 11;
    const int shift = lo - nb;
    const uint64_t dmask = (1ull << nb) - 1ull;
#pragma unroll
    for (int u = 0; u < BPT; ++u) sm.bins[tid * BPT + u] = 0u;
    __syncthreads();
    for (uint32_t i = tid; i < n; i += NT) {
      const uint64_t k = key_at(i);
      if (k && (k & fixed) == prefix) atomicAdd(&sm.bins[(k >> shift) & dmask], 1u);
    }
    __syncthreads();
    uint32_t c[BPT], sum = 0;   // thread t: bins 2047 - BPT t - u, from the top
#pragma unroll
    for (int u = 0; u < BPT; ++u) {
      c[u] = sm.bins[2047 - BPT * tid - u];
      sum += c[u];
    }
    uint64_t tot;
    const uint32_t before = (uint32_t)sel_scan<NT>(sum, wtmp, &tot);
    if ((int64_t)before < rem && (int64_t)before + sum >= rem) {
      uint32_t acc = before;
#pragma unroll
      for (int u = 0; u < BPT; ++u) {
        if ((int64_t)acc + c[u] >= rem) {
          sm.prefix = prefix | ((uint64_t)(2047 - BPT * tid - u) << shift);
          sm.rem = rem - (int32_t)acc;
          sm.cnt = c[u];
          break;
        }
        acc += c[u];
      }
    }
    __syncthreads();
    prefix = sm.prefix;
    rem = sm.rem;
    const uint32_t cnt = sm.cnt;
    fixed |= dmask << shift;
    lo = shift;
    if (lo == 0) return prefix;   // every bit decided
    if ((uint32_t)rem == cnt) {   // the digit holds exactly the keys wanted: its smallest
      for (uint32_t i = tid; i < n; i += NT) {
        const uint64_t k = key_at(i);
        if (k && (k & fixed) == prefix) atomicMin(&sm.res, (unsigned long long)k);
      }
      __syncthreads();
      return sm.res;
    }
    __syncthreads();   // sm.prefix/rem/cnt are read everywhere before the next pass
  }
}

}  // namespace csa2
