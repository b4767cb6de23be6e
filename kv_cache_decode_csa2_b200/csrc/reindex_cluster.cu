// K3 on thread-block clusters: the reindex scoring and top-K of one (layer,
// query) pool inside ONE cluster of C CTAs, with no grid-wide barrier and no
// global atomics.
//
// A reindex layer re-scores only the candidate pool of the full layer and
// keeps its best K ("later layers search only that much smaller pool instead
// of rescanning everything": "DeepSeek V4.1-Flash: 552B runs like 16B",
// Act 2).  Ties go to the lower position and the selection is written in
// ascending position order.
//
// Each CTA owns 1024 consecutive pool slots (C = 1024-slot blocks of the pool,
// rounded up to a power of two, at most 16).  It
//   1. gathers its slots' key rows by position (16-byte cp.async) into eight
//      swizzled K-major 128-row tiles, and scores all eight with one tcgen05
//      int8 MMA group, D[128 slots x N heads] per tile in TMEM; the epilogue
//      applies ReLU and the integer head weights (the full-mode formula);
//   2. counts its scores into a 13-bit bucket histogram in shared memory;
//   3. cluster barrier; CTA r sums bucket slice r over the cluster through
//      distributed shared memory (DSMEM);
//   4. cluster barrier; every CTA reads the C slice totals, finds the slice
//      that holds the K-th best score, and walks that slice (remote) for the
//      threshold bucket b* and the count above it;
//   5. classifies its slots (above b*, tie at b*), publishes its counts and
//      its tie keys; cluster barrier;
//   6. if the ties must be split, every CTA gathers the cluster's tie list
//      and ranks its own ties against it (or, for a very flat pool, the
//      cluster runs a radix select of the need-th tie key), publishes its
//      tie-member count; cluster barrier;
//   7. from the counts of the CTAs before it, writes its members in slot
//      order, which is position order because pool positions ascend.
// The cluster barriers are the hardware's (barrier.cluster with release /
// acquire semantics); every CTA of a cluster passes the same barriers on every
// path, and no CTA leaves while another may still read its shared memory.
// Clusters are independent, so a launch of many problems needs no
// co-residency beyond one cluster at a time.
#include <cooperative_groups.h>

#include "csa2_device.cuh"
#include "internal.h"
#include "select_common.cuh"

namespace cg = cooperative_groups;

namespace csa2 {

CSA2_TRACE_UNIT(rcluster)

namespace {

constexpr int kRcSlots = 1024;                  // pool slots per CTA
constexpr int kRcNT = 256;                      // threads per CTA
constexpr int kRcPer = kRcSlots / kRcNT;        // slots per thread: local slot tid + j * kRcNT
constexpr int kRcTiles = kRcSlots / 128;        // 128-slot MMA tiles per CTA
constexpr int kRcMaxC = 16;                     // CTAs per cluster (above 8: a non-portable size)
constexpr int kRcGather = 4096;                 // ties gathered into every CTA for the exact rank

struct RcJob {
  const int8_t* q;          // [nq][H][D]
  const int8_t* w;          // [nq][H]
  const uint8_t* base;      // index keys
  int64_t row_bytes;
  RowMap rows;
  int32_t* scores;          // [nq][P] or nullptr
  int32_t* sel_idx;         // [nq][K]
  int32_t* sel_cnt;         // [nq] or nullptr
};

struct RcArgs {
  RcJob job[kMaxReindexJobs];
  const int32_t* seq_of_query;
  const int32_t* pool_idx;
  const int32_t* pool_cnt;
  int32_t H, P, K, nq, C;
  int32_t* status;
};

__device__ __forceinline__ void rc_cp_async16(void* dst, const void* src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(smem_u32(dst)), "l"(src) : "memory");
}
__device__ __forceinline__ void rc_cp_async_wait_all() { asm volatile("cp.async.wait_all;" ::: "memory"); }

// Dynamic shared memory.  The A tiles are dead once the MMA has completed;
// their bytes then hold the local histogram and the gathered tie list.
template <int D, int N>
struct RcLayout {
  static constexpr size_t a_bytes = (size_t)kRcSlots * D;
  static constexpr size_t hist_off = 0;                                 // [kBuckets] u32   (after the MMA)
  static constexpr size_t gath_off = (size_t)kBuckets * 4;              // [kRcGather] u64  (after the MMA)
  static_assert(gath_off + (size_t)kRcGather * 8 <= a_bytes, "histogram and tie list fit in the A tiles");
  static constexpr size_t b_off = a_bytes;                              // N x D (swizzled)
  static constexpr size_t red_off = b_off + (size_t)N * D;              // [kBuckets / 2] u32: reduced slice
  static constexpr size_t own_off = red_off + (size_t)kBuckets * 2;     // [kRcSlots] u64: own tie keys
  static constexpr size_t pos_off = own_off + (size_t)kRcSlots * 8;     // [kRcSlots] i32: pool positions
  static constexpr size_t row_off = pos_off + (size_t)kRcSlots * 4;     // [kRcSlots] i64: physical rows
  static constexpr size_t w_off = row_off + (size_t)kRcSlots * 8;       // [N] i32: head weights
  static constexpr size_t bar_off = w_off + (size_t)N * 4;              // u64 MMA barrier, u32 TMEM slot
  static constexpr size_t total = 1024 + bar_off + 64;                  // + alignment of the tiles
};

// Sum of v over the CTA's threads, returned to every thread.
__device__ __forceinline__ uint32_t rc_block_sum(uint32_t v, uint32_t* tmp) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  __syncthreads();
  if (lane == 0) tmp[warp] = v;
  __syncthreads();
  uint32_t t = 0;
#pragma unroll
  for (int w = 0; w < kRcNT / 32; ++w) t += tmp[w];
  return t;
}

template <int D, int N>
__global__ void __launch_bounds__(kRcNT, 1) reindex_cluster_kernel(const __grid_constant__ RcArgs a) {
  using Lay = RcLayout<D, N>;
  static_assert(kRcTiles * N <= 512, "every tile's accumulator fits in TMEM");
  constexpr uint32_t TMEM_COLS = kRcTiles * N <= 32    ? 32
                                 : kRcTiles * N <= 64  ? 64
                                 : kRcTiles * N <= 128 ? 128
                                 : kRcTiles * N <= 256 ? 256
                                                       : 512;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* atile = smem;
  uint32_t* hist = reinterpret_cast<uint32_t*>(smem + Lay::hist_off);
  uint64_t* gath = reinterpret_cast<uint64_t*>(smem + Lay::gath_off);
  uint8_t* bmat = smem + Lay::b_off;
  uint32_t* red = reinterpret_cast<uint32_t*>(smem + Lay::red_off);
  uint64_t* own = reinterpret_cast<uint64_t*>(smem + Lay::own_off);
  int32_t* pos_s = reinterpret_cast<int32_t*>(smem + Lay::pos_off);
  int64_t* row_s = reinterpret_cast<int64_t*>(smem + Lay::row_off);
  int32_t* w_s = reinterpret_cast<int32_t*>(smem + Lay::w_off);
  uint64_t* bar = reinterpret_cast<uint64_t*>(smem + Lay::bar_off);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bar + 1);
  __shared__ uint64_t wtmp[kRcNT / 32];
  __shared__ uint32_t utmp[kRcNT / 32];
  __shared__ int32_t bstar_s, above_s;
  __shared__ uint32_t tot_s, cabove_s, ctie_s, ctm_s;
  __shared__ unsigned long long kmin_s;
  __shared__ uint32_t c_above[kRcMaxC], c_tie[kRcMaxC], c_tm[kRcMaxC], c_tot[kRcMaxC];
  __shared__ uint32_t mbits[kRcSlots / 32], mpre[kRcSlots / 32];
  __shared__ uint32_t dh[256];
  __shared__ unsigned long long rprefix_s;
  __shared__ int32_t rneed_s;

  cg::cluster_group cl = cg::this_cluster();
  const int C = a.C;
  const int rank = (int)cl.block_rank();
  const int q = blockIdx.y, jb = blockIdx.z;
  const RcJob& J = a.job[jb];
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int32_t K = a.K;
  // trace points: 1 own inputs staged, 2 grid before done, 3 rows gathered,
  // 4 scored, 5 histogram barrier, 6 slice barrier, 7 threshold, 8 count
  // barrier, 9 ties resolved, 10 written
  CSA2_TRACE_BEGIN(kTrRCluster, tid == 0);

  // ---- prologue on this layer's own inputs: TMEM, the MMA barrier, the
  // query rows (B operand), the head weights
  if (warp == 0) {
    tmem_alloc(tmem_slot, TMEM_COLS);
    tmem_relinquish();
  }
  if (tid == 0) {
    mbar_init(bar, 1);
    fence_mbar_init();
    bstar_s = -1;
    above_s = 0;
    cabove_s = 0;
    ctie_s = 0;
    ctm_s = 0;
    kmin_s = ~0ull;
  }
  if (tid < kRcSlots / 32) mbits[tid] = 0u;
  {
    const int8_t* qsrc = J.q + (int64_t)q * a.H * D;
    for (int idx = tid; idx < N * (D / 16); idx += kRcNT) {
      const int r = idx / (D / 16), c = idx % (D / 16);
      int4 v = make_int4(0, 0, 0, 0);
      if (r < a.H) v = __ldg(reinterpret_cast<const int4*>(qsrc + r * D) + c);
      *reinterpret_cast<int4*>(bmat + swizzled_chunk(r, c, D)) = v;
    }
    if (tid < N) w_s[tid] = tid < a.H ? (int32_t)__ldg(J.w + (int64_t)q * a.H + tid) : 0;
  }
  CSA2_MARK(kTrRCluster, 1, tid == 0);
  pdl_wait();      // the pool comes from the grid before
  pdl_trigger();
  CSA2_MARK(kTrRCluster, 2, tid == 0);

  // ---- this CTA's slots: positions, physical rows, then the key rows
  int32_t cnt = __ldg(a.pool_cnt + q);
  cnt = cnt < 0 ? 0 : (cnt > a.P ? a.P : cnt);
  const int32_t slot0 = rank * kRcSlots;
  const int32_t* pidx = a.pool_idx + (int64_t)q * a.P;
  const int32_t seq = a.seq_of_query ? __ldg(a.seq_of_query + q) : q;
  uint32_t vmask = 0u;   // bit j: local slot tid + j kRcNT holds a scorable pool entry
#pragma unroll
  for (int j = 0; j < kRcPer; ++j) {
    const int s = tid + j * kRcNT;
    const int32_t slot = slot0 + s;
    int32_t p = -1;
    int64_t r = -1;
    if (slot < cnt) {
      p = __ldg(pidx + slot);
      const int32_t prev = slot > 0 ? __ldg(pidx + slot - 1) : INT32_MIN;
      if (p <= prev) record_error(a.status, CSA2_ERR_ORDER);   // pool positions ascend
      r = p >= 0 ? map_row(J.rows, seq, p) : -1;
      if (r < 0) record_error(a.status, CSA2_ERR_INDEX_RANGE);
      else vmask |= 1u << j;
    }
    pos_s[s] = p;
    row_s[s] = r;
  }
  __syncthreads();
  const int n_valid_slots = cnt - slot0 < 0 ? 0 : (cnt - slot0 > kRcSlots ? kRcSlots : cnt - slot0);
  const int n_tiles = (n_valid_slots + 127) / 128;   // CTA-uniform
  {
    constexpr int CH = D / 16;   // 16-byte chunks per row; consecutive threads read one row together
    for (int i = tid; i < n_tiles * 128 * CH; i += kRcNT) {
      const int s = i / CH, c = i % CH;
      uint8_t* dst = atile + (s >> 7) * 128 * D + swizzled_chunk(s & 127, c, D);
      const int64_t r = row_s[s];
      if (r >= 0) rc_cp_async16(dst, J.base + r * J.row_bytes + 16 * c);
      else *reinterpret_cast<int4*>(dst) = make_int4(0, 0, 0, 0);
    }
  }
  rc_cp_async_wait_all();
  fence_async_smem();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  CSA2_MARK(kTrRCluster, 3, tid == 0);
  const uint32_t tmem_base = *tmem_slot;
  if (tid == 0 && n_tiles > 0) {
    constexpr uint32_t idesc = idesc_i8(128, N);
    const uint32_t a_addr = smem_u32(atile), b_addr = smem_u32(bmat);
    for (int t = 0; t < n_tiles; ++t)   // tile t accumulates in TMEM columns [t N, t N + N)
#pragma unroll
      for (int k = 0; k < D / 32; ++k)
        mma_i8(tmem_base + t * N, smem_desc_kmajor(a_addr + t * 128 * D + 32 * k, D),
               smem_desc_kmajor(b_addr + 32 * k, D), idesc, k > 0 ? 1u : 0u);
    mma_commit(bar);
  }

  // ---- scores of this thread's slots (the full-mode formula)
  int32_t sc[kRcPer];
#pragma unroll
  for (int j = 0; j < kRcPer; ++j) sc[j] = 0;
  if (n_tiles > 0) {
    volatile int32_t never = 0;
    const bool ok = __all_sync(0xffffffffu, mbar_wait(bar, 0, &never));
    if (ok) {
      tc_fence_after();
#pragma unroll
      for (int j = 0; j < kRcPer; ++j) {
        const int t = (tid >> 7) + 2 * j;   // local slot tid + 256 j lies in tile t, row tid % 128
        if (t < n_tiles) {                  // warp-uniform
          const uint32_t taddr = tmem_base + ((uint32_t)((warp & 3) * 32) << 16) + (uint32_t)(t * N);
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
          sc[j] = s;
        }
      }
    } else if (tid == 0) {
      record_error(a.status, CSA2_ERR_TIMEOUT);
      vmask = 0u;
    }
  }
  tc_fence_before();
  __syncthreads();   // the MMA has completed and TMEM is read: the tiles become the histogram
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem_base, TMEM_COLS);
  }
  CSA2_MARK(kTrRCluster, 4, tid == 0);
  if (J.scores) {
#pragma unroll
    for (int j = 0; j < kRcPer; ++j)
      if ((vmask >> j) & 1u) J.scores[(int64_t)q * a.P + slot0 + tid + j * kRcNT] = sc[j];
  }

  // ---- the CTA's bucket histogram, then the cluster's, slice by slice
  for (int i = tid; i < kBuckets; i += kRcNT) hist[i] = 0u;
  __syncthreads();
  int32_t bk[kRcPer];
#pragma unroll
  for (int j = 0; j < kRcPer; ++j) {
    bk[j] = (int32_t)score_bucket(sc[j]);
    if ((vmask >> j) & 1u) atomicAdd(&hist[bk[j]], 1u);
  }
  cl.sync();   // every CTA's histogram is complete
  CSA2_MARK(kTrRCluster, 5, tid == 0);
  const int BS = kBuckets / C;                       // buckets per slice
  const uint32_t* slice_mine = C > 1 ? red : hist;   // slice `rank` summed over the cluster
  {
    uint32_t part = 0;
    if (C > 1) {
      for (int b4 = tid; b4 < BS / 4; b4 += kRcNT) {
        uint4 v = make_uint4(0, 0, 0, 0);
        for (int c = 0; c < C; ++c) {
          const uint4 x = reinterpret_cast<const uint4*>(cl.map_shared_rank(hist, c) + rank * BS)[b4];
          v.x += x.x;
          v.y += x.y;
          v.z += x.z;
          v.w += x.w;
        }
        reinterpret_cast<uint4*>(red)[b4] = v;
        part += v.x + v.y + v.z + v.w;
      }
    } else {
#pragma unroll
      for (int j = 0; j < kRcPer; ++j) part += (vmask >> j) & 1u;
    }
    const uint32_t t = rc_block_sum(part, utmp);
    if (tid == 0) tot_s = t;
  }
  cl.sync();   // the reduced slices and their totals are published
  CSA2_MARK(kTrRCluster, 6, tid == 0);

  // ---- threshold bucket b*: the slice that holds the K-th best score
  // (counted from the top), then the bucket inside it
  if (tid < C) c_tot[tid] = *cl.map_shared_rank(&tot_s, tid);
  __syncthreads();
  {
    uint32_t total = 0;
    for (int c = 0; c < C; ++c) total += c_tot[c];
    if ((int64_t)total > K) {
      int rs = 0;
      uint32_t acc = 0;
      for (int c = C - 1; c >= 0; --c) {
        if (acc + c_tot[c] >= (uint32_t)K) {
          rs = c;
          break;
        }
        acc += c_tot[c];
      }
      const uint32_t* sl = C > 1 ? cl.map_shared_rank(red, rs) : hist;
      const int per = BS / kRcNT;   // buckets per thread: 2 .. 32
      uint32_t hsum = 0;
      for (int i = 0; i < per; ++i) hsum += sl[tid * per + i];
      uint64_t stot;
      const uint64_t ex = sel_scan<kRcNT>(hsum, wtmp, &stot);
      const int64_t above_me = (int64_t)stot - (int64_t)ex - hsum;
      const int64_t kk = (int64_t)K - acc;   // rank wanted inside the slice
      if (above_me < kk && above_me + hsum >= kk) {
        int64_t run = above_me;
        for (int i = per - 1; i >= 0; --i) {
          const uint32_t v = sl[tid * per + i];
          if (run + v >= kk) {
            bstar_s = rs * BS + tid * per + i;
            above_s = (int32_t)(acc + run);
            break;
          }
          run += v;
        }
      }
    }
    (void)slice_mine;
  }
  __syncthreads();
  CSA2_MARK(kTrRCluster, 7, tid == 0);
  const int32_t bstar = bstar_s;   // -1: every scorable slot is a member

  // ---- classify this CTA's slots; publish the counts and the tie keys
  uint32_t above_m = 0u, tie_m = 0u;
  uint64_t key[kRcPer];
#pragma unroll
  for (int j = 0; j < kRcPer; ++j) {
    key[j] = cand_key(sc[j], slot0 + tid + j * kRcNT);
    if ((vmask >> j) & 1u) {
      if (bk[j] > bstar) above_m |= 1u << j;
      else if (bk[j] == bstar) {
        tie_m |= 1u << j;
        own[atomicAdd(&ctie_s, 1u)] = key[j];
      }
    }
  }
  {
    const uint32_t t = rc_block_sum((uint32_t)__popc(above_m), utmp);
    if (tid == 0) cabove_s = t;
  }
  cl.sync();   // counts and tie lists are published
  CSA2_MARK(kTrRCluster, 8, tid == 0);
  if (tid < C) {
    c_above[tid] = *cl.map_shared_rank(&cabove_s, tid);
    c_tie[tid] = *cl.map_shared_rank(&ctie_s, tid);
  }
  __syncthreads();
  uint32_t T = 0;
  for (int c = 0; c < C; ++c) T += c_tie[c];
  const int32_t need = K - above_s;
  // ties that are members: all of them unless they must be split
  const bool split = bstar >= 0 && T > (uint32_t)need;   // cluster-uniform
  if (split) {
    if (T <= (uint32_t)kRcGather) {
      // every CTA gathers the cluster's tie keys and ranks its own against
      // them: a tie is a member when fewer than `need` ties beat it
      uint32_t pre = 0;
      for (int c = 0; c < C; ++c) {
        const uint64_t* src = cl.map_shared_rank(own, c);
        for (uint32_t i = tid; i < c_tie[c]; i += kRcNT) gath[pre + i] = src[i];
        pre += c_tie[c];
      }
      __syncthreads();
      const uint32_t mine = ctie_s;
      for (uint32_t i = warp; i < mine; i += kRcNT / 32) {
        const uint64_t ki = own[i];
        uint32_t r = 0;
        for (uint32_t j = lane; j < T; j += 32) r += gath[j] > ki;
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) r += __shfl_xor_sync(0xffffffffu, r, o);
        if (lane == 0 && (int32_t)r < need) {
          atomicAdd(&ctm_s, 1u);
          atomicMin(&kmin_s, (unsigned long long)ki);
        }
      }
    } else {
      // a very flat pool: radix select of the need-th tie key over the
      // cluster, one 8-bit digit of the 64-bit key per pass
      if (tid == 0) {
        rprefix_s = 0ull;
        rneed_s = need;
      }
      unsigned long long mask = 0ull;
#pragma unroll 1
      for (int pass = 0; pass < 8; ++pass) {
        const int shift = 56 - 8 * pass;
        dh[tid] = 0u;   // kRcNT == 256 digits
        __syncthreads();
        const unsigned long long prefix = rprefix_s;
        for (uint32_t i = tid; i < ctie_s; i += kRcNT) {
          const uint64_t k = own[i];
          if ((k & mask) == prefix) atomicAdd(&dh[(k >> shift) & 255u], 1u);
        }
        const int32_t nd = rneed_s;
        cl.sync();   // every CTA's digit counts of this pass
        {
          const int d = 255 - tid;   // thread 0 takes the highest digit
          uint32_t v = 0;
          for (int c = 0; c < C; ++c) v += cl.map_shared_rank(dh, c)[d];
          uint64_t dtot;
          const uint64_t ex = sel_scan<kRcNT>(v, wtmp, &dtot);   // tie keys above digit d
          if ((int64_t)ex < nd && (int64_t)(ex + v) >= nd) {
            rprefix_s = prefix | ((unsigned long long)d << shift);
            rneed_s = nd - (int32_t)ex;
          }
        }
        cl.sync();   // nobody clears its digit counts while another may read them
        mask |= 0xFFull << shift;
      }
      const unsigned long long kth = rprefix_s;   // the need-th best tie key, exactly
      uint32_t m = 0;
      for (uint32_t i = tid; i < ctie_s; i += kRcNT) m += own[i] >= kth;
      const uint32_t t = rc_block_sum(m, utmp);
      if (tid == 0) {
        ctm_s = t;
        kmin_s = kth;
      }
    }
    cl.sync();   // every CTA's tie-member count is published
    if (tid < C) c_tm[tid] = *cl.map_shared_rank(&ctm_s, tid);
    __syncthreads();
  } else if (tid < C) {
    c_tm[tid] = bstar >= 0 ? c_tie[tid] : 0u;
  }
  __syncthreads();
  CSA2_MARK(kTrRCluster, 9, tid == 0);

  // ---- members in slot order: the counts of the CTAs before, then ranks
  // inside the CTA from a bitmap of its slots
  uint32_t off = 0, grand = 0;
  for (int c = 0; c < C; ++c) {
    const uint32_t m = c_above[c] + c_tm[c];
    grand += m;
    if (c < rank) off += m;
  }
  const unsigned long long kthr = split ? kmin_s : 0ull;   // split: own member ties are those >= kthr
  uint32_t mem = above_m;
#pragma unroll
  for (int j = 0; j < kRcPer; ++j)
    if (((tie_m >> j) & 1u) && key[j] >= kthr) mem |= 1u << j;
#pragma unroll
  for (int j = 0; j < kRcPer; ++j) {
    const int s = tid + j * kRcNT;
    if ((mem >> j) & 1u) atomicOr(&mbits[s >> 5], 1u << (s & 31));
  }
  __syncthreads();
  if (warp == 0) {
    const uint32_t c0 = (uint32_t)__popc(mbits[lane]);
    uint32_t x = c0;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const uint32_t y = __shfl_up_sync(0xffffffffu, x, o);
      if (lane >= o) x += y;
    }
    mpre[lane] = x - c0;
  }
  __syncthreads();
  int32_t* dst = J.sel_idx + (int64_t)q * K;
#pragma unroll
  for (int j = 0; j < kRcPer; ++j) {
    if ((mem >> j) & 1u) {
      const int s = tid + j * kRcNT;
      const uint32_t r = off + mpre[s >> 5] + (uint32_t)__popc(mbits[s >> 5] & ((1u << (s & 31)) - 1u));
      if (r < (uint32_t)K) dst[r] = pos_s[s];
    }
  }
  if (rank == C - 1) {
    const int32_t n_out = grand < (uint32_t)K ? (int32_t)grand : K;
    for (int32_t i = n_out + tid; i < K; i += kRcNT) dst[i] = -1;
    if (tid == 0 && J.sel_cnt) J.sel_cnt[q] = n_out;
  }
  CSA2_MARK(kTrRCluster, 10, tid == 0);
  cl.sync();   // no CTA leaves while another may still read its shared memory
}

struct RcDev {
  std::atomic<int> ok[kRcMaxC + 1];   // per cluster size: 1 fits, 2 does not, 0 unknown
};
RcDev g_rc_dev[64];

template <int D, int N>
cudaError_t launch_rc_t(const RcArgs& a, int n_jobs, cudaStream_t st) {
  using Lay = RcLayout<D, N>;
  const auto kern = reindex_cluster_kernel<D, N>;
  static SetupMask done{0};
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev >= 64) return cudaErrorNotSupported;
  e = ensure_smem(kern, (int)Lay::total, done);
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(a.C, a.nq, n_jobs);
  cfg.blockDim = dim3(kRcNT);
  cfg.dynamicSmemBytes = Lay::total;
  cfg.stream = st;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = a.C;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  std::atomic<int>& ok = g_rc_dev[dev].ok[a.C];
  if (ok.load() == 0) {   // can one cluster of this size be resident at all?
    if (a.C > 8 && cudaFuncSetAttribute(kern, cudaFuncAttributeNonPortableClusterSizeAllowed, 1) != cudaSuccess) {
      (void)cudaGetLastError();
      ok = 2;
      return cudaErrorNotSupported;
    }
    int n = 0;
    if (cudaOccupancyMaxActiveClusters(&n, kern, &cfg) != cudaSuccess || n < 1) {
      (void)cudaGetLastError();
      ok = 2;
      return cudaErrorNotSupported;
    }
    ok = 1;
  }
  if (ok.load() != 1) return cudaErrorNotSupported;
  const bool pdl = launch_opts().pdl;
  if (pdl) {
    attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[1].val.programmaticStreamSerializationAllowed = 1;
    cfg.numAttrs = 2;
  }
  e = cudaLaunchKernelEx(&cfg, kern, a);
  if (e != cudaSuccess && pdl) {   // retry without the programmatic attribute
    (void)cudaGetLastError();
    cfg.numAttrs = 1;
    e = cudaLaunchKernelEx(&cfg, kern, a);
  }
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

}  // namespace

// Scores and top-K of up to kMaxReindexJobs reindex layers that search the
// same pool, one cluster per (layer, query).  Returns cudaErrorNotSupported,
// having queued nothing, when the pool is larger than 16 x 1024 slots, the
// head count is above 64, or no cluster of the size needed fits the device.
cudaError_t launch_reindex_cluster(const ReindexJobDesc* jobs, int32_t n_jobs, const int32_t* seq_of_query,
                                   const int32_t* pool_idx, const int32_t* pool_cnt, int32_t nq, int32_t H,
                                   int32_t D, int32_t P, int32_t K, int32_t* status, cudaStream_t st) {
  if (n_jobs < 1 || n_jobs > kMaxReindexJobs || nq < 1 || nq > 65535) return cudaErrorInvalidValue;
  if (P < 1 || P > kRcMaxC * kRcSlots || H > 64 || (D != 64 && D != 128)) return cudaErrorNotSupported;
  int C = 1;
  while (C * kRcSlots < P) C <<= 1;
  RcArgs a{};
  for (int j = 0; j < n_jobs; ++j) {
    const ReindexJobDesc& d = jobs[j];
    a.job[j] = RcJob{d.q,      d.w,      static_cast<const uint8_t*>(d.keys->base), d.keys->row_bytes,
                     to_rowmap(*d.keys), d.scores, d.sel_idx, d.sel_cnt};
  }
  a.seq_of_query = seq_of_query;
  a.pool_idx = pool_idx;
  a.pool_cnt = pool_cnt;
  a.H = H;
  a.P = P;
  a.K = K;
  a.nq = nq;
  a.C = C;
  a.status = status;
  const int N = H <= 16 ? 16 : H <= 32 ? 32 : 64;
  if (D == 128) {
    switch (N) {
      case 16: return launch_rc_t<128, 16>(a, n_jobs, st);
      case 32: return launch_rc_t<128, 32>(a, n_jobs, st);
      default: return launch_rc_t<128, 64>(a, n_jobs, st);
    }
  }
  switch (N) {
    case 16: return launch_rc_t<64, 16>(a, n_jobs, st);
    case 32: return launch_rc_t<64, 32>(a, n_jobs, st);
    default: return launch_rc_t<64, 64>(a, n_jobs, st);
  }
}

}  // namespace csa2
