// K3: reindex scoring.  A reindex layer re-scores only the candidate pool
// ("later layers search only that much smaller pool instead of rescanning
// everything": "DeepSeek V4.1-Flash: 552B runs like 16B", Act 2).
//
// One CTA per (query, 128 pool slots).  The CTA gathers the pool rows of this
// layer's index keys by position into a swizzled K-major tile (16-byte cp.async
// per chunk: a pool row is one 128-byte line).  It runs one tcgen05 int8 MMA
// group, D[128 slots x N heads] in TMEM, and applies the ReLU and head-weight
// epilogue of the full-mode scorer.  The top-K then runs on these P scores in
// shared memory (topk_small).
#include "csa2_device.cuh"
#include "internal.h"

namespace csa2 {

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
  static unsigned long long done = 0;
  cudaError_t e = ensure_smem(reindex_score_kernel<D, N>, (int)smem, done);
  if (e != cudaSuccess) return e;
  const dim3 grid((a.P + 127) / 128, nq);
  reindex_score_kernel<D, N><<<grid, 128, smem, st>>>(a);
  return cudaGetLastError();
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

}  // namespace csa2
