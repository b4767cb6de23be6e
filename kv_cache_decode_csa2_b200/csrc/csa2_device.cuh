// Device-side building blocks for the sm_100a kernels of libcsa2: shared-memory
// mbarriers with bounded waits, TMA tile loads, tcgen05 (5th-generation tensor
// core) MMA, TMEM allocation and loads, and the shared-memory matrix
// descriptors that tcgen05.mma reads.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "csa2.h"

namespace csa2 {

// Every spin-wait in these kernels gives up after this many nanoseconds of
// global time.  It then records CSA2_ERR_TIMEOUT and returns.  No correct run
// comes anywhere near this limit.
constexpr uint64_t kWaitLimitNs = 2000000000ull;   // 2 s

__device__ __forceinline__ void record_error(int32_t* status, int32_t code) {
  if (status) atomicCAS(status, 0, code);
}

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ uint64_t global_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

// ------------------------------------------------------------------ tracing
// Phase markers.  The normal build compiles them to nothing.  The traced build
// (-DCSA2_TRACE, libcsa2_trace.so) has one chosen thread of every CTA record
// two values at each marked point: the global timer, and the SM cycles since
// the thread entered the kernel.  They go into a caller-owned table attached
// with csa2_trace_attach(): uint64 [kTraceKernels][kTraceCtas][kTracePhases][2].
// Entries stay zero for points that were not reached, and CTAs past
// kTraceCtas are not recorded.  A later launch of the same kernel overwrites
// the entries of an earlier one.
constexpr int kTraceKernels = 8;
constexpr int kTraceCtas = 1024;
constexpr int kTracePhases = 16;
enum TraceKernel : int { kTrIndex = 0, kTrSelect = 1, kTrReindex = 2, kTrAttn = 3, kTrRowSel = 4, kTrZero = 5,
                          kTrRCluster = 6 };
#ifdef CSA2_TRACE
__device__ __forceinline__ void trace_mark(uint64_t* table, int kernel, int phase, long long t0) {
  const uint32_t cta = blockIdx.x + gridDim.x * (blockIdx.y + gridDim.y * blockIdx.z);
  if (!table || cta >= (uint32_t)kTraceCtas || (uint32_t)phase >= (uint32_t)kTracePhases ||
      (uint32_t)kernel >= (uint32_t)kTraceKernels)
    return;
  uint64_t* e = table + (((size_t)kernel * kTraceCtas + cta) * kTracePhases + phase) * 2;
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  e[0] = t;
  e[1] = (uint64_t)(clock64() - t0);
}
// Once per translation unit with markers, at namespace csa2 scope before its
// kernels: the unit's table pointer and the host function that sets it.
#define CSA2_TRACE_UNIT(name)                               \
  static __device__ uint64_t* trace_table_ = nullptr;       \
  cudaError_t trace_attach_##name(uint64_t* p) {            \
    return cudaMemcpyToSymbol(trace_table_, &p, sizeof(p)); \
  }
// At the top of a kernel (phase 0), then at each marked point; `who` picks the
// recording thread.
#define CSA2_TRACE_BEGIN(kernel, who)        \
  const long long trace_t0_ = clock64();     \
  if (who) trace_mark(trace_table_, kernel, 0, trace_t0_)
#define CSA2_MARK(kernel, phase, who)                                   \
  do {                                                                  \
    if (who) trace_mark(trace_table_, kernel, phase, trace_t0_);        \
  } while (0)
#else
#define CSA2_TRACE_UNIT(name)
#define CSA2_TRACE_BEGIN(kernel, who) ((void)0)
#define CSA2_MARK(kernel, phase, who) ((void)0)
#endif

// Programmatic dependent launch.  pdl_wait() blocks until the grid this one
// depends on has completed and its writes are visible (a no-op when the
// launch has no such dependency); pdl_trigger() lets the next grid of the
// stream be launched early.  Work before pdl_wait() may touch only inputs that
// no earlier grid of the stream writes.
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_trigger() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }

__device__ __forceinline__ bool elect_one() {
  uint32_t pred = 0;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "elect.sync _|p, 0xffffffff;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(pred));
  return pred != 0;
}

// ------------------------------------------------------------------ mbarrier
__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count));
}
__device__ __forceinline__ void fence_mbar_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}
// Makes generic-proxy writes to shared memory visible to the async proxy
// (TMA, tcgen05.mma operand reads).
__device__ __forceinline__ void fence_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}
__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}
__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)),
               "r"(bytes)
               : "memory");
}
__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}
// Waits for the phase with the given parity to complete.  Returns false if the
// CTA-wide abort flag is raised or the time limit passes; the caller then
// stops its loop.
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity,
                                          volatile int32_t* abort_flag,
                                          uint64_t limit_ns = kWaitLimitNs) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = global_ns();
  while (true) {
    if (mbar_try_wait(bar, parity)) return true;
    if (*abort_flag) return false;
    if (global_ns() - t0 > limit_ns) {
      *abort_flag = 1;
      return false;
    }
  }
}

// ------------------------------------------------------------------ TMA
__device__ __forceinline__ void tma_load_2d(void* dst, const CUtensorMap* map, int32_t x,
                                            int32_t y, uint64_t* bar, uint64_t policy) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      ".L2::cache_hint [%0], [%1, {%2, %3}], [%4], %5;" ::"r"(smem_u32(dst)),
      "l"(map), "r"(x), "r"(y), "r"(smem_u32(bar)), "l"(policy)
      : "memory");
}
__device__ __forceinline__ uint64_t l2_policy_evict_first() {
  uint64_t p;
  asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(p));
  return p;
}
__device__ __forceinline__ void prefetch_tensormap(const CUtensorMap* map) {
  asm volatile("prefetch.tensormap [%0];" ::"l"(map) : "memory");
}

// ------------------------------------------------------------------ tcgen05
__device__ __forceinline__ void tmem_alloc(uint32_t* dst_smem, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                   smem_u32(dst_smem)),
               "r"(ncols)
               : "memory");
}
__device__ __forceinline__ void tmem_relinquish() {
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols)
               : "memory");
}
__device__ __forceinline__ void tc_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}
// D[tmem] (+)= A[smem] * B[smem]^T, int8 x int8 -> int32, issued by one thread.
__device__ __forceinline__ void mma_i8(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc,
                                       uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::i8 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}
// D[tmem] (+)= A[smem] * B[smem]^T, bf16 x bf16 -> fp32, issued by one thread.
__device__ __forceinline__ void mma_bf16(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc,
                                         uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}
// Arrives on `bar` once every tcgen05 operation issued so far by this thread
// has completed.
__device__ __forceinline__ void mma_commit(uint64_t* bar) {
  asm volatile(
      "tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
          smem_u32(bar))
      : "memory");
}
__device__ __forceinline__ void tmem_wait_ld() {
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}

#define CSA2_R8(i) "=r"(r[i]), "=r"(r[i + 1]), "=r"(r[i + 2]), "=r"(r[i + 3]), \
                   "=r"(r[i + 4]), "=r"(r[i + 5]), "=r"(r[i + 6]), "=r"(r[i + 7])
// Warp-collective: thread t receives 32 consecutive 32-bit columns of TMEM lane
// (lane base of taddr) + t.
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
      "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
      "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
      : CSA2_R8(0), CSA2_R8(8), CSA2_R8(16), CSA2_R8(24)
      : "r"(taddr));
}
__device__ __forceinline__ void tmem_ld16(uint32_t taddr, uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
      "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
      : CSA2_R8(0), CSA2_R8(8)
      : "r"(taddr));
}
#undef CSA2_R8

// Shared-memory matrix descriptor for a K-major operand tile whose rows are
// `row_bytes` (64 or 128) long and which TMA (or our own stores) laid out with
// the matching 64B/128B swizzle.  An 8-row swizzle atom spans 8*row_bytes
// bytes (the stride-dimension offset).  The tile base must be aligned to the
// atom.  Bits: start>>4 [0,14), leading offset>>4 [16,30) (unused when
// swizzled, set to 1), stride offset>>4 [32,46), version 1 [46,48), layout
// type [61,64) (2 = 128B swizzle, 4 = 64B swizzle).
__device__ __forceinline__ uint64_t smem_desc_kmajor(uint32_t saddr, uint32_t row_bytes) {
  const uint64_t layout = (row_bytes == 128) ? 2ull : 4ull;
  const uint64_t sbo = (8ull * row_bytes) >> 4;
  return (uint64_t)((saddr & 0x3FFFFu) >> 4) | (1ull << 16) | (sbo << 32) | (1ull << 46) |
         (layout << 61);
}

// Instruction descriptor for kind::i8 (s8 x s8 -> s32), both operands K-major.
__host__ __device__ constexpr uint32_t idesc_i8(uint32_t M, uint32_t N) {
  return (2u << 4)            // D format: s32
         | (1u << 7)          // A: signed 8-bit
         | (1u << 10)         // B: signed 8-bit
         | ((N >> 3) << 17)   // N / 8
         | ((M >> 4) << 24);  // M / 16
}
// Instruction descriptor for kind::f16 with bf16 inputs and fp32 accumulation.
// a_mn / b_mn select MN-major operands.
__host__ __device__ constexpr uint32_t idesc_bf16(uint32_t M, uint32_t N, uint32_t a_mn,
                                                  uint32_t b_mn) {
  return (1u << 4)            // D format: f32
         | (1u << 7)          // A: bf16
         | (1u << 10)         // B: bf16
         | (a_mn << 15) | (b_mn << 16) | ((N >> 3) << 17) | ((M >> 4) << 24);
}

// Offset of the 16-byte chunk `c` of row `r` in a K-major tile stored with
// the 128B (row_bytes 128) or 64B (row_bytes 64) swizzle.
__host__ __device__ __forceinline__ uint32_t swizzled_chunk(uint32_t r, uint32_t c,
                                                            uint32_t row_bytes) {
  return row_bytes == 128 ? r * 128u + ((c ^ (r & 7u)) << 4)
                          : r * 64u + ((c ^ ((r >> 1) & 3u)) << 4);
}

// ------------------------------------------------------------------ scores
// 13-bit bucket, non-decreasing in the score, used by the radix top-k.
// Non-negative scores map to 4096 + f(s); negative ones to 4095 - f(-s-1).
// f keeps the position of the leading bit and the 7 bits below it, so for
// s >= 128 a bucket spans 2^(e-7) consecutive scores, where e is the leading bit.
__host__ __device__ __forceinline__ uint32_t score_f(uint32_t s) {
  if (s < 128u) return s;
#ifdef __CUDA_ARCH__
  const uint32_t e = 31u - __clz(s);
#else
  const uint32_t e = 31u - __builtin_clz(s);
#endif
  return (e - 6u) * 128u + ((s >> (e - 7u)) & 127u);
}
__host__ __device__ __forceinline__ uint32_t score_bucket(int32_t s) {
  return s >= 0 ? 4096u + score_f((uint32_t)s) : 4095u - score_f((uint32_t)(-(s + 1)));
}
constexpr int kBuckets = 8192;
// The smallest score whose bucket is >= b (the bucket is monotone in the
// score), by binary search; INT32_MAX if no score reaches bucket b, and
// INT32_MIN for b <= 0.
__host__ __device__ __forceinline__ int32_t bucket_min_score(int32_t b) {
  if (b <= 0) return INT32_MIN;
  if (b >= kBuckets) return INT32_MAX;
  int64_t lo = INT32_MIN, hi = INT32_MAX;   // invariant: bucket(hi) >= b
  if ((int32_t)score_bucket(INT32_MAX) < b) return INT32_MAX;
  while (lo + 1 < hi) {
    const int64_t mid = lo + (hi - lo) / 2;
    if ((int32_t)score_bucket((int32_t)mid) >= b) hi = mid;
    else lo = mid;
  }
  return (int32_t)hi;
}

// Ordering key of a candidate: larger key = better (higher score, then lower
// position).  All keys of distinct positions differ.
__host__ __device__ __forceinline__ uint64_t cand_key(int32_t score, int32_t pos) {
  return ((uint64_t)((uint32_t)score ^ 0x80000000u) << 32) | (uint64_t)(0xFFFFFFFFu - (uint32_t)pos);
}
__host__ __device__ __forceinline__ int32_t key_pos(uint64_t key) {
  return (int32_t)(0xFFFFFFFFu - (uint32_t)key);
}
__host__ __device__ __forceinline__ int32_t key_score(uint64_t key) {
  return (int32_t)((uint32_t)(key >> 32) ^ 0x80000000u);
}

// Physical row of position `pos` of sequence `seq` in a csa2_rows view;
// -1 if the page table entry or the row is out of range.
struct RowMap {
  const int32_t* page_table;
  int64_t n_rows;
  int64_t seq_rows;
  int32_t page_rows;
  int32_t max_pages;
};
__device__ __forceinline__ int64_t map_row(const RowMap& m, int32_t seq, int32_t pos) {
  int64_t r;
  if (m.page_table) {
    const int32_t pg = pos / m.page_rows;
    if (pg >= m.max_pages) return -1;
    const int32_t phys = __ldg(m.page_table + (int64_t)seq * m.max_pages + pg);
    r = (int64_t)phys * m.page_rows + (pos - pg * m.page_rows);
    if (phys < 0) return -1;
  } else {
    r = (int64_t)seq * m.seq_rows + pos;
  }
  return (r >= 0 && r < m.n_rows) ? r : -1;
}
inline RowMap to_rowmap(const csa2_rows& v) {
  return RowMap{v.page_table, v.n_rows, v.seq_rows, v.page_rows, v.max_pages};
}

}  // namespace csa2
