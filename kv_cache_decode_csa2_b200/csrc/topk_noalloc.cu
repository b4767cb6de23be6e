// csa2_topk_pool_noalloc: the exact top-k of csa2_topk_pool for callers that
// cannot allocate device memory.
//
// Some callers of this library own no device allocator.  Examples are plugin
// code inside a host framework that hands it only its input and output
// buffers, and latency-critical serving loops that reserve all device memory
// at start-up because cudaMalloc can block on the device and fragment the
// pool.  Such callers cannot provide the workspace that csa2_topk_pool needs
// for more than 16,384 candidates.  This entry point takes its scratch from
// one fixed array in the library's own device memory instead.  Every GPU that
// loads the library holds the array until the process exits.
#include "csa2_device.cuh"
#include "internal.h"

namespace {

constexpr size_t kNoallocScratchBytes = (size_t)CSA2_NOALLOC_SCRATCH_BYTES;

// The shared scratch.  In host code this name is only a host-side handle, not
// a device address: the device address comes from cudaGetSymbolAddress.
static __device__ __align__(256) unsigned char g_topk_scratch[kNoallocScratchBytes];

std::atomic<void*> g_scratch_addr[64];   // device address of g_topk_scratch, per device id (set-up once)

// Looks up the array's address on the current device the first time the
// entry point runs there.
int32_t scratch_for_current_device(void** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return CSA2_ERR_CUDA;
  if (!g_scratch_addr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_topk_scratch) != cudaSuccess || !p) return CSA2_ERR_CUDA;
    g_scratch_addr[dev] = p;
  }
  *out = g_scratch_addr[dev];
  return CSA2_OK;
}

}  // namespace

extern "C" int32_t csa2_topk_pool_noalloc(const int32_t* scores, int64_t ld, const int32_t* n_valid,
                                          const int32_t* cand_pos, int32_t nq, int32_t n_max, int32_t k,
                                          int32_t* out_idx, int32_t* out_cnt, int32_t* status, void* stream) {
  using namespace csa2;
  if (!out_idx || !status || nq < 1 || n_max < 0 || n_max > (1 << 30) || k < 1 || k > 65536)
    return CSA2_ERR_INVALID_ARG;
  if (n_max > 0 && (!scores || ld < n_max)) return CSA2_ERR_INVALID_ARG;
  if (nq > 65535) return CSA2_ERR_UNSUPPORTED;   // queries index a grid dimension
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (n_max <= kSmallMax)   // the one-CTA path keeps everything in shared memory
    return launch_topk_small(scores, ld, n_valid, cand_pos, nq, n_max, k, out_idx, out_cnt, status, st) ==
                   cudaSuccess
               ? CSA2_OK
               : CSA2_ERR_CUDA;
  if (topk_scratch_bytes(nq, n_max) > kNoallocScratchBytes) return CSA2_ERR_WORKSPACE;
  void* base = nullptr;
  const int32_t r = scratch_for_current_device(&base);
  if (r != CSA2_OK) return r;
  Carver c(base);
  TopkScratch ts = carve_topk(c, nq, n_max);   // the histogram and counters are zeroed by the launcher
  TopkOut o{out_idx, out_cnt, k};
  return launch_topk_large(scores, ld, n_valid, nullptr, cand_pos, nq, n_max, &o, 1, ts, false, status, st) ==
                 cudaSuccess
             ? CSA2_OK
             : CSA2_ERR_CUDA;
}
