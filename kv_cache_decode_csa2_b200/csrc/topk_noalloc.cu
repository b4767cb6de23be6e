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
#include <mutex>

#include "csa2_device.cuh"
#include "internal.h"

namespace {

constexpr size_t kNoallocScratchBytes = (size_t)CSA2_NOALLOC_SCRATCH_BYTES;

// The shared scratch.  In host code this name is only a host-side handle, not
// a device address: the device address comes from cudaGetSymbolAddress.
static __device__ __align__(256) unsigned char g_topk_scratch[kNoallocScratchBytes];

// The array's device address per device, with the context it was looked up
// in: a device reset (or a new primary context) reloads the module, and the
// array may then sit elsewhere, so a changed context means a new look-up.
struct ScratchAddr {
  CUcontext ctx = nullptr;
  void* addr = nullptr;
};
ScratchAddr g_scratch[64];
std::mutex g_scratch_mu;

typedef CUresult (*CtxGetCurrentFn)(CUcontext*);
CtxGetCurrentFn ctx_get_current_fn() {
  static std::atomic<CtxGetCurrentFn> cached{nullptr};
  CtxGetCurrentFn fn = cached.load(std::memory_order_acquire);
  if (!fn) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult qr;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &qr) == cudaSuccess &&
        qr == cudaDriverEntryPointSuccess) {
      fn = reinterpret_cast<CtxGetCurrentFn>(p);
      cached.store(fn, std::memory_order_release);
    }
  }
  return fn;
}

// The array's address on the current device, looked up the first time the
// entry point runs in this device's current context.
int32_t scratch_for_current_device(void** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return CSA2_ERR_CUDA;
  CtxGetCurrentFn get = ctx_get_current_fn();
  CUcontext ctx = nullptr;
  if (!get || get(&ctx) != CUDA_SUCCESS) return CSA2_ERR_CUDA;
  std::lock_guard<std::mutex> lock(g_scratch_mu);
  ScratchAddr& s = g_scratch[dev];
  if (!ctx || s.ctx != ctx || !s.addr) {
    void* p = nullptr;   // the look-up also makes the device's primary context current if none was
    if (cudaGetSymbolAddress(&p, g_topk_scratch) != cudaSuccess || !p) return CSA2_ERR_CUDA;
    if (!ctx && (get(&ctx) != CUDA_SUCCESS || !ctx)) return CSA2_ERR_CUDA;
    s.ctx = ctx;
    s.addr = p;
  }
  *out = s.addr;
  return CSA2_OK;
}

}  // namespace

extern "C" int32_t csa2_topk_pool_noalloc(const int32_t* scores, int64_t ld, const int32_t* n_valid,
                                          const int32_t* cand_pos, int32_t nq, int32_t n_max, int32_t k,
                                          int32_t* out_idx, int32_t* out_cnt, int32_t* status, void* stream) {
  using namespace csa2;
  CSA2_API_RANGE("csa2_topk_pool_noalloc");
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
