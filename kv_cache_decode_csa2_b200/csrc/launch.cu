// Kernel launches with optional cooperative and programmatic-dependence
// attributes, and the per-thread launch options of a layer-plan call.
#include "csa2_device.cuh"
#include "internal.h"

namespace csa2 {

CSA2_TRACE_UNIT(zero)

namespace {
thread_local LaunchOpts t_opts;
// Set when a launch with the programmatic-serialisation attribute failed and
// the same launch without it succeeded: later launches leave it out.
std::atomic<bool> g_pdl_off{false};
}  // namespace

LaunchOpts& launch_opts() { return t_opts; }

cudaError_t launch_ex(const void* kernel, void** args, dim3 grid, dim3 block, size_t smem, cudaStream_t st,
                      bool cooperative, bool pdl) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[2];
  int n = 0;
  if (cooperative) {
    attr[n].id = cudaLaunchAttributeCooperative;
    attr[n].val.cooperative = 1;
    ++n;
  }
  const bool use_pdl = pdl && !g_pdl_off.load(std::memory_order_relaxed);
  if (use_pdl) {
    attr[n].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[n].val.programmaticStreamSerializationAllowed = 1;
    ++n;
  }
  cfg.attrs = attr;
  cfg.numAttrs = n;
  cudaError_t e = cudaLaunchKernelExC(&cfg, kernel, args);
  if (e != cudaSuccess && use_pdl) {   // retry without the programmatic attribute (the last one)
    (void)cudaGetLastError();
    cfg.numAttrs = n - 1;
    e = cudaLaunchKernelExC(&cfg, kernel, args);
    if (e == cudaSuccess) g_pdl_off.store(true, std::memory_order_relaxed);
  }
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

namespace {
struct ZeroArgs {
  uint32_t* ptr[kMaxZeroRegions];
  uint32_t words[kMaxZeroRegions];
  int32_t n;
};
// The grid after it (the index-score kernel of a plan step) may launch at
// once: it touches these regions only after its programmatic wait, which
// returns when this grid has finished and its writes are visible.
__global__ void __launch_bounds__(256) zero_kernel(const __grid_constant__ ZeroArgs a) {
  pdl_trigger();
  CSA2_TRACE_BEGIN(kTrZero, threadIdx.x == 0);   // trace point 1: done
  for (int r = 0; r < a.n; ++r)
    for (uint32_t i = blockIdx.x * 256 + threadIdx.x; i < a.words[r]; i += gridDim.x * 256) a.ptr[r][i] = 0u;
  CSA2_MARK(kTrZero, 1, threadIdx.x == 0);
}
}  // namespace

cudaError_t launch_zero(void* const* ptrs, const size_t* bytes, int n, cudaStream_t st) {
  if (n < 0 || n > kMaxZeroRegions) return cudaErrorInvalidValue;
  ZeroArgs a{};
  size_t most = 0;
  for (int i = 0; i < n; ++i) {
    a.ptr[i] = static_cast<uint32_t*>(ptrs[i]);
    a.words[i] = (uint32_t)(bytes[i] / 4);
    most = a.words[i] > most ? a.words[i] : most;
  }
  a.n = n;
  const int grid = (int)((most + 255) / 256 < 64 ? (most + 255) / 256 : 64);
  zero_kernel<<<grid > 0 ? grid : 1, 256, 0, st>>>(a);
  return cudaGetLastError();
}

}  // namespace csa2
