// Combine of partial attention results over disjoint row sets.
//
// When the context of a sequence is split over R parts (one per GPU of a
// context-sharded decode, or several launches on one GPU), each part attends
// to the rows of the attention set it holds and returns, per query head, its
// output o_r (the softmax-weighted sum over its rows) and its log-sum-exp
// lse_r (natural log of the sum of exp(logit) over its rows).  Attention over
// the union of the rows is then
//     LSE = log sum_r exp(lse_r),   o = sum_r exp(lse_r - LSE) o_r,
// because softmax over the union is each part's softmax rescaled by its share
// of the total mass.  A part with no row has lse_r = -inf and weight 0.
//
// One warp per (query, head): the R partial rows are read with 16-byte loads
// (8 bf16 per lane per load), combined in fp32, written once as bf16.
#include <cuda_bf16.h>

#include "csa2_device.cuh"
#include "internal.h"

namespace csa2 {

namespace {

struct CombineArgs {
  const uint16_t* o;      // [R][nq][Hq][D] bf16
  const float* lse;       // [R][nq][Hq]
  int32_t R, rows, D;     // rows = nq * Hq
  uint16_t* out;          // [nq][Hq][D] bf16
  float* lse_out;         // [nq][Hq] or nullptr
};

constexpr int kCombineMaxChunks = 4;   // 16-byte chunks per lane: D <= 32 * 8 * 4 = 1024

__global__ void __launch_bounds__(256) attn_combine_kernel(const __grid_constant__ CombineArgs a) {
  const int warp = (int)((blockIdx.x * 256 + threadIdx.x) >> 5), lane = threadIdx.x & 31;
  if (warp >= a.rows) return;
  // the total mass: M = max_r lse_r, L = sum_r exp(lse_r - M)
  float M = -INFINITY;
  for (int r = lane; r < a.R; r += 32) M = fmaxf(M, __ldg(a.lse + (size_t)r * a.rows + warp));
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, o));
  float L = 0.f;
  if (M != -INFINITY)
    for (int r = lane; r < a.R; r += 32) {
      const float l = __ldg(a.lse + (size_t)r * a.rows + warp);
      if (l != -INFINITY) L += expf(l - M);
    }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) L += __shfl_xor_sync(0xffffffffu, L, o);
  const float inv = L > 0.f ? 1.f / L : 0.f;
  const int chunks = a.D / 8;   // 16-byte chunks of a row
  float acc[kCombineMaxChunks][8];
#pragma unroll
  for (int c = 0; c < kCombineMaxChunks; ++c)
#pragma unroll
    for (int e = 0; e < 8; ++e) acc[c][e] = 0.f;
  for (int r = 0; r < a.R; ++r) {
    const float l = __ldg(a.lse + (size_t)r * a.rows + warp);
    if (l == -INFINITY || M == -INFINITY) continue;   // warp-uniform
    const float wgt = expf(l - M) * inv;
    const uint4* src = reinterpret_cast<const uint4*>(a.o + ((size_t)r * a.rows + warp) * a.D);
#pragma unroll
    for (int c = 0; c < kCombineMaxChunks; ++c) {
      const int ch = lane + 32 * c;
      if (ch < chunks) {
        const uint4 v = __ldg(src + ch);
        const uint32_t w4[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const __nv_bfloat162 b = *reinterpret_cast<const __nv_bfloat162*>(&w4[e]);
          const float2 f = __bfloat1622float2(b);
          acc[c][2 * e] += wgt * f.x;
          acc[c][2 * e + 1] += wgt * f.y;
        }
      }
    }
  }
  uint4* dst = reinterpret_cast<uint4*>(a.out + (size_t)warp * a.D);
#pragma unroll
  for (int c = 0; c < kCombineMaxChunks; ++c) {
    const int ch = lane + 32 * c;
    if (ch < chunks) {
      uint32_t w4[4];
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const __nv_bfloat162 b = __floats2bfloat162_rn(acc[c][2 * e], acc[c][2 * e + 1]);
        w4[e] = *reinterpret_cast<const uint32_t*>(&b);
      }
      dst[ch] = make_uint4(w4[0], w4[1], w4[2], w4[3]);
    }
  }
  if (lane == 0 && a.lse_out) a.lse_out[warp] = M == -INFINITY ? -INFINITY : M + logf(L);
}

}  // namespace

cudaError_t launch_attn_combine(const uint16_t* o, const float* lse, int32_t R, int32_t nq, int32_t Hq, int32_t D,
                                uint16_t* out, float* lse_out, cudaStream_t st) {
  if (D % 8 || D > 32 * 8 * kCombineMaxChunks) return cudaErrorInvalidValue;
  CombineArgs a{o, lse, R, nq * Hq, D, out, lse_out};
  const int64_t threads = (int64_t)a.rows * 32;
  const int grid = (int)((threads + 255) / 256);
  attn_combine_kernel<<<grid, 256, 0, st>>>(a);
  return cudaGetLastError();
}

}  // namespace csa2
