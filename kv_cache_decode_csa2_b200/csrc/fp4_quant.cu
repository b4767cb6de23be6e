// K7: FP4 cache write.  Each block of 32 values is stored as 32 E2M1 codes
// plus one E4M3 scale (the FP4 main KV cache: "DeepSeek V4.1-Flash: 552B runs
// like 16B", Act 3; "compressed from FP8 (8 bits) to FP4 (4 bits)": "How
// DeepSeek V4.1 Flash Actually Works", item 2).
//
//   scale = E4M3 nearest to amax/6 (ties to even, saturating at 448)
//   code  = E2M1 nearest to x/scale (ties to even, saturating at +-6)
//
// Both roundings are decided by exact comparisons.  |x| (fp32) is compared
// with a product of an E2M1 midpoint (at most 3 significant bits) and the
// scale (4 bits), and amax with 3 * (v_c + v_{c+1}) for adjacent E4M3 values
// (at most 8 bits).  Every such product is exact in fp32, so no division
// rounds.  The result is the nearest code of the exact quotient.
//
// The input is fp32 or bf16 rows (bf16 widens to fp32 exactly, so both give
// the codes of the same values).
#include "csa2_device.cuh"
#include "internal.h"

namespace csa2 {

namespace {

// Non-negative E4M3 value of byte c (0..126).
__device__ __forceinline__ float e4m3_pos(uint32_t c) {
  const uint32_t e = c >> 3, m = c & 7u;
  return e == 0 ? (float)m * 0.001953125f : __int_as_float((int)(((e + 120u) << 23) | (m << 20)));
}

__device__ __forceinline__ uint32_t e4m3_scale_for(float amax) {
  if (amax >= 6.0f * 448.0f) return 0x7Eu;
  // largest c with 6*v(c) <= amax (v is increasing in c)
  uint32_t lo = 0, hi = 126;
  while (lo < hi) {
    const uint32_t mid = (lo + hi + 1) >> 1;
    if (6.0f * e4m3_pos(mid) <= amax) lo = mid; else hi = mid - 1;
  }
  const uint32_t c = lo;
  if (c == 126u) return c;
  const float mid2 = 3.0f * (e4m3_pos(c) + e4m3_pos(c + 1));   // 6 * midpoint, exact
  if (amax > mid2) return c + 1;
  if (amax < mid2) return c;
  return (c & 1u) ? c + 1 : c;
}

__device__ __forceinline__ uint32_t e2m1_code(float x, float s) {
  const float ax = fabsf(x);
  // midpoints between magnitudes 0,.5,1,1.5,2,3,4,6
  const float mids[7] = {0.25f, 0.75f, 1.25f, 1.75f, 2.5f, 3.5f, 5.0f};
  uint32_t idx = 0;
#pragma unroll
  for (int i = 0; i < 7; ++i) {
    const float t = mids[i] * s;
    if (ax > t) idx = i + 1;
    else if (ax == t && idx == (uint32_t)i) idx = (i & 1) ? i + 1 : i;
  }
  return idx == 0 ? 0u : (idx | (x < 0.f ? 8u : 0u));
}

struct QuantArgs {
  const void* x;      // float or bf16 (uint16 bit patterns) rows
  int64_t n_rows, ld_x;
  int32_t D;
  const int32_t* dst_rows;
  uint8_t* codes;
  int64_t ld_codes;
  uint8_t* scales;
  int64_t ld_scales;
  int64_t n_dst_rows;
  int32_t* status;
};

template <bool BF16>
__global__ void __launch_bounds__(256) fp4_quantize_kernel(const QuantArgs a) {
  const int blocks_per_row = a.D / 32;
  const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= a.n_rows * blocks_per_row) return;
  const int64_t r = i / blocks_per_row;
  const int b = (int)(i % blocks_per_row);
  int64_t dr = a.dst_rows ? (int64_t)__ldg(a.dst_rows + r) : r;
  if (dr < 0 || dr >= a.n_dst_rows) {
    record_error(a.status, CSA2_ERR_INDEX_RANGE);
    return;
  }
  float v[32];
  if constexpr (BF16) {
    const uint4* src = reinterpret_cast<const uint4*>(static_cast<const uint16_t*>(a.x) + r * a.ld_x + b * 32);
#pragma unroll
    for (int k = 0; k < 4; ++k) {   // 8 bf16 per load; bf16 bits << 16 is the same value in fp32
      const uint4 u = __ldg(src + k);
      const uint32_t w4[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        v[8 * k + 2 * j] = __uint_as_float(w4[j] << 16);
        v[8 * k + 2 * j + 1] = __uint_as_float(w4[j] & 0xFFFF0000u);
      }
    }
  } else {
    const float4* src = reinterpret_cast<const float4*>(static_cast<const float*>(a.x) + r * a.ld_x + b * 32);
#pragma unroll
    for (int k = 0; k < 8; ++k) {
      const float4 f = __ldg(src + k);
      v[4 * k] = f.x;
      v[4 * k + 1] = f.y;
      v[4 * k + 2] = f.z;
      v[4 * k + 3] = f.w;
    }
  }
  float amax = 0.f;
#pragma unroll
  for (int k = 0; k < 32; ++k) amax = fmaxf(amax, fabsf(v[k]));
  const uint32_t sb = e4m3_scale_for(amax);
  const float s = e4m3_pos(sb);
  uint32_t w[4] = {0, 0, 0, 0};
  if (s > 0.f) {
#pragma unroll
    for (int k = 0; k < 32; ++k) w[k / 8] |= e2m1_code(v[k], s) << (4 * (k % 8));
  }
  *reinterpret_cast<uint4*>(a.codes + dr * a.ld_codes + b * 16) = make_uint4(w[0], w[1], w[2], w[3]);
  a.scales[dr * a.ld_scales + b] = (uint8_t)sb;
}

}  // namespace

cudaError_t launch_fp4_quantize(const void* x, bool bf16, int64_t n_rows, int32_t D, int64_t ld_x,
                                const int32_t* dst_rows, uint8_t* codes, int64_t ld_codes,
                                uint8_t* scales, int64_t ld_scales, int64_t n_dst_rows,
                                int32_t* status, cudaStream_t st) {
  QuantArgs a{x, n_rows, ld_x, D, dst_rows, codes, ld_codes, scales, ld_scales, n_dst_rows, status};
  const int64_t items = n_rows * (D / 32);
  if (items == 0) return cudaSuccess;
  const int64_t grid = (items + 255) / 256;
  if (bf16) fp4_quantize_kernel<true><<<(unsigned)grid, 256, 0, st>>>(a);
  else fp4_quantize_kernel<false><<<(unsigned)grid, 256, 0, st>>>(a);
  return cudaGetLastError();
}

}  // namespace csa2
