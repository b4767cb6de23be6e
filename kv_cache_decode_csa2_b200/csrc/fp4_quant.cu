// K7: FP4 cache write.  Each block of 32 values is stored as 32 E2M1 codes
// plus one E4M3 scale (the FP4 main KV cache: "DeepSeek V4.1-Flash: 552B runs
// like 16B", Act 3; "compressed from FP8 (8 bits) to FP4 (4 bits)": "How
// DeepSeek V4.1 Flash Actually Works", item 2).
//
//   scale = E4M3 nearest to amax/6 (ties to even, saturating at 448)
//   code  = E2M1 nearest to x/scale (ties to even, saturating at +-6)
//
// The scale: the E4M3 code read off amax/6's exponent and top mantissa bits,
// moved to the largest c with 6 v(c) <= amax by exact comparisons, then the
// nearest of c and c+1 decided against 3 (v(c) + v(c+1)), an exact product.
//
// The codes: q = x/scale from one multiply by the reciprocal and two fused
// corrections (the residual x - q s is exact, so q is within half an ulp of
// the quotient plus a term 2^-24 below it, and an exact midpoint stays
// exact), then sm_100's E2M1 conversion (round to nearest, ties to even,
// saturating), two values per instruction.  A quotient that is not a
// midpoint can still round onto one only if the value carries more than 8
// significant bits: for bf16 input it is at least 2^-8 (relative) away from
// every midpoint, for fp32 input a q that lands exactly on a midpoint is
// moved one ulp toward the side the exact residual x - m s gives.  A result
// of magnitude zero is stored as +0.
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
  // a first guess from amax / 6 (approximate), then the exact largest c with 6 v(c) <= amax
  const float y = amax * (1.0f / 6.0f);
  int c;
  if (y < 0.015625f) {   // below the smallest normal 2^-6: v = m 2^-9
    c = (int)(y * 512.0f);
  } else {
    const uint32_t bits = __float_as_uint(y);
    c = (int)((((bits >> 23) - 120u) << 3) | ((bits >> 20) & 7u));
  }
  c = c < 0 ? 0 : (c > 126 ? 126 : c);
  while (c < 126 && 6.0f * e4m3_pos((uint32_t)c + 1) <= amax) ++c;
  while (c > 0 && 6.0f * e4m3_pos((uint32_t)c) > amax) --c;
  if (c == 126) return 126u;
  const float mid2 = 3.0f * (e4m3_pos((uint32_t)c) + e4m3_pos((uint32_t)c + 1));   // 6 * midpoint, exact
  if (amax > mid2) return (uint32_t)c + 1;
  if (amax < mid2) return (uint32_t)c;
  return (c & 1) ? (uint32_t)c + 1 : (uint32_t)c;
}

// x / s, correctly rounded except within 2^-24 (relative) of a rounding
// boundary between two floats; exact whenever the quotient is representable.
__device__ __forceinline__ float quot(float x, float s, float r) {
  const float q0 = x * r;
  return fmaf(fmaf(-q0, s, x), r, q0);
}

// fp32 input only: a quotient on an E2M1 midpoint is moved one ulp toward
// the side of the exact value (the residual x - q s is exact there).
__device__ __forceinline__ float off_midpoint(float q, float x, float s) {
  const float a = fabsf(q);
  const bool mid = a == 0.25f || a == 0.75f || a == 1.25f || a == 1.75f || a == 2.5f || a == 3.5f || a == 5.0f;
  if (!mid) return q;
  const float res = fmaf(-q, s, x);
  return res > 0.f ? nextafterf(q, INFINITY) : (res < 0.f ? nextafterf(q, -INFINITY) : q);
}

// Eight E2M1 codes in one word, element k in nibble k (the conversion puts
// its first operand in the high nibble); magnitude-zero codes lose their sign.
__device__ __forceinline__ uint32_t e2m1x8(const float* y) {
  uint32_t w;
  asm("{ .reg .b8 b0, b1, b2, b3;\n"
      " cvt.rn.satfinite.e2m1x2.f32 b0, %2, %1;\n"
      " cvt.rn.satfinite.e2m1x2.f32 b1, %4, %3;\n"
      " cvt.rn.satfinite.e2m1x2.f32 b2, %6, %5;\n"
      " cvt.rn.satfinite.e2m1x2.f32 b3, %8, %7;\n"
      " mov.b32 %0, {b0, b1, b2, b3}; }"
      : "=r"(w)
      : "f"(y[0]), "f"(y[1]), "f"(y[2]), "f"(y[3]), "f"(y[4]), "f"(y[5]), "f"(y[6]), "f"(y[7]));
  const uint32_t m = w & 0x77777777u;
  const uint32_t nz = (m + 0x77777777u) & 0x88888888u;   // bit 3 of a nibble: its magnitude is not 0
  return w & (0x77777777u | nz);
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
    const float r = 1.0f / s;
#pragma unroll
    for (int k = 0; k < 32; ++k) {
      const float q = quot(v[k], s, r);
      v[k] = BF16 ? q : off_midpoint(q, v[k], s);
    }
#pragma unroll
    for (int k = 0; k < 4; ++k) w[k] = e2m1x8(v + 8 * k);
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
