// K4: sparse attention over the FP4 main KV cache.
//
// S = the selected global positions U the window [max(0,pos-W+1), pos], each
// position once ("512 most relevant KV entries, plus a local 128-token
// window": "How DeepSeek V4.1 Flash Actually Works", item 2; FP4 main KV:
// "DeepSeek V4.1-Flash: 552B runs like 16B", Act 3).  Because the selection is
// ascending, S is the selection entries below the window start, followed by
// the window itself, and row j of S has a closed form.
//
// One CTA handles 64 rows of S for up to 64 query heads of one (layer,
// query).  It gathers each row's E2M1 codes and E4M3 scales by position and
// dequantises them exactly into bf16 in shared memory (a value with 2
// significant bits times a scale with 4 significant bits fits bf16's 8 bits).
// Then it computes logits = Q K^T and the unnormalised P V on bf16 tensor
// cores with fp32 accumulation, and writes a (max, sum, O) partial per head.
// A combine kernel merges the partials of every (layer, query, head).
// Several layers of a plan go into one launch (a job array), so independent
// layers run side by side.
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include "csa2_device.cuh"
#include "internal.h"

namespace csa2 {

namespace {

constexpr int kRows = 64;        // rows of S per CTA
constexpr int kSelCache = 1024;  // selection entries kept in shared memory per CTA
constexpr int kMaxJobs = kMaxAttnJobs;

struct AttnJob {
  const uint16_t* q;
  const uint8_t* codes;
  int64_t codes_rb;
  RowMap cmap;
  const uint8_t* scales;
  int64_t scales_rb;
  RowMap smap;
  const int32_t* sel_idx;
  const int32_t* sel_cnt;
  uint16_t* out;
  float* lse;
  float* part_o;     // [nq][Hq][n_chunks][D]
  float* part_ml;    // [nq][Hq][n_chunks][2]
};

struct AttnArgs {
  AttnJob jobs[kMaxJobs];
  const int32_t* seq_of_query;
  const int32_t* query_pos;
  int32_t nq, Hq, K, window, n_chunks, n_jobs;
  float scale_log2;
  int32_t* status;
};

// Two E2M1 codes (low nibble = first element) -> f16x2, exactly (every E2M1
// value is an f16 value).
__device__ __forceinline__ uint32_t e2m1x2_to_f16x2(uint32_t byte) {
  uint32_t r;
  asm("{\n\t.reg .b8 t;\n\tcvt.u8.u32 t, %1;\n\tcvt.rn.f16x2.e2m1x2 %0, t;\n\t}" : "=r"(r) : "r"(byte));
  return r;
}
// One E4M3 byte -> the f16x2 pair (s, s), exactly (E4M3 spans 2^-9..448).
__device__ __forceinline__ uint32_t e4m3_to_f16x2_pair(uint32_t byte) {
  uint32_t r;
  const uint16_t two = (uint16_t)(byte | (byte << 8));
  asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(r) : "h"(two));
  return r;
}
// Four packed codes (8 elements) times their block scale -> 4 bf16x2 words.
// The f16 product is exact (at most 6 significant bits, between 2^-10 and
// 2688), and so is its bf16 copy.
__device__ __forceinline__ void dequant8(uint32_t codes, uint32_t scale_byte, uint32_t (&out)[4]) {
  const __half2 s2 = __halves2half2(__ushort_as_half((uint16_t)(e4m3_to_f16x2_pair(scale_byte) & 0xFFFFu)),
                                    __ushort_as_half((uint16_t)(e4m3_to_f16x2_pair(scale_byte) & 0xFFFFu)));
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    const uint32_t h = e2m1x2_to_f16x2((codes >> (8 * e)) & 0xFFu);
    __half2 v = *reinterpret_cast<const __half2*>(&h);
    v = __hmul2(v, s2);
    const float2 f = __half22float2(v);
    const __nv_bfloat162 b = __floats2bfloat162_rn(f.x, f.y);
    out[e] = *reinterpret_cast<const uint32_t*>(&b);
  }
}

__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3) : "r"(addr));
}
__device__ __forceinline__ void ldsm_x2(uint32_t addr, uint32_t& r0, uint32_t& r1) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x2.shared.b16 {%0,%1}, [%2];" : "=r"(r0), "=r"(r1) : "r"(addr));
}
__device__ __forceinline__ void ldsm_x4_t(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3) : "r"(addr));
}
__device__ __forceinline__ void mma16816(float (&c)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                         uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

template <int D, int HG>
struct AttnSmem {
  static constexpr int kKV = 2 * D + 16;           // bytes per K/V row (padded against bank conflicts)
  static constexpr int kQ = 2 * D + 16;            // bytes per Q row
  static constexpr int kP = 2 * kRows + 16;        // bytes per P row (bf16)
  static constexpr int kS = kRows + 4;             // floats per logit row
  static constexpr size_t kv = 0;
  static constexpr size_t qo = kv + (size_t)kRows * kKV;
  static constexpr size_t po = qo + (size_t)HG * kQ;
  static constexpr size_t so = po + (size_t)HG * kP;
  static constexpr size_t mo = so + (size_t)HG * kS * 4;
  static constexpr size_t pos_o = mo + (size_t)HG * 8;
  static constexpr size_t row_o = pos_o + kRows * 4;
  static constexpr size_t sel_o = row_o + 2 * kRows * 8;
  static constexpr size_t total = sel_o + kSelCache * 4 + 64;
};

template <int D, int HG>
__global__ void __launch_bounds__(256, 1) sparse_attn_kernel(const __grid_constant__ AttnArgs a) {
  using L = AttnSmem<D, HG>;
  constexpr int NM = HG / 16;          // m-tiles (16 heads each)
  constexpr int WPM = 8 / NM;          // warps per m-tile
  constexpr int NT_S = 8 / WPM;        // 8-row n-tiles of logits per warp
  constexpr int DW = D / WPM;          // output columns per warp
  constexpr int NT_O = DW / 8;         // 8-column n-tiles of output per warp
  extern __shared__ __align__(16) uint8_t sm[];
  uint8_t* kv_s = sm + L::kv;
  uint8_t* q_s = sm + L::qo;
  uint8_t* p_s = sm + L::po;
  float* s_s = reinterpret_cast<float*>(sm + L::so);
  float* ml_s = reinterpret_cast<float*>(sm + L::mo);     // [HG][2]: running max (log2 units), sum
  int32_t* pos_s = reinterpret_cast<int32_t*>(sm + L::pos_o);
  int64_t* row_s = reinterpret_cast<int64_t*>(sm + L::row_o);     // [2][kRows]: code row, scale row
  int32_t* sel_s = reinterpret_cast<int32_t*>(sm + L::sel_o);     // first kSelCache selection entries
  __shared__ int32_t meta[4];

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int chunk = blockIdx.x, hg = blockIdx.y;
  const int job_i = blockIdx.z / a.nq, q = blockIdx.z % a.nq;
  const AttnJob& J = a.jobs[job_i];
  const int h0 = hg * HG;

  // ---- Every load that does not depend on another is issued first: the Q
  // rows of this head group, the query position and the selection count.
  constexpr int QPER = HG * (D / 8) / 256;
  int4 qv[QPER];
#pragma unroll
  for (int i = 0; i < QPER; ++i) {
    const int idx = tid + i * 256, h = idx / (D / 8), c = idx % (D / 8);
    qv[i] = h0 + h < a.Hq ? __ldg(reinterpret_cast<const int4*>(J.q + ((size_t)q * a.Hq + h0 + h) * D) + c)
                          : make_int4(0, 0, 0, 0);
  }
  const int32_t pos = __ldg(a.query_pos + q);
  int32_t cnt = J.sel_cnt ? __ldg(J.sel_cnt + q) : a.K;
  if (tid == 0) meta[2] = 0;
#pragma unroll
  for (int i = 0; i < QPER; ++i) {
    const int idx = tid + i * 256, h = idx / (D / 8), c = idx % (D / 8);
    *reinterpret_cast<int4*>(q_s + h * L::kQ + c * 16) = qv[i];
  }
  // ---- S = (selection entries below the window start) followed by the window.
  // The selection is ascending, so those entries are a prefix of it.  Count
  // them in parallel, keeping the first kSelCache entries in shared memory
  // for the row positions below.
  cnt = cnt < 0 ? 0 : (cnt > a.K ? a.K : cnt);
  const int32_t wstart = pos - a.window + 1 > 0 ? pos - a.window + 1 : 0;
  __syncthreads();
  {
    const int32_t* sel = J.sel_idx + (int64_t)q * a.K;
    int32_t below = 0;
    for (int base = 0; base < cnt; base += 4 * 256) {
      int32_t v[4];
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int i = base + u * 256 + tid;
        v[u] = i < cnt ? __ldg(sel + i) : 0x7fffffff;
      }
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int i = base + u * 256 + tid;
        below += v[u] < wstart;
        if (i < kSelCache) sel_s[i] = v[u];
      }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) below += __shfl_xor_sync(0xffffffffu, below, o);
    if (lane == 0 && below) atomicAdd(&meta[2], below);
  }
  if (tid == 0 && pos < 0) record_error(a.status, CSA2_ERR_INDEX_RANGE);
  __syncthreads();
  const int32_t nsel = meta[2];
  const int32_t nS = pos >= 0 ? nsel + (pos - wstart + 1) : 0;
  const int32_t r0 = chunk * kRows;
  const int nrows = nS - r0 < kRows ? nS - r0 : kRows;
  const size_t pidx = ((size_t)q * a.Hq) * a.n_chunks + chunk;   // + h * n_chunks
  if (nrows <= 0) {
    for (int h = tid; h < HG && h0 + h < a.Hq; h += blockDim.x) {
      float* ml = J.part_ml + (pidx + (size_t)(h0 + h) * a.n_chunks) * 2;
      ml[0] = -INFINITY;
      ml[1] = 0.f;
    }
    return;
  }
  const int32_t seq = a.seq_of_query ? __ldg(a.seq_of_query + q) : q;

  // ---- positions and physical rows of this chunk's rows
  if (tid < kRows) {
    int32_t p = -1;
    int64_t cr = -1, sr = -1;
    const int j = r0 + tid;
    if (tid < nrows) {
      p = j < nsel ? (j < kSelCache ? sel_s[j] : __ldg(J.sel_idx + (int64_t)q * a.K + j)) : wstart + (j - nsel);
      if (p < 0 || p > pos) {
        record_error(a.status, CSA2_ERR_INDEX_RANGE);
        p = -1;
      }
    }
    if (p >= 0) {
      cr = map_row(J.cmap, seq, p);
      sr = map_row(J.smap, seq, p);
      if (cr < 0 || sr < 0) {
        record_error(a.status, CSA2_ERR_INDEX_RANGE);
        p = -1;
        cr = sr = -1;
      }
    }
    pos_s[tid] = p;
    row_s[tid] = cr;
    row_s[kRows + tid] = sr;
  }
  __syncthreads();
  // ---- gather + dequantise: one (row, 8-element group) per item, so a warp
  // reads 128 consecutive code bytes of a row and writes 512 consecutive bytes
  // of shared memory (no bank conflicts).  All code words and scales of a
  // thread are loaded before any is used.
  {
    constexpr int DPER = kRows * (D / 8) / 256;
    uint32_t cw[DPER];
    uint32_t sb[DPER];
#pragma unroll
    for (int u = 0; u < DPER; ++u) {
      const int i = tid + u * 256, r = i / (D / 8), g = i % (D / 8);
      const int64_t cr = row_s[r], sr = row_s[kRows + r];
      cw[u] = cr >= 0 ? __ldg(reinterpret_cast<const uint32_t*>(J.codes + cr * J.codes_rb) + g) : 0u;
      sb[u] = cr >= 0 ? (uint32_t)__ldg(J.scales + sr * J.scales_rb + g / 4) : 0u;
    }
#pragma unroll
    for (int u = 0; u < DPER; ++u) {
      const int i = tid + u * 256, r = i / (D / 8), g = i % (D / 8);
      uint32_t packed[4];
      dequant8(cw[u], sb[u], packed);
      *reinterpret_cast<uint4*>(kv_s + r * L::kKV + g * 16) = make_uint4(packed[0], packed[1], packed[2], packed[3]);
    }
  }
  __syncthreads();

  // ---- logits: S[h][r] = Q[h] . KV[r]  (tensor cores, fp32 accumulate)
  {
    const int mt = warp / WPM, nt0 = (warp % WPM) * NT_S;
    float acc[NT_S][4];
#pragma unroll
    for (int n = 0; n < NT_S; ++n) acc[n][0] = acc[n][1] = acc[n][2] = acc[n][3] = 0.f;
    const uint32_t qa = smem_u32(q_s + (mt * 16 + (lane & 15)) * L::kQ + (lane >> 4) * 16);
#pragma unroll 4
    for (int k = 0; k < D / 16; ++k) {
      uint32_t a0, a1, a2, a3;
      ldsm_x4(qa + k * 32, a0, a1, a2, a3);
#pragma unroll
      for (int n = 0; n < NT_S; ++n) {
        uint32_t b0, b1;
        const int row = (nt0 + n) * 8 + (lane & 7);
        ldsm_x2(smem_u32(kv_s + row * L::kKV + ((lane >> 3) & 1) * 16 + k * 32), b0, b1);
        mma16816(acc[n], a0, a1, a2, a3, b0, b1);
      }
    }
    const int g = lane >> 2, t = lane & 3;
#pragma unroll
    for (int n = 0; n < NT_S; ++n) {
      const int c = (nt0 + n) * 8 + 2 * t;
      s_s[(mt * 16 + g) * L::kS + c] = acc[n][0];
      s_s[(mt * 16 + g) * L::kS + c + 1] = acc[n][1];
      s_s[(mt * 16 + g + 8) * L::kS + c] = acc[n][2];
      s_s[(mt * 16 + g + 8) * L::kS + c + 1] = acc[n][3];
    }
  }
  __syncthreads();
  // ---- per-head softmax over this chunk (4 threads per head, 16 rows each)
  {
    const int h = tid >> 2, part = tid & 3;
    if (h < HG) {
      float v[16];
      float mx = -INFINITY;
#pragma unroll
      for (int i = 0; i < 16; ++i) {
        const int r = part * 16 + i;
        v[i] = (r < nrows && pos_s[r] >= 0) ? s_s[h * L::kS + r] * a.scale_log2 : -INFINITY;
        mx = fmaxf(mx, v[i]);
      }
      mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 1));
      mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 2));
      float sum = 0.f;
      uint16_t* prow = reinterpret_cast<uint16_t*>(p_s + h * L::kP);
#pragma unroll
      for (int i = 0; i < 16; ++i) {
        const float p = (v[i] == -INFINITY) ? 0.f : exp2f(v[i] - mx);
        const __nv_bfloat16 pb = __float2bfloat16_rn(p);
        sum += __bfloat162float(pb);      // the denominator uses exactly the weights applied to V
        prow[part * 16 + i] = __bfloat16_as_ushort(pb);
      }
      sum += __shfl_xor_sync(0xffffffffu, sum, 1);
      sum += __shfl_xor_sync(0xffffffffu, sum, 2);
      if (part == 0) {
        ml_s[h * 2] = mx;
        ml_s[h * 2 + 1] = sum;
      }
    }
  }
  __syncthreads();
  // ---- O[h][d] = sum_r P[h][r] KV[r][d]
  {
    const int mt = warp / WPM, d0 = (warp % WPM) * DW;
    float acc[NT_O][4];
#pragma unroll
    for (int n = 0; n < NT_O; ++n) acc[n][0] = acc[n][1] = acc[n][2] = acc[n][3] = 0.f;
    const uint32_t pa = smem_u32(p_s + (mt * 16 + (lane & 15)) * L::kP + (lane >> 4) * 16);
#pragma unroll
    for (int k = 0; k < kRows / 16; ++k) {
      uint32_t a0, a1, a2, a3;
      ldsm_x4(pa + k * 32, a0, a1, a2, a3);
      const int vrow = k * 16 + (lane & 7) + ((lane >> 3) & 1) * 8;
#pragma unroll
      for (int n = 0; n < NT_O; n += 2) {
        uint32_t b0, b1, b2, b3;
        const int col = d0 + n * 8 + (lane >> 4) * 8;
        ldsm_x4_t(smem_u32(kv_s + vrow * L::kKV + col * 2), b0, b1, b2, b3);
        mma16816(acc[n], a0, a1, a2, a3, b0, b1);
        mma16816(acc[n + 1], a0, a1, a2, a3, b2, b3);
      }
    }
    const int g = lane >> 2, t = lane & 3;
#pragma unroll
    for (int half = 0; half < 2; ++half) {
      const int h = mt * 16 + g + half * 8;
      if (h0 + h < a.Hq) {
        float* dst = J.part_o + (pidx + (size_t)(h0 + h) * a.n_chunks) * D;
#pragma unroll
        for (int n = 0; n < NT_O; ++n)
          *reinterpret_cast<float2*>(dst + d0 + n * 8 + 2 * t) = make_float2(acc[n][2 * half], acc[n][2 * half + 1]);
      }
    }
  }
  for (int h = tid; h < HG; h += blockDim.x) {
    if (h0 + h < a.Hq) {
      float* ml = J.part_ml + (pidx + (size_t)(h0 + h) * a.n_chunks) * 2;
      ml[0] = ml_s[h * 2];
      ml[1] = ml_s[h * 2 + 1];
    }
  }
}

// Merges the chunk partials of one (job, query, head): o = sum_c 2^(m_c-M) O_c / L.
// Each thread owns 4 output columns; every chunk's (max, sum) and partial
// columns are loaded up front so the loads overlap.
template <int D>
__global__ void __launch_bounds__(D / 4) attn_combine_kernel(const __grid_constant__ AttnArgs a) {
  constexpr int kMaxChunks = 24;
  const int h = blockIdx.x;
  const int job_i = blockIdx.y / a.nq, q = blockIdx.y % a.nq;
  const AttnJob& J = a.jobs[job_i];
  const size_t base = ((size_t)q * a.Hq + h) * a.n_chunks;
  const int d = threadIdx.x * 4;
  float M = -INFINITY;
  float Lsum = 0.f;
  float4 o = make_float4(0.f, 0.f, 0.f, 0.f);
  if (a.n_chunks > kMaxChunks) {   // long selections: plain two-pass loop
    for (int c = 0; c < a.n_chunks; ++c) M = fmaxf(M, J.part_ml[(base + c) * 2]);
    for (int c = 0; c < a.n_chunks; ++c) {
      const float mc = J.part_ml[(base + c) * 2];
      if (mc == -INFINITY) continue;
      const float e = exp2f(mc - M);
      Lsum += e * J.part_ml[(base + c) * 2 + 1];
      const float4 vc = *reinterpret_cast<const float4*>(J.part_o + (base + c) * D + d);
      o.x += e * vc.x;
      o.y += e * vc.y;
      o.z += e * vc.z;
      o.w += e * vc.w;
    }
  } else {
  float m[kMaxChunks], l[kMaxChunks];
  float4 v[kMaxChunks];
#pragma unroll
  for (int c = 0; c < kMaxChunks; ++c) {
    if (c < a.n_chunks) {
      const float2 ml = *reinterpret_cast<const float2*>(J.part_ml + (base + c) * 2);
      m[c] = ml.x;
      l[c] = ml.y;
      v[c] = ml.x == -INFINITY ? make_float4(0.f, 0.f, 0.f, 0.f)
                               : *reinterpret_cast<const float4*>(J.part_o + (base + c) * D + d);
      M = fmaxf(M, ml.x);
    }
  }
#pragma unroll
  for (int c = 0; c < kMaxChunks; ++c) {
    if (c < a.n_chunks && m[c] != -INFINITY) {
      const float e = exp2f(m[c] - M);
      Lsum += e * l[c];
      o.x += e * v[c].x;
      o.y += e * v[c].y;
      o.z += e * v[c].z;
      o.w += e * v[c].w;
    }
  }
  }
  const float inv = Lsum > 0.f ? 1.f / Lsum : 0.f;
  uint16_t* dst = J.out + ((size_t)q * a.Hq + h) * D + d;
  const __nv_bfloat16 b[4] = {__float2bfloat16_rn(o.x * inv), __float2bfloat16_rn(o.y * inv),
                              __float2bfloat16_rn(o.z * inv), __float2bfloat16_rn(o.w * inv)};
  uint2 pk;
  pk.x = (uint32_t)__bfloat16_as_ushort(b[0]) | ((uint32_t)__bfloat16_as_ushort(b[1]) << 16);
  pk.y = (uint32_t)__bfloat16_as_ushort(b[2]) | ((uint32_t)__bfloat16_as_ushort(b[3]) << 16);
  *reinterpret_cast<uint2*>(dst) = pk;
  if (threadIdx.x == 0 && J.lse) J.lse[(size_t)q * a.Hq + h] = (M + log2f(Lsum)) * 0.69314718055994531f;
}

template <int D, int HG>
cudaError_t launch_attn_t(const AttnArgs& a, cudaStream_t st) {
  using L = AttnSmem<D, HG>;
  static unsigned long long done = 0;
  cudaError_t e = ensure_smem(sparse_attn_kernel<D, HG>, (int)L::total, done);
  if (e != cudaSuccess) return e;
  const dim3 grid(a.n_chunks, (a.Hq + HG - 1) / HG, a.nq * a.n_jobs);
  sparse_attn_kernel<D, HG><<<grid, 256, L::total, st>>>(a);
  attn_combine_kernel<D><<<dim3(a.Hq, a.nq * a.n_jobs), D / 4, 0, st>>>(a);
  return cudaGetLastError();
}

}  // namespace

size_t attn_scratch_bytes(int32_t nq, int32_t Hq, int32_t D, int32_t K, int32_t window) {
  const int64_t n_chunks = ((int64_t)K + window + kRows - 1) / kRows;
  return (size_t)nq * Hq * n_chunks * ((size_t)D * 4 + 8) + 1024;
}

// Runs n_jobs attention problems that share shapes, positions and sizes.
cudaError_t launch_sparse_attn_jobs(const AttnJobDesc* jobs, int n_jobs, const int32_t* seq_of_query,
                                    const int32_t* query_pos, int32_t nq, int32_t Hq, int32_t D,
                                    int32_t K, int32_t window, float scale, void* ws, int32_t* status,
                                    cudaStream_t st) {
  if (n_jobs < 1 || n_jobs > kMaxJobs) return cudaErrorInvalidValue;
  AttnArgs a;
  a.n_chunks = (int32_t)(((int64_t)K + window + kRows - 1) / kRows);
  a.seq_of_query = seq_of_query;
  a.query_pos = query_pos;
  a.nq = nq;
  a.Hq = Hq;
  a.K = K;
  a.window = window;
  a.n_jobs = n_jobs;
  a.scale_log2 = scale * 1.4426950408889634f;
  a.status = status;
  Carver c(ws);
  for (int j = 0; j < n_jobs; ++j) {
    AttnJob& J = a.jobs[j];
    J.q = jobs[j].q;
    J.codes = static_cast<const uint8_t*>(jobs[j].codes->base);
    J.codes_rb = jobs[j].codes->row_bytes;
    J.cmap = to_rowmap(*jobs[j].codes);
    J.scales = static_cast<const uint8_t*>(jobs[j].scales->base);
    J.scales_rb = jobs[j].scales->row_bytes;
    J.smap = to_rowmap(*jobs[j].scales);
    J.sel_idx = jobs[j].sel_idx;
    J.sel_cnt = jobs[j].sel_cnt;
    J.out = jobs[j].out;
    J.lse = jobs[j].lse;
    J.part_o = c.take<float>((size_t)nq * Hq * a.n_chunks * D);
    J.part_ml = c.take<float>((size_t)nq * Hq * a.n_chunks * 2);
  }
  const int HG = Hq <= 16 ? 16 : (Hq <= 32 ? 32 : 64);
  if (D == 512) {
    if (HG == 16) return launch_attn_t<512, 16>(a, st);
    if (HG == 32) return launch_attn_t<512, 32>(a, st);
    return launch_attn_t<512, 64>(a, st);
  }
  if (HG == 16) return launch_attn_t<128, 16>(a, st);
  if (HG == 32) return launch_attn_t<128, 32>(a, st);
  return launch_attn_t<128, 64>(a, st);
}

cudaError_t launch_sparse_attn(const uint16_t* q, const csa2_rows& codes, const csa2_rows& scales,
                               const int32_t* seq_of_query, const int32_t* query_pos,
                               const int32_t* sel_idx, const int32_t* sel_cnt, int32_t nq,
                               int32_t Hq, int32_t D, int32_t K, int32_t window, float scale,
                               uint16_t* out, float* lse, void* ws, size_t /*ws_bytes*/,
                               int32_t* status, cudaStream_t st) {
  AttnJobDesc j{q, &codes, &scales, sel_idx, sel_cnt, out, lse};
  return launch_sparse_attn_jobs(&j, 1, seq_of_query, query_pos, nq, Hq, D, K, window, scale, ws,
                                 status, st);
}

}  // namespace csa2
