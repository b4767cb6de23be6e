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

#include "csa2_device.cuh"
#include "internal.h"

namespace csa2 {

namespace {

constexpr int kRows = 64;        // rows of S per CTA
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

__device__ __forceinline__ float e4m3_to_float(uint32_t b) {
  const uint32_t e = (b >> 3) & 15u, m = b & 7u;
  float v = (e == 0) ? (float)m * 0.001953125f                                   // m * 2^-9
                     : __int_as_float((int)(((e + 120u) << 23) | (m << 20)));   // 2^(e-7) * (1 + m/8)
  if (e == 15u && m == 7u) v = __int_as_float(0x7fc00000);
  return (b & 0x80u) ? -v : v;
}

__device__ __forceinline__ float e2m1_to_float(uint32_t c) {
  // magnitudes of codes 0..7: 0, .5, 1, 1.5, 2, 3, 4, 6
  const uint32_t e = (c >> 1) & 3u, m = c & 1u;
  const float mag = (e == 0) ? 0.5f * (float)m : __int_as_float((int)(((e + 126u) << 23) | (m << 22)));
  return (c & 8u) ? -mag : mag;
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
  static constexpr size_t total = pos_o + kRows * 4 + 64;
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
  __shared__ int32_t meta[4];

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int chunk = blockIdx.x, hg = blockIdx.y;
  const int job_i = blockIdx.z / a.nq, q = blockIdx.z % a.nq;
  const AttnJob& J = a.jobs[job_i];
  const int h0 = hg * HG;

  if (tid == 0) {
    const int32_t pos = __ldg(a.query_pos + q);
    int32_t cnt = J.sel_cnt ? __ldg(J.sel_cnt + q) : a.K;
    cnt = cnt < 0 ? 0 : (cnt > a.K ? a.K : cnt);
    const int32_t ws = pos - a.window + 1 > 0 ? pos - a.window + 1 : 0;
    int l = 0, r = cnt;   // selection entries below the window start
    const int32_t* sel = J.sel_idx + (int64_t)q * a.K;
    while (l < r) {
      const int m = (l + r) >> 1;
      if (__ldg(sel + m) < ws) l = m + 1; else r = m;
    }
    meta[0] = pos;
    meta[1] = ws;
    meta[2] = l;                             // selection rows before the window
    meta[3] = pos >= 0 ? l + (pos - ws + 1) : 0;   // |S|
    if (pos < 0) record_error(a.status, CSA2_ERR_INDEX_RANGE);
  }
  __syncthreads();
  const int32_t pos = meta[0], wstart = meta[1], nsel = meta[2], nS = meta[3];
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

  // ---- positions of this chunk's rows
  if (tid < kRows) {
    int32_t p = -1;
    const int j = r0 + tid;
    if (tid < nrows) {
      p = j < nsel ? __ldg(J.sel_idx + (int64_t)q * a.K + j) : wstart + (j - nsel);
      if (p < 0 || p > pos) {
        record_error(a.status, CSA2_ERR_INDEX_RANGE);
        p = -1;
      }
    }
    pos_s[tid] = p;
  }
  // ---- Q rows of this head group
  for (int i = tid; i < HG * (D / 8); i += blockDim.x) {
    const int h = i / (D / 8), c = i % (D / 8);
    int4 v = make_int4(0, 0, 0, 0);
    if (h0 + h < a.Hq) v = __ldg(reinterpret_cast<const int4*>(J.q + ((size_t)q * a.Hq + h0 + h) * D) + c);
    *reinterpret_cast<int4*>(q_s + h * L::kQ + c * 16) = v;
  }
  __syncthreads();
  // ---- gather + dequantise: one (row, 32-element block) per item
  for (int i = tid; i < kRows * (D / 32); i += blockDim.x) {
    const int r = i / (D / 32), blk = i % (D / 32);
    const int32_t p = pos_s[r];
    uint4 codes = make_uint4(0, 0, 0, 0);
    float sc = 0.f;
    if (p >= 0) {
      const int64_t cr = map_row(J.cmap, seq, p), sr = map_row(J.smap, seq, p);
      if (cr < 0 || sr < 0) {
        record_error(a.status, CSA2_ERR_INDEX_RANGE);
      } else {
        codes = __ldg(reinterpret_cast<const uint4*>(J.codes + cr * J.codes_rb) + blk);
        sc = e4m3_to_float(__ldg(J.scales + sr * J.scales_rb + blk));
      }
    }
    const uint32_t cw[4] = {codes.x, codes.y, codes.z, codes.w};
    uint32_t packed[16];
#pragma unroll
    for (int wv = 0; wv < 4; ++wv)
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const uint32_t byte = (cw[wv] >> (8 * e)) & 0xFFu;
        const __nv_bfloat16 lo = __float2bfloat16_rn(e2m1_to_float(byte & 0xFu) * sc);
        const __nv_bfloat16 hi = __float2bfloat16_rn(e2m1_to_float(byte >> 4) * sc);
        packed[wv * 4 + e] = (uint32_t)__bfloat16_as_ushort(lo) | ((uint32_t)__bfloat16_as_ushort(hi) << 16);
      }
    uint4* dst = reinterpret_cast<uint4*>(kv_s + r * L::kKV + blk * 64);
#pragma unroll
    for (int k = 0; k < 4; ++k) dst[k] = make_uint4(packed[4 * k], packed[4 * k + 1], packed[4 * k + 2], packed[4 * k + 3]);
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
template <int D>
__global__ void __launch_bounds__(D / 4) attn_combine_kernel(const __grid_constant__ AttnArgs a) {
  const int h = blockIdx.x;
  const int job_i = blockIdx.y / a.nq, q = blockIdx.y % a.nq;
  const AttnJob& J = a.jobs[job_i];
  const size_t base = ((size_t)q * a.Hq + h) * a.n_chunks;
  float M = -INFINITY;
  for (int c = 0; c < a.n_chunks; ++c) M = fmaxf(M, J.part_ml[(base + c) * 2]);
  float Lsum = 0.f;
  float4 o = make_float4(0.f, 0.f, 0.f, 0.f);
  const int d = threadIdx.x * 4;
  for (int c = 0; c < a.n_chunks; ++c) {
    const float m = J.part_ml[(base + c) * 2];
    if (m == -INFINITY) continue;
    const float e = exp2f(m - M);
    Lsum += e * J.part_ml[(base + c) * 2 + 1];
    const float4 v = *reinterpret_cast<const float4*>(J.part_o + (base + c) * D + d);
    o.x += e * v.x;
    o.y += e * v.y;
    o.z += e * v.z;
    o.w += e * v.w;
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
