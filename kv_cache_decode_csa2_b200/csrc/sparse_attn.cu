// K4: sparse attention over the FP4 main KV cache.
//
// S = the selected global positions U the window [max(0,pos-W+1), pos], each
// position once ("512 most relevant KV entries, plus a local 128-token
// window": "How DeepSeek V4.1 Flash Actually Works", item 2; FP4 main KV:
// "DeepSeek V4.1-Flash: 552B runs like 16B", Act 3).  Because the selection is
// ascending, S is the selection entries below the window start, followed by
// the window itself, and row j of S has a closed form.
//
// A group of kCl CTAs handles one (layer, query, group of up to 32 heads).
// CTA r of the group takes slice r of the selection entries (entries at or
// above the window start are left to the window) and slice r of the window,
// so no CTA waits for a count of the others.  It gathers each
// row's E2M1 codes and E4M3 scales by position and dequantises them exactly
// into bf16 in shared memory (a value with 2 significant bits times a scale
// with 4 significant bits fits bf16's 8 bits).  Then it computes logits =
// Q K^T and the unnormalised P V on bf16 tensor cores with fp32 accumulation,
// tile by tile with an online softmax, and writes its partial (max, sum, O)
// per head to L2.  When all CTAs of the launch fit on the device at once
// (checked at launch), the group meets at a bounded barrier and CTA r merges
// columns [r D / kCl, (r + 1) D / kCl) of every head; otherwise a merge kernel
// does the same.  Several layers of a plan go into one launch (a job array),
// so independent layers run side by side.
//
// A layer may keep its own cache of the most recent tokens beside the FP4
// main cache ("How DeepSeek V4.1 Flash Actually Works", the three KV-cache
// optimizations, item 3: V4 kept a separate per-layer local KV of the latest
// 128 tokens, and V4.1 keeps it while a session is active).  Its rows are
// bf16, in a ring of R >= window rows per sequence (position p in slot
// p mod R).  The LOCAL instantiation reads the window rows from that ring
// with 16-byte loads and the selection rows from the FP4 cache.
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include "csa2_device.cuh"
#include "internal.h"
#include "select_common.cuh"

namespace csa2 {

CSA2_TRACE_UNIT(attn)

namespace {

constexpr int kCl = 8;       // CTAs per group: row slices of one (layer, query, head group)
constexpr int kTile = 80;    // rows of S per tile (a multiple of 16)
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
};

// A job's local window cache (LOCAL instantiation; base nullptr: none).
struct AttnLocal {
  const uint8_t* base;
  int64_t row_bytes;
  int64_t ring;     // rows per sequence: position p of sequence s is row s ring + p mod ring
  int64_t n_rows;   // rows in the buffer
};

struct AttnArgs {
  AttnJob jobs[kMaxJobs];
  const int32_t* seq_of_query;
  const int32_t* query_pos;
  int32_t nq, Hq, K, window, n_jobs;
  float scale_log2;
  float* part_o;      // [groups][kCl][HG][D]   partial O of every CTA
  float2* part_ml;    // [groups][kCl][HG]      its (max in log2 units, sum)
  uint32_t* bar;      // [groups]               barrier counts (zeroed before a fused launch)
  int32_t fused;      // the group merges in the same launch
  int32_t* status;
  AttnLocal local[kMaxJobs];
};
static_assert(sizeof(AttnArgs) <= 4096, "kernel parameters");

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
  static constexpr int kP = 2 * kTile + 16;        // bytes per P row (bf16)
  static constexpr int kS = kTile + 4;             // floats per logit row
  static constexpr size_t kv = 0;                  // K/V tile; at the end the partial O [HG][D] fp32
  static constexpr size_t qo = kv + (size_t)kTile * kKV;
  static constexpr size_t po = qo + (size_t)HG * kQ;
  static constexpr size_t so = po + (size_t)HG * kP;
  static constexpr size_t mo = so + (size_t)HG * kS * 4;    // [HG][4]: max (log2 units), sum, rescale
  static constexpr size_t pos_o = mo + (size_t)HG * 16;
  static constexpr size_t row_o = pos_o + kTile * 4;
  static constexpr size_t total = row_o + 2 * kTile * 8 + 64;
  static_assert((size_t)(3 * kCl + 2) * HG * 4 <= (size_t)HG * kS * 4, "merge tables fit in the logits");
};

// Merges the kCl partials of group gidx for columns [r CW, r CW + CW) of
// every head: per head the overall max M, the denominator L and the weight
// 2^(m_c - M) / L of every CTA c, then float4 items of the weighted sum.
template <int D, int HG, int NTHR>
__device__ __forceinline__ void merge_slice(const AttnArgs& a, const AttnJob& J, int q, int h0, int gidx, int r,
                                            float* tab) {
  const int tid = threadIdx.x;
  float* mtab = tab;                  // [kCl][HG]
  float* ltab = mtab + kCl * HG;      // [kCl][HG]
  float* ftab = ltab + kCl * HG;      // [kCl][HG]
  float* Mh = ftab + kCl * HG;        // [HG]
  float* Lh = Mh + HG;                // [HG]
  const float2* pml = a.part_ml + (size_t)gidx * kCl * HG;
  for (int i = tid; i < kCl * HG; i += NTHR) {
    const float2 ml = __ldcg(pml + i);
    mtab[i] = ml.x;
    ltab[i] = ml.y;
  }
  __syncthreads();
  if (tid < HG) {
    float M = -INFINITY;
#pragma unroll
    for (int c = 0; c < kCl; ++c) M = fmaxf(M, mtab[c * HG + tid]);
    float Ls = 0.f;
#pragma unroll
    for (int c = 0; c < kCl; ++c) {
      const float mc = mtab[c * HG + tid];
      if (mc != -INFINITY) Ls += exp2f(mc - M) * ltab[c * HG + tid];
    }
    const float inv = Ls > 0.f ? 1.f / Ls : 0.f;
#pragma unroll
    for (int c = 0; c < kCl; ++c) {
      const float mc = mtab[c * HG + tid];
      ftab[c * HG + tid] = mc == -INFINITY ? 0.f : exp2f(mc - M) * inv;
    }
    Mh[tid] = M;
    Lh[tid] = Ls;
  }
  __syncthreads();
  constexpr int CW = D / kCl;
  constexpr int C4 = CW / 4;
  constexpr int F4 = HG * C4;
  const float* po = a.part_o + (size_t)gidx * kCl * HG * D;
  for (int f = tid; f < F4; f += NTHR) {
    const int h = f / C4, col = r * CW + (f % C4) * 4;
    float4 v[kCl];
#pragma unroll
    for (int c = 0; c < kCl; ++c)
      v[c] = __ldcg(reinterpret_cast<const float4*>(po + ((size_t)c * HG + h) * D + col));
    float4 o = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
    for (int c = 0; c < kCl; ++c) {
      const float w = ftab[c * HG + h];
      o.x += w * v[c].x;
      o.y += w * v[c].y;
      o.z += w * v[c].z;
      o.w += w * v[c].w;
    }
    if (h0 + h < a.Hq) {
      const __nv_bfloat162 lo = __floats2bfloat162_rn(o.x, o.y), hi = __floats2bfloat162_rn(o.z, o.w);
      uint2 pk;
      pk.x = *reinterpret_cast<const uint32_t*>(&lo);
      pk.y = *reinterpret_cast<const uint32_t*>(&hi);
      *reinterpret_cast<uint2*>(J.out + ((size_t)q * a.Hq + h0 + h) * D + col) = pk;
    }
  }
  if (r == 0 && tid < HG && h0 + tid < a.Hq && J.lse)
    J.lse[(size_t)q * a.Hq + h0 + tid] = (Mh[tid] + log2f(Lh[tid])) * 0.69314718055994531f;
}

template <int D, int HG, int NTHR, bool LOCAL>
__global__ void __launch_bounds__(NTHR, 1) sparse_attn_kernel(const __grid_constant__ AttnArgs a) {
  using L = AttnSmem<D, HG>;
  constexpr int NW = NTHR / 32;                      // warps
  constexpr int NM = HG / 16;                        // m-tiles (16 heads each)
  constexpr int WPM = NW / NM;                       // warps per m-tile
  constexpr int NTS = kTile / 8;                     // 8-row n-tiles of logits per tile
  constexpr int NTS_W = (NTS + WPM - 1) / WPM;       // of them per warp (at most)
  constexpr int DW = D / WPM;                        // output columns per warp
  constexpr int NT_O = DW / 8;                       // 8-column n-tiles of output per warp
  constexpr int TPH = NTHR / HG;                     // softmax threads per head
  constexpr int RPT = kTile / TPH;                   // rows per softmax thread
  static_assert(kTile % 16 == 0 && kTile % TPH == 0 && NT_O % 2 == 0 && TPH <= 32, "tile shapes");
  extern __shared__ __align__(16) uint8_t sm[];
  uint8_t* kv_s = sm + L::kv;
  uint8_t* q_s = sm + L::qo;
  uint8_t* p_s = sm + L::po;
  float* s_s = reinterpret_cast<float*>(sm + L::so);
  float* ml_s = reinterpret_cast<float*>(sm + L::mo);
  int32_t* pos_s = reinterpret_cast<int32_t*>(sm + L::pos_o);
  int64_t* row_s = reinterpret_cast<int64_t*>(sm + L::row_o);     // [2][kTile]: code row, scale row

  const int rank = blockIdx.x;
  const int gidx = blockIdx.z * gridDim.y + blockIdx.y;   // (job, query, head group)
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int hg = blockIdx.y;
  const int job_i = blockIdx.z / a.nq, q = blockIdx.z % a.nq;
  const AttnJob& J = a.jobs[job_i];
  const int h0 = hg * HG;
  // trace points: 1 Q staged, 2 grid before done, 3 row positions, 4 rows
  // gathered and dequantised, 5 logits, 6 softmax, 7 P V done, 8 partial
  // written, 9 group barrier, 10 merged (3-6: the last tile)
  CSA2_TRACE_BEGIN(kTrAttn, tid == 0);

  // ---- independent loads first: Q rows of this head group, position, count
  constexpr int QPER = HG * (D / 8) / NTHR;
  static_assert(HG * (D / 8) % NTHR == 0, "whole Q items per thread");
  int4 qv[QPER];
#pragma unroll
  for (int i = 0; i < QPER; ++i) {
    const int idx = tid + i * NTHR, h = idx / (D / 8), c = idx % (D / 8);
    qv[i] = h0 + h < a.Hq ? __ldg(reinterpret_cast<const int4*>(J.q + ((size_t)q * a.Hq + h0 + h) * D) + c)
                          : make_int4(0, 0, 0, 0);
  }
  const int32_t pos = __ldg(a.query_pos + q);
  const int32_t seq = a.seq_of_query ? __ldg(a.seq_of_query + q) : q;
#pragma unroll
  for (int i = 0; i < QPER; ++i) {
    const int idx = tid + i * NTHR, h = idx / (D / 8), c = idx % (D / 8);
    *reinterpret_cast<int4*>(q_s + h * L::kQ + c * 16) = qv[i];
  }
  if (tid < HG) {
    ml_s[tid * 4 + 0] = -INFINITY;
    ml_s[tid * 4 + 1] = 0.f;
  }
  CSA2_MARK(kTrAttn, 1, tid == 0);
  pdl_wait();      // the selection comes from the grid before
  pdl_trigger();
  CSA2_MARK(kTrAttn, 2, tid == 0);
  int32_t cnt = J.sel_cnt ? __ldg(J.sel_cnt + q) : a.K;
  if (tid == 0 && rank == 0 && pos < 0) record_error(a.status, CSA2_ERR_INDEX_RANGE);

  // ---- this CTA's rows: selection entries [e0, e1) below the window start,
  // then window offsets [o0, o1)
  cnt = cnt < 0 ? 0 : (cnt > a.K ? a.K : cnt);
  const int32_t wstart = pos - a.window + 1 > 0 ? pos - a.window + 1 : 0;
  const int32_t wlen = pos >= 0 ? pos - wstart + 1 : 0;
  const int32_t Ks = (a.K + kCl - 1) / kCl, Ws = (a.window + kCl - 1) / kCl;
  const int32_t e0 = rank * Ks, o0 = rank * Ws;
  const int32_t ns = (e0 + Ks < cnt ? e0 + Ks : cnt) - e0 > 0 ? (e0 + Ks < cnt ? e0 + Ks : cnt) - e0 : 0;
  const int32_t nw = (o0 + Ws < wlen ? o0 + Ws : wlen) - o0 > 0 ? (o0 + Ws < wlen ? o0 + Ws : wlen) - o0 : 0;
  const int32_t nrows = ns + nw;
  const int32_t* sel = J.sel_idx + (int64_t)q * a.K + e0;

  float acc[NT_O][4];
#pragma unroll
  for (int n = 0; n < NT_O; ++n) acc[n][0] = acc[n][1] = acc[n][2] = acc[n][3] = 0.f;
  const int mt = warp / WPM, wj = warp % WPM;

  for (int32_t t0 = 0; t0 < nrows; t0 += kTile) {
    const int32_t tr = nrows - t0 < kTile ? nrows - t0 : kTile;
    // ---- positions and physical rows of this tile
    if (tid < kTile) {
      int32_t p = -1;
      int64_t cr = -1, sr = -1;
      const int32_t r = t0 + tid;
      if (tid < tr) {
        if (r < ns) {
          p = __ldg(sel + r);
          if (p < 0 || p > pos) {
            record_error(a.status, CSA2_ERR_INDEX_RANGE);
            p = -1;
          } else if (p >= wstart) {
            p = -1;   // inside the window: counted there
          }
        } else {
          p = wstart + o0 + (r - ns);
        }
      }
      bool in_ring = false;   // a window row read from the layer's local cache
      if constexpr (LOCAL) {
        const AttnLocal& lw = a.local[job_i];
        if (p >= 0 && lw.base && r >= ns) {
          in_ring = true;
          const int64_t lr = (int64_t)seq * lw.ring + p % lw.ring;
          if (lr < 0 || lr >= lw.n_rows) {
            record_error(a.status, CSA2_ERR_INDEX_RANGE);
            p = -1;
          } else {
            cr = -2 - lr;   // ring rows are coded below -1; the FP4 pass leaves them to the ring pass
          }
        }
      }
      if (p >= 0 && !in_ring) {
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
      row_s[kTile + tid] = sr;
    }
    __syncthreads();
    CSA2_MARK(kTrAttn, 3, tid == 0);
    // ---- gather + dequantise: one (row, 8-element group) per item, so a warp
    // reads 128 consecutive code bytes of a row and writes 512 consecutive
    // bytes of shared memory.  All loads of a thread are issued before any use.
    {
      constexpr int DPER = kTile * (D / 8) / NTHR;
      static_assert(kTile * (D / 8) % NTHR == 0, "whole items per thread");
      uint32_t cw[DPER];
      uint32_t sb[DPER];
#pragma unroll
      for (int u = 0; u < DPER; ++u) {
        const int i = tid + u * NTHR, r = i / (D / 8), g = i % (D / 8);
        const int64_t cr = row_s[r], sr = row_s[kTile + r];
        cw[u] = cr >= 0 ? __ldg(reinterpret_cast<const uint32_t*>(J.codes + cr * J.codes_rb) + g) : 0u;
        sb[u] = cr >= 0 ? (uint32_t)__ldg(J.scales + sr * J.scales_rb + g / 4) : 0u;
      }
#pragma unroll
      for (int u = 0; u < DPER; ++u) {
        const int i = tid + u * NTHR, r = i / (D / 8), g = i % (D / 8);
        uint32_t packed[4];
        dequant8(cw[u], sb[u], packed);
        *reinterpret_cast<uint4*>(kv_s + r * L::kKV + g * 16) = make_uint4(packed[0], packed[1], packed[2], packed[3]);
      }
      if constexpr (LOCAL) {
        // ring rows: the bf16 values as they are, four 16-byte loads in flight
        // per thread; the same thread wrote zeros at these items just above
        const AttnLocal& lw = a.local[job_i];
        if (lw.base) {
          constexpr int CH = 4;
#pragma unroll
          for (int u0 = 0; u0 < DPER; u0 += CH) {
            int4 v[CH];
            int64_t at[CH];
#pragma unroll
            for (int c = 0; c < CH; ++c) {
              at[c] = -1;
              const int u = u0 + c;
              if (u < DPER) {
                const int i = tid + u * NTHR, r = i / (D / 8), g = i % (D / 8);
                const int64_t cr = row_s[r];
                if (cr <= -2) {
                  v[c] = __ldg(reinterpret_cast<const int4*>(lw.base + (-2 - cr) * lw.row_bytes) + g);
                  at[c] = (int64_t)r * L::kKV + g * 16;
                }
              }
            }
#pragma unroll
            for (int c = 0; c < CH; ++c)
              if (at[c] >= 0) *reinterpret_cast<int4*>(kv_s + at[c]) = v[c];
          }
        }
      }
    }
    __syncthreads();
    CSA2_MARK(kTrAttn, 4, tid == 0);
    // ---- logits: S[h][r] = Q[h] . KV[r]
    {
      // with registers to spare, two accumulators per n-tile (even and odd k)
      // halve the dependent MMA chain
      constexpr int NACC = NTHR <= 256 ? 2 : 1;
      float sacc[2][NTS_W][4];
#pragma unroll
      for (int e = 0; e < 2; ++e)
#pragma unroll
        for (int n = 0; n < NTS_W; ++n) sacc[e][n][0] = sacc[e][n][1] = sacc[e][n][2] = sacc[e][n][3] = 0.f;
      const uint32_t qa = smem_u32(q_s + (mt * 16 + (lane & 15)) * L::kQ + (lane >> 4) * 16);
#pragma unroll 4
      for (int k = 0; k < D / 16; ++k) {
        uint32_t a0, a1, a2, a3;
        ldsm_x4(qa + k * 32, a0, a1, a2, a3);
#pragma unroll
        for (int n = 0; n < NTS_W; ++n) {
          const int nt = wj + n * WPM;
          if (nt < NTS) {
            uint32_t b0, b1;
            const int row = nt * 8 + (lane & 7);
            ldsm_x2(smem_u32(kv_s + row * L::kKV + ((lane >> 3) & 1) * 16 + k * 32), b0, b1);
            mma16816(sacc[NACC == 2 ? (k & 1) : 0][n], a0, a1, a2, a3, b0, b1);
          }
        }
      }
      if (NACC == 2) {
#pragma unroll
        for (int n = 0; n < NTS_W; ++n)
#pragma unroll
          for (int i = 0; i < 4; ++i) sacc[0][n][i] += sacc[1][n][i];
      }
      const int g = lane >> 2, t = lane & 3;
#pragma unroll
      for (int n = 0; n < NTS_W; ++n) {
        const int nt = wj + n * WPM;
        if (nt < NTS) {
          const int c = nt * 8 + 2 * t;
          s_s[(mt * 16 + g) * L::kS + c] = sacc[0][n][0];
          s_s[(mt * 16 + g) * L::kS + c + 1] = sacc[0][n][1];
          s_s[(mt * 16 + g + 8) * L::kS + c] = sacc[0][n][2];
          s_s[(mt * 16 + g + 8) * L::kS + c + 1] = sacc[0][n][3];
        }
      }
    }
    __syncthreads();
    CSA2_MARK(kTrAttn, 5, tid == 0);
    // ---- online softmax: TPH threads per head, RPT rows each
    {
      const int h = tid / TPH, part = tid % TPH;
      float v[RPT];
      float mx = -INFINITY;
#pragma unroll
      for (int i = 0; i < RPT; ++i) {
        const int r = part * RPT + i;
        v[i] = pos_s[r] >= 0 ? s_s[h * L::kS + r] * a.scale_log2 : -INFINITY;
        mx = fmaxf(mx, v[i]);
      }
#pragma unroll
      for (int o = 1; o < TPH; o <<= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
      const float m_old = ml_s[h * 4 + 0], l_old = ml_s[h * 4 + 1];
      const float m_new = fmaxf(m_old, mx);
      const float alpha = m_old == -INFINITY ? 0.f : exp2f(m_old - m_new);
      float sum = 0.f;
      uint16_t* prow = reinterpret_cast<uint16_t*>(p_s + h * L::kP);
#pragma unroll
      for (int i = 0; i < RPT; ++i) {
        const float pr = v[i] == -INFINITY ? 0.f : exp2f(v[i] - m_new);
        const __nv_bfloat16 pb = __float2bfloat16_rn(pr);
        sum += __bfloat162float(pb);      // the denominator uses exactly the weights applied to V
        prow[part * RPT + i] = __bfloat16_as_ushort(pb);
      }
#pragma unroll
      for (int o = 1; o < TPH; o <<= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
      if (part == 0) {
        ml_s[h * 4 + 0] = m_new;
        ml_s[h * 4 + 1] = alpha * l_old + sum;
        ml_s[h * 4 + 2] = alpha;
      }
    }
    __syncthreads();
    CSA2_MARK(kTrAttn, 6, tid == 0);
    // ---- O[h][d] = alpha[h] O[h][d] + sum_r P[h][r] KV[r][d]
    {
      const int d0 = wj * DW, g = lane >> 2;
      const float al0 = ml_s[(mt * 16 + g) * 4 + 2], al1 = ml_s[(mt * 16 + g + 8) * 4 + 2];
#pragma unroll
      for (int n = 0; n < NT_O; ++n) {
        acc[n][0] *= al0;
        acc[n][1] *= al0;
        acc[n][2] *= al1;
        acc[n][3] *= al1;
      }
      const uint32_t pa = smem_u32(p_s + (mt * 16 + (lane & 15)) * L::kP + (lane >> 4) * 16);
#pragma unroll
      for (int k = 0; k < kTile / 16; ++k) {
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
    }
    // the next tile's position pass ends with a barrier before the K/V tile is rewritten
  }
  CSA2_MARK(kTrAttn, 7, tid == 0);

  // ---- this CTA's partial (max, sum, O) to L2, then the merge of the group
  {
    float* po = a.part_o + ((size_t)gidx * kCl + rank) * HG * D;
    const int d0 = wj * DW, g = lane >> 2, t = lane & 3;
#pragma unroll
    for (int half = 0; half < 2; ++half) {
      float* row = po + (size_t)(mt * 16 + g + half * 8) * D + d0 + 2 * t;
#pragma unroll
      for (int n = 0; n < NT_O; ++n)
        *reinterpret_cast<float2*>(row + n * 8) = make_float2(acc[n][2 * half], acc[n][2 * half + 1]);
    }
    if (tid < HG) a.part_ml[((size_t)gidx * kCl + rank) * HG + tid] = make_float2(ml_s[tid * 4], ml_s[tid * 4 + 1]);
  }
  CSA2_MARK(kTrAttn, 8, tid == 0);
  if (!a.fused) return;
  sel_grid_sync(a.bar + gidx, kCl, a.status);
  CSA2_MARK(kTrAttn, 9, tid == 0);
  merge_slice<D, HG, NTHR>(a, J, q, h0, gidx, rank, s_s);
  CSA2_MARK(kTrAttn, 10, tid == 0);
}

// The merge of every group, when the attention CTAs could not all be resident.
template <int D, int HG, int NTHR>
__global__ void __launch_bounds__(NTHR) attn_merge_kernel(const __grid_constant__ AttnArgs a) {
  using L = AttnSmem<D, HG>;
  __shared__ float tab[(3 * kCl + 2) * HG];
  static_assert((3 * kCl + 2) * HG * 4 <= L::kS * HG * 4, "the same tables as the fused merge");
  const int gidx = blockIdx.z * gridDim.y + blockIdx.y;
  const int job_i = blockIdx.z / a.nq, q = blockIdx.z % a.nq;
  merge_slice<D, HG, NTHR>(a, a.jobs[job_i], q, blockIdx.y * HG, gidx, blockIdx.x, tab);
}

template <int D, int HG, int NTHR, bool LOCAL>
cudaError_t launch_attn_t(AttnArgs& a, cudaStream_t st) {
  using L = AttnSmem<D, HG>;
  static SetupMask done{0};
  static std::atomic<int> max_ctas[64];   // co-resident CTAs per device (0: not yet known)
  cudaError_t e = ensure_smem(sparse_attn_kernel<D, HG, NTHR, LOCAL>, (int)L::total, done);
  if (e != cudaSuccess) return e;
  int dev = 0;
  e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 64 && !max_ctas[dev]) {
    int per_sm = 0;
    e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, sparse_attn_kernel<D, HG, NTHR, LOCAL>, NTHR,
                                                      L::total);
    if (e != cudaSuccess) return e;
    max_ctas[dev] = per_sm * sm_count();
  }
  const dim3 grid(kCl, (a.Hq + HG - 1) / HG, a.nq * a.n_jobs);
  const int64_t ctas = (int64_t)grid.x * grid.y * grid.z;
  a.fused = dev < 64 && ctas <= max_ctas[dev];
  if (a.fused) {
    if (!launch_opts().prezeroed) {
      e = cudaMemsetAsync(a.bar, 0, (size_t)grid.y * grid.z * sizeof(uint32_t), st);
      if (e != cudaSuccess) return e;
    }
    return launch_k(sparse_attn_kernel<D, HG, NTHR, LOCAL>, grid, dim3(NTHR), L::total, st, false,
                    launch_opts().pdl, a);
  }
  sparse_attn_kernel<D, HG, NTHR, LOCAL><<<grid, NTHR, L::total, st>>>(a);
  attn_merge_kernel<D, HG, NTHR><<<grid, NTHR, 0, st>>>(a);
  return cudaGetLastError();
}

}  // namespace

constexpr int kAttnHG = 32;   // heads per group (fewer when Hq is smaller)

size_t attn_scratch_bytes(int32_t nq, int32_t Hq, int32_t D, int32_t K, int32_t window) {
  (void)K, (void)window;
  const int HG = Hq <= 16 ? 16 : kAttnHG;
  const size_t groups = (size_t)nq * ((Hq + HG - 1) / HG);
  // partial O and (max, sum) of every CTA, barrier counts; 256-byte aligned pieces
  return groups * kCl * HG * ((size_t)D * 4 + 8) + groups * 4 + 3 * 256;
}

// The barrier counts inside an attention workspace of n_jobs layers: they must
// be zero before a launch that merges in place.
void attn_bar_region(void* ws, int32_t n_jobs, int32_t nq, int32_t Hq, int32_t D, void** ptr, size_t* bytes) {
  const int HG = Hq <= 16 ? 16 : kAttnHG;
  const size_t groups = (size_t)n_jobs * nq * ((Hq + HG - 1) / HG);
  Carver c(ws);
  c.take<float>(groups * kCl * HG * D);
  c.take<float2>(groups * kCl * HG);
  *ptr = c.take<uint32_t>(groups);
  *bytes = groups * sizeof(uint32_t);
}

// Runs n_jobs attention problems that share shapes, positions and sizes.
cudaError_t launch_sparse_attn_jobs(const AttnJobDesc* jobs, int n_jobs, const int32_t* seq_of_query,
                                    const int32_t* query_pos, int32_t nq, int32_t Hq, int32_t D,
                                    int32_t K, int32_t window, float scale, void* ws, int32_t* status,
                                    cudaStream_t st) {
  if (n_jobs < 1 || n_jobs > kMaxJobs) return cudaErrorInvalidValue;
  AttnArgs a;
  a.seq_of_query = seq_of_query;
  a.query_pos = query_pos;
  a.nq = nq;
  a.Hq = Hq;
  a.K = K;
  a.window = window;
  a.n_jobs = n_jobs;
  a.scale_log2 = scale * 1.4426950408889634f;
  a.status = status;
  bool any_local = false;
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
    const csa2_rows* lk = jobs[j].local_kv;
    a.local[j] = lk && lk->base ? AttnLocal{static_cast<const uint8_t*>(lk->base), lk->row_bytes, lk->seq_rows,
                                            lk->n_rows}
                                : AttnLocal{nullptr, 0, 1, 0};
    any_local |= a.local[j].base != nullptr;
  }
  const int HG = Hq <= 16 ? 16 : kAttnHG;
  const size_t groups = (size_t)n_jobs * nq * ((Hq + HG - 1) / HG);
  Carver c(ws);
  a.part_o = c.take<float>(groups * kCl * HG * D);
  a.part_ml = c.take<float2>(groups * kCl * HG);
  a.bar = c.take<uint32_t>(groups);
  if (any_local) {
    if (D == 512)
      return HG == 16 ? launch_attn_t<512, 16, 256, true>(a, st) : launch_attn_t<512, kAttnHG, 256, true>(a, st);
    return HG == 16 ? launch_attn_t<128, 16, 256, true>(a, st) : launch_attn_t<128, kAttnHG, 256, true>(a, st);
  }
  if (D == 512)
    return HG == 16 ? launch_attn_t<512, 16, 256, false>(a, st) : launch_attn_t<512, kAttnHG, 256, false>(a, st);
  return HG == 16 ? launch_attn_t<128, 16, 256, false>(a, st) : launch_attn_t<128, kAttnHG, 256, false>(a, st);
}

cudaError_t launch_sparse_attn(const uint16_t* q, const csa2_rows& codes, const csa2_rows& scales,
                               const csa2_rows* local_kv, const int32_t* seq_of_query, const int32_t* query_pos,
                               const int32_t* sel_idx, const int32_t* sel_cnt, int32_t nq,
                               int32_t Hq, int32_t D, int32_t K, int32_t window, float scale,
                               uint16_t* out, float* lse, void* ws, size_t /*ws_bytes*/,
                               int32_t* status, cudaStream_t st) {
  AttnJobDesc j{q, &codes, &scales, sel_idx, sel_cnt, out, lse, local_kv};
  return launch_sparse_attn_jobs(&j, 1, seq_of_query, query_pos, nq, Hq, D, K, window, scale, ws,
                                 status, st);
}

}  // namespace csa2
