// fb_step_small.cu -- the block step for short blocks on warp-level MMA.
//
// The in-block partial and the merge of the Core Mechanism ("FlashBlock:
// Attention Caching for Efficient Long-Context Block Diffusion", Technical
// Summary §2): for each query row of the active block, softmax attention over
// the block's own S keys (bidirectional), merged in log space with the cached
// block-external pair (O_pre, LSE_pre):
//     m = max(L_pre, L_in),  O = (e^{L_pre-m} O_pre + e^{L_in-m} O_in) / (e^{L_pre-m} + e^{L_in-m}).
//
// With a short block (S <= 64) and few query rows the step is pure latency:
// a 16-row x S-key x 128-dim tile is far too small to pay for tensor-memory
// allocation and mbarrier round trips of tcgen05, so each CTA keeps its whole
// tile in registers and runs it on warp-level mma.sync (m16n8k16, bf16
// operands, f32 accumulators):
//  * a CTA takes 16 packed query rows (token, group head) of one (b, kv head)
//    and the unit's K and V block rows; every global load of the CTA is in
//    flight at once right after the grid-dependency wait (K, V and Q into
//    shared memory rows padded to 272 bytes, so ldmatrix hits distinct banks;
//    the cached O_pre and LSE_pre entries straight into registers);
//  * each of the four warps computes S = Q K^T for all 16 rows and S_pad
//    keys (the whole tile: 16 S_pad 128-term dot products), the softmax of
//    its rows in base 2 with quad shuffles, and then its quarter (32 dims)
//    of O = P V with P taken from the score registers as bf16 A fragments;
//  * the merge in base 2 and bf16 stores of the warp's 32 dims of each row.
#include <cuda_bf16.h>
#include <math_constants.h>

#include <atomic>
#include <cstring>

#include "fb_internal.h"
#include "fb_ptx.cuh"

namespace fb {

namespace {

constexpr int SS_WARPS = 4;
constexpr int SS_THREADS = SS_WARPS * 32;
constexpr int SS_ROWS = 16;                  // packed query rows per CTA: one m16 tile
constexpr int SS_D = 128;
constexpr int SS_MAX_S = 64;
constexpr int SS_ROW_BYTES = SS_D * 2 + 16;  // padded K/V/Q row in shared memory
constexpr float SS_LN2 = 0.6931471805599453f;
constexpr float SS_LOG2E = 1.4426950408889634f;
static_assert(SS_D == 32 * SS_WARPS, "one 32-dim quarter of the output per warp");

struct SmallStepParams {
  int B, Hq, Hkv, G, S;
  float scale_log2;  // softmax scale * log2(e)
  const __nv_bfloat16* Q;   // [B, S, Hq, D]
  const __nv_bfloat16* Kb;  // [B, S, Hkv, D]
  const __nv_bfloat16* Vb;
  const float* pre_o;       // [B, S, Hq, D]
  const float* pre_lse;     // [B, Hq, S] natural log
  __nv_bfloat16* out_o;     // [B, S, Hq, D]
  float* out_lse;           // [B, Hq, S] or null
  // The block append fused into the last step of a block (append != 0): the
  // first CTA of each (b, kv head) writes the block's K/V rows into the cache
  // rows [L_b, L_b + S), L_b = lens[b] read after the dependency wait; a
  // block that does not fit is reported and not written.
  int append;
  CacheGeom cache;
  const int32_t* lens;
  __nv_bfloat16* Kc;
  __nv_bfloat16* Vc;
  int32_t* status;
};

// 16-byte chunk c of block row k into the cache (the append of the block's
// K or V); returns false when the row has no cache row to go to.
__device__ __forceinline__ bool append_chunk(const SmallStepParams& p, __nv_bfloat16* cache, int b, int kvh, int L,
                                             int k, int c, const uint4& v) {
  const long long off = cache_offset(p.cache, b, L + k, kvh);
  if (off < 0) return false;
  *reinterpret_cast<uint4*>(cache + off + c * 8) = v;
  return true;
}

// L_b of the append, or -1 (reported) when the block does not fit.
__device__ __forceinline__ int append_start(const SmallStepParams& p, int b) {
  const int L = p.lens[b];
  if (L < 0 || L + p.S > p.cache.cap) {
    if (threadIdx.x == 0) report(p.status, FB_ERR_BOUNDS);
    return -1;
  }
  return L;
}

// SP: keys padded to a multiple of 16 (16, 32 or 64); keys S .. SP - 1 are
// zero rows in shared memory and masked out of the softmax.
template <int SP>
__global__ void __launch_bounds__(SS_THREADS) block_step_small_kernel(const SmallStepParams p) {
  static_assert(SP % 16 == 0 && SP <= SS_MAX_S, "padded key count");
  __shared__ __align__(16) uint8_t sQ[SS_ROWS * SS_ROW_BYTES];
  __shared__ __align__(16) uint8_t sK[SP * SS_ROW_BYTES];
  __shared__ __align__(16) uint8_t sV[SP * SS_ROW_BYTES];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int rows_unit = p.S * p.G;
  const int cpu = (rows_unit + SS_ROWS - 1) / SS_ROWS;  // CTAs per unit
  const int unit = blockIdx.x / cpu;
  const int b = unit / p.Hkv, kvh = unit % p.Hkv;
  const int pr0 = (blockIdx.x % cpu) * SS_ROWS;
  // the two tile rows of this lane's accumulator entries: lane / 4 and + 8
  bool row_ok[2];
  int row_t[2], row_h[2];
  size_t row_q[2];
#pragma unroll
  for (int i = 0; i < 2; ++i) {
    const int pr = pr0 + (lane >> 2) + 8 * i;
    row_ok[i] = pr < rows_unit;
    row_t[i] = row_ok[i] ? pr / p.G : 0;
    row_h[i] = kvh * p.G + (row_ok[i] ? pr % p.G : 0);
    row_q[i] = ((size_t)b * p.S + row_t[i]) * p.Hq + row_h[i];
  }

  pdl_wait();
  pdl_launch_dependents();

  // ---- every global load of the CTA in flight at once
  constexpr int KCH = SP * 16 / SS_THREADS;       // 16-byte chunks of K (and of V) per thread
  constexpr int QCH = SS_ROWS * 16 / SS_THREADS;  // of Q
  uint4 kr[KCH], vr[KCH], qr[QCH];
#pragma unroll
  for (int j = 0; j < KCH; ++j) {
    const int i = threadIdx.x + j * SS_THREADS;
    const int k = i >> 4, c = i & 15;
    kr[j] = vr[j] = make_uint4(0u, 0u, 0u, 0u);  // padding keys: zero rows (never NaN)
    if (k < p.S) {
      const size_t src = (((size_t)b * p.S + k) * p.Hkv + kvh) * SS_D + c * 8;
      kr[j] = __ldg(reinterpret_cast<const uint4*>(p.Kb + src));
      vr[j] = __ldg(reinterpret_cast<const uint4*>(p.Vb + src));
    }
  }
#pragma unroll
  for (int j = 0; j < QCH; ++j) {
    const int i = threadIdx.x + j * SS_THREADS;
    const int row = i >> 4, c = i & 15;
    const int pr = pr0 + row;
    qr[j] = make_uint4(0u, 0u, 0u, 0u);  // rows past the unit: zero queries, not stored
    if (pr < rows_unit) {
      const size_t q = ((size_t)b * p.S + pr / p.G) * p.Hq + kvh * p.G + pr % p.G;
      qr[j] = __ldg(reinterpret_cast<const uint4*>(p.Q + q * SS_D + c * 8));
    }
  }
  // cached pair of this lane's entries: dims 32 warp + 8 j + 2 (lane % 4) + {0, 1}
  float2 op[2][4];
  float lp[2];
#pragma unroll
  for (int i = 0; i < 2; ++i) {
    lp[i] = -CUDART_INF_F;
#pragma unroll
    for (int j = 0; j < 4; ++j) op[i][j] = make_float2(0.f, 0.f);
    if (row_ok[i]) {
      const float* src = p.pre_o + row_q[i] * SS_D + 32 * warp + 2 * (lane & 3);
#pragma unroll
      for (int j = 0; j < 4; ++j) op[i][j] = __ldg(reinterpret_cast<const float2*>(src + 8 * j));
      lp[i] = __ldg(p.pre_lse + ((size_t)b * p.Hq + row_h[i]) * p.S + row_t[i]);
    }
  }
#pragma unroll
  for (int j = 0; j < KCH; ++j) {
    const int i = threadIdx.x + j * SS_THREADS;
    const int k = i >> 4, c = i & 15;
    *reinterpret_cast<uint4*>(sK + k * SS_ROW_BYTES + c * 16) = kr[j];
    *reinterpret_cast<uint4*>(sV + k * SS_ROW_BYTES + c * 16) = vr[j];
  }
  // (after every load of the CTA is in flight)
  if (p.append && blockIdx.x % cpu == 0) {
    // the last step of a block: this unit's K/V rows join the cache
    const int L = append_start(p, b);
    bool ok = true;
#pragma unroll
    for (int j = 0; j < KCH; ++j) {
      const int i = threadIdx.x + j * SS_THREADS;
      const int k = i >> 4, c = i & 15;
      if (L >= 0 && k < p.S)
        ok = append_chunk(p, p.Kc, b, kvh, L, k, c, kr[j]) && append_chunk(p, p.Vc, b, kvh, L, k, c, vr[j]) && ok;
    }
    if (!ok) report(p.status, FB_ERR_BOUNDS);
  }

#pragma unroll
  for (int j = 0; j < QCH; ++j) {
    const int i = threadIdx.x + j * SS_THREADS;
    *reinterpret_cast<uint4*>(sQ + (i >> 4) * SS_ROW_BYTES + (i & 15) * 16) = qr[j];
  }
  __syncthreads();

  // ---- S = Q K^T over the whole tile (16 rows x SP keys, 8 steps of 16 dims)
  const uint32_t q_base = smem_u32(sQ), k_base = smem_u32(sK), v_base = smem_u32(sV);
  // A fragments: lanes 0-15 address rows 0-15 at the step's first 8 dims,
  // lanes 16-31 the same rows at its last 8
  uint32_t qa[SS_D / 16][4];
#pragma unroll
  for (int kk = 0; kk < SS_D / 16; ++kk)
    ldmatrix_x4(qa[kk], q_base + ((lane & 7) + 8 * ((lane >> 3) & 1)) * SS_ROW_BYTES + (16 * kk + 8 * (lane >> 4)) * 2);
  float sacc[SP / 8][4];
#pragma unroll
  for (int nt = 0; nt < SP / 8; ++nt) sacc[nt][0] = sacc[nt][1] = sacc[nt][2] = sacc[nt][3] = 0.f;
#pragma unroll
  for (int np = 0; np < SP / 16; ++np) {
#pragma unroll
    for (int kk = 0; kk < SS_D / 16; ++kk) {
      // B fragments of key tiles 2 np and 2 np + 1: K rows are the n index,
      // their dims the k index (no transpose)
      uint32_t bf[4];
      ldmatrix_x4(bf, k_base + (16 * np + 8 * (lane >> 4) + (lane & 7)) * SS_ROW_BYTES +
                          (16 * kk + 8 * ((lane >> 3) & 1)) * 2);
      mma_bf16_16816(sacc[2 * np], qa[kk], bf[0], bf[1]);
      mma_bf16_16816(sacc[2 * np + 1], qa[kk], bf[2], bf[3]);
    }
  }

  // ---- softmax of rows lane / 4 (entries 0, 1) and lane / 4 + 8 (entries 2, 3)
  float m[2] = {-CUDART_INF_F, -CUDART_INF_F};
#pragma unroll
  for (int nt = 0; nt < SP / 8; ++nt)
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const int key = 8 * nt + 2 * (lane & 3) + (e & 1);
      sacc[nt][e] = key < p.S ? sacc[nt][e] * p.scale_log2 : -CUDART_INF_F;
      m[e >> 1] = fmaxf(m[e >> 1], sacc[nt][e]);
    }
  float l[2] = {0.f, 0.f};
#pragma unroll
  for (int i = 0; i < 2; ++i) {
    // the four lanes of a quad hold one row
    m[i] = fmaxf(m[i], __shfl_xor_sync(0xffffffffu, m[i], 1));
    m[i] = fmaxf(m[i], __shfl_xor_sync(0xffffffffu, m[i], 2));
  }
#pragma unroll
  for (int nt = 0; nt < SP / 8; ++nt)
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      sacc[nt][e] = exp2f(sacc[nt][e] - m[e >> 1]);  // 0 for the masked keys
      l[e >> 1] += sacc[nt][e];
    }
#pragma unroll
  for (int i = 0; i < 2; ++i) {
    l[i] += __shfl_xor_sync(0xffffffffu, l[i], 1);
    l[i] += __shfl_xor_sync(0xffffffffu, l[i], 2);
  }

  // ---- O_in = P V for this warp's 32 dims (unnormalised)
  float oacc[4][4];
#pragma unroll
  for (int j = 0; j < 4; ++j) oacc[j][0] = oacc[j][1] = oacc[j][2] = oacc[j][3] = 0.f;
#pragma unroll
  for (int kk = 0; kk < SP / 16; ++kk) {
    // the score accumulators of key tiles 2 kk and 2 kk + 1 are the A
    // fragment of this 16-key step
    const uint32_t pa[4] = {pack_bf16x2(sacc[2 * kk][0], sacc[2 * kk][1]),
                            pack_bf16x2(sacc[2 * kk][2], sacc[2 * kk][3]),
                            pack_bf16x2(sacc[2 * kk + 1][0], sacc[2 * kk + 1][1]),
                            pack_bf16x2(sacc[2 * kk + 1][2], sacc[2 * kk + 1][3])};
#pragma unroll
    for (int jp = 0; jp < 2; ++jp) {
      // B fragments of dim tiles 2 jp and 2 jp + 1: V rows are the k index,
      // so the 8 x 8 blocks are transposed on load
      uint32_t bf[4];
      ldmatrix_x4_trans(bf, v_base + (16 * kk + 8 * ((lane >> 3) & 1) + (lane & 7)) * SS_ROW_BYTES +
                                (32 * warp + 16 * jp + 8 * (lane >> 4)) * 2);
      mma_bf16_16816(oacc[2 * jp], pa, bf[0], bf[1]);
      mma_bf16_16816(oacc[2 * jp + 1], pa, bf[2], bf[3]);
    }
  }

  // ---- merge in base 2 (the block always has keys, so l > 0) and store
#pragma unroll
  for (int i = 0; i < 2; ++i) {
    if (!row_ok[i]) continue;
    const float lin2 = m[i] + log2f(l[i]);
    const float lp2 = lp[i] * SS_LOG2E;
    const float M = fmaxf(lp2, lin2);
    const float wp = exp2f(lp2 - M);  // 0 when the prefix is empty (lp = -inf)
    const float wi = exp2f(lin2 - M);
    const float inv_den = 1.f / (wp + wi);
    const float ao = exp2f(m[i] - M) * inv_den;  // = wi / l / den
    const float ap = wp * inv_den;
    __nv_bfloat16* dst = p.out_o + row_q[i] * SS_D + 32 * warp + 2 * (lane & 3);
#pragma unroll
    for (int j = 0; j < 4; ++j)
      *reinterpret_cast<uint32_t*>(dst + 8 * j) = pack_bf16x2(fmaf(ap, op[i][j].x, ao * oacc[j][2 * i]),
                                                              fmaf(ap, op[i][j].y, ao * oacc[j][2 * i + 1]));
    if (warp == 0 && (lane & 3) == 0 && p.out_lse)
      p.out_lse[((size_t)b * p.Hq + row_h[i]) * p.S + row_t[i]] = (M + log2f(wp + wi)) * SS_LN2;
  }
}

// The same step for many query rows: a CTA takes 128 packed rows of one
// (b, kv head), 16 per warp of eight, and each warp runs its own rows over
// all 128 dims (no work repeated across warps).  K, V and Q reach shared
// memory by cp.async (70 KB at 64 keys; two CTAs share an SM, so the batched
// sparse step's 256 CTAs run in one wave, and each unit's K/V block is
// brought in by two CTAs: 13.1 us against 13.9 us with 64 rows per CTA, four
// CTAs per SM).
// The cached O_pre entries are loaded at the start straight into the P V
// accumulators: the merge is taken as one more online-softmax update,
//     M* = max(m, L2_pre),  a = 2^(L2_pre - M*),  P' = 2^(s - M*),
//     O = (a O_pre + P' V) / (a + sum P'),  L2 = M* + log2(a + sum P'),
// which is the merge equation with both weights at most 1, so the O_pre
// loads are in flight with those of K, V and Q.
constexpr int SR_WARPS = 8;
constexpr int SR_THREADS = SR_WARPS * 32;
constexpr int SR_ROWS = 16 * SR_WARPS;  // packed query rows per CTA

template <int SP>
constexpr uint32_t rows_smem_bytes() {
  return (uint32_t)(SR_ROWS + 2 * SP) * SS_ROW_BYTES;
}

template <int SP>
__global__ void __launch_bounds__(SR_THREADS, 16 / SR_WARPS) block_step_rows_kernel(const SmallStepParams p) {
  static_assert(SP % 16 == 0 && SP <= SS_MAX_S, "padded key count");
  extern __shared__ __align__(16) uint8_t rows_smem[];
  uint8_t* sQ = rows_smem;                      // [SR_ROWS][272]
  uint8_t* sK = sQ + SR_ROWS * SS_ROW_BYTES;    // [SP][272]
  uint8_t* sV = sK + SP * SS_ROW_BYTES;         // [SP][272]
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int rows_unit = p.S * p.G;
  const int cpu = (rows_unit + SR_ROWS - 1) / SR_ROWS;  // CTAs per unit
  const int unit = blockIdx.x / cpu;
  const int b = unit / p.Hkv, kvh = unit % p.Hkv;
  const int pr0 = (blockIdx.x % cpu) * SR_ROWS;
  const int wr0 = 16 * warp;  // this warp's first row in the CTA tile
  const int dl = 2 * (lane & 3);
  bool row_ok[2];
  int row_t[2], row_h[2];
  size_t row_q[2];
#pragma unroll
  for (int i = 0; i < 2; ++i) {
    const int pr = pr0 + wr0 + (lane >> 2) + 8 * i;
    row_ok[i] = pr < rows_unit;
    row_t[i] = row_ok[i] ? pr / p.G : 0;
    row_h[i] = kvh * p.G + (row_ok[i] ? pr % p.G : 0);
    row_q[i] = ((size_t)b * p.S + row_t[i]) * p.Hq + row_h[i];
  }

  pdl_wait();
  pdl_launch_dependents();

  // ---- K, V and Q into shared memory (padding keys and rows past the unit
  // zero-filled); the cached pair of this lane's entries into registers:
  // O_pre dims 8 j + 2 (lane % 4) + {0, 1} of the rows lane / 4 (entries 0,
  // 1 of accumulator j) and lane / 4 + 8 (entries 2, 3)
  for (int i = threadIdx.x; i < SP * 16; i += SR_THREADS) {
    const int k = i >> 4, c = i & 15;
    const bool ok = k < p.S;
    const size_t src = ok ? (((size_t)b * p.S + k) * p.Hkv + kvh) * SS_D + c * 8 : 0;
    cp_async16(smem_u32(sK + k * SS_ROW_BYTES + c * 16), p.Kb + src, ok ? 16u : 0u);
    cp_async16(smem_u32(sV + k * SS_ROW_BYTES + c * 16), p.Vb + src, ok ? 16u : 0u);
  }
  for (int i = threadIdx.x; i < SR_ROWS * 16; i += SR_THREADS) {
    const int row = i >> 4, c = i & 15;
    const int pr = pr0 + row;
    const bool ok = pr < rows_unit;
    const size_t q = ok ? ((size_t)b * p.S + pr / p.G) * p.Hq + kvh * p.G + pr % p.G : 0;
    cp_async16(smem_u32(sQ + row * SS_ROW_BYTES + c * 16), p.Q + q * SS_D + c * 8, ok ? 16u : 0u);
  }
  cp_async_commit();
  float lp2[2];
  float oacc[SS_D / 8][4];
#pragma unroll
  for (int i = 0; i < 2; ++i) {
    lp2[i] = row_ok[i] ? __ldg(p.pre_lse + ((size_t)b * p.Hq + row_h[i]) * p.S + row_t[i]) * SS_LOG2E
                       : -CUDART_INF_F;
#pragma unroll
    for (int j = 0; j < SS_D / 8; ++j) {
      const float2 v = row_ok[i] ? __ldg(reinterpret_cast<const float2*>(p.pre_o + row_q[i] * SS_D + 8 * j + dl))
                                 : make_float2(0.f, 0.f);
      oacc[j][2 * i] = v.x;
      oacc[j][2 * i + 1] = v.y;
    }
  }
  cp_async_wait_all();
  __syncthreads();
  if (p.append && blockIdx.x % cpu == 0) {
    // the last step of a block: this unit's K/V rows join the cache
    const int L = append_start(p, b);
    bool ok = true;
    for (int i = threadIdx.x; L >= 0 && i < p.S * 16; i += SR_THREADS) {
      const int k = i >> 4, c = i & 15;
      ok = append_chunk(p, p.Kc, b, kvh, L, k, c, *reinterpret_cast<const uint4*>(sK + k * SS_ROW_BYTES + c * 16)) &&
           append_chunk(p, p.Vc, b, kvh, L, k, c, *reinterpret_cast<const uint4*>(sV + k * SS_ROW_BYTES + c * 16)) &&
           ok;
    }
    if (!ok) report(p.status, FB_ERR_BOUNDS);
  }
  if (pr0 + wr0 >= rows_unit) return;  // this warp has no rows (no barrier follows)

  // ---- S = Q K^T for the warp's 16 rows
  const uint32_t q_base = smem_u32(sQ) + wr0 * SS_ROW_BYTES, k_base = smem_u32(sK), v_base = smem_u32(sV);
  float sacc[SP / 8][4];
#pragma unroll
  for (int nt = 0; nt < SP / 8; ++nt) sacc[nt][0] = sacc[nt][1] = sacc[nt][2] = sacc[nt][3] = 0.f;
#pragma unroll
  for (int kk = 0; kk < SS_D / 16; ++kk) {
    uint32_t qa[4];
    ldmatrix_x4(qa, q_base + ((lane & 7) + 8 * ((lane >> 3) & 1)) * SS_ROW_BYTES + (16 * kk + 8 * (lane >> 4)) * 2);
#pragma unroll
    for (int np = 0; np < SP / 16; ++np) {
      uint32_t bf[4];
      ldmatrix_x4(bf, k_base + (16 * np + 8 * (lane >> 4) + (lane & 7)) * SS_ROW_BYTES +
                          (16 * kk + 8 * ((lane >> 3) & 1)) * 2);
      mma_bf16_16816(sacc[2 * np], qa, bf[0], bf[1]);
      mma_bf16_16816(sacc[2 * np + 1], qa, bf[2], bf[3]);
    }
  }

  // ---- softmax against M* = max(row max, L2_pre) of rows lane / 4
  // (entries 0, 1) and lane / 4 + 8 (entries 2, 3)
  float mx[2] = {-CUDART_INF_F, -CUDART_INF_F};
#pragma unroll
  for (int nt = 0; nt < SP / 8; ++nt)
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const int key = 8 * nt + 2 * (lane & 3) + (e & 1);
      sacc[nt][e] = key < p.S ? sacc[nt][e] * p.scale_log2 : -CUDART_INF_F;
      mx[e >> 1] = fmaxf(mx[e >> 1], sacc[nt][e]);
    }
  float a[2], l[2] = {0.f, 0.f};
#pragma unroll
  for (int i = 0; i < 2; ++i) {
    mx[i] = fmaxf(mx[i], __shfl_xor_sync(0xffffffffu, mx[i], 1));
    mx[i] = fmaxf(mx[i], __shfl_xor_sync(0xffffffffu, mx[i], 2));
    mx[i] = fmaxf(mx[i], lp2[i]);  // M* (finite: the block always has keys)
    a[i] = exp2f(lp2[i] - mx[i]);  // 0 when the prefix is empty
  }
#pragma unroll
  for (int nt = 0; nt < SP / 8; ++nt)
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      sacc[nt][e] = exp2f(sacc[nt][e] - mx[e >> 1]);
      l[e >> 1] += sacc[nt][e];
    }
#pragma unroll
  for (int i = 0; i < 2; ++i) {
    l[i] += __shfl_xor_sync(0xffffffffu, l[i], 1);
    l[i] += __shfl_xor_sync(0xffffffffu, l[i], 2);
  }
#pragma unroll
  for (int j = 0; j < SS_D / 8; ++j)
#pragma unroll
    for (int e = 0; e < 4; ++e) oacc[j][e] *= a[e >> 1];

  // ---- O = a O_pre + P' V over all 128 dims
#pragma unroll
  for (int kk = 0; kk < SP / 16; ++kk) {
    const uint32_t pa[4] = {pack_bf16x2(sacc[2 * kk][0], sacc[2 * kk][1]),
                            pack_bf16x2(sacc[2 * kk][2], sacc[2 * kk][3]),
                            pack_bf16x2(sacc[2 * kk + 1][0], sacc[2 * kk + 1][1]),
                            pack_bf16x2(sacc[2 * kk + 1][2], sacc[2 * kk + 1][3])};
#pragma unroll
    for (int jp = 0; jp < SS_D / 16; ++jp) {
      uint32_t bf[4];
      ldmatrix_x4_trans(bf, v_base + (16 * kk + 8 * ((lane >> 3) & 1) + (lane & 7)) * SS_ROW_BYTES +
                                (16 * jp + 8 * (lane >> 4)) * 2);
      mma_bf16_16816(oacc[2 * jp], pa, bf[0], bf[1]);
      mma_bf16_16816(oacc[2 * jp + 1], pa, bf[2], bf[3]);
    }
  }

  // ---- normalise and store
#pragma unroll
  for (int i = 0; i < 2; ++i) {
    if (!row_ok[i]) continue;
    const float den = a[i] + l[i];  // >= 1: one of the two weights is 2^0
    const float inv = 1.f / den;
    __nv_bfloat16* dst = p.out_o + row_q[i] * SS_D + dl;
#pragma unroll
    for (int j = 0; j < SS_D / 8; ++j)
      *reinterpret_cast<uint32_t*>(dst + 8 * j) = pack_bf16x2(oacc[j][2 * i] * inv, oacc[j][2 * i + 1] * inv);
    if ((lane & 3) == 0 && p.out_lse)
      p.out_lse[((size_t)b * p.Hq + row_h[i]) * p.S + row_t[i]] = (mx[i] + log2f(den)) * SS_LN2;
  }
}

}  // namespace

bool small_step_fits(const fb_desc& d, int num_sms) {
  const long long ctas = (long long)d.batch * d.num_kv_heads *
                         ((d.block_len * (d.num_q_heads / d.num_kv_heads) + SS_ROWS - 1) / SS_ROWS);
  // short blocks whose tiles fit one wave of these CTAs
  return d.dtype == FB_BF16 && d.head_dim == SS_D && d.block_len <= SS_MAX_S && ctas > 0 &&
         ctas <= (long long)num_sms;
}

bool rows_step_fits(const fb_desc& d) {
  return d.dtype == FB_BF16 && d.head_dim == SS_D && d.block_len <= SS_MAX_S && d.batch > 0 && d.block_len > 0;
}

namespace {
SmallStepParams step_params(const fb_desc& d, const void* Q, const void* Kb, const void* Vb, const float* O_pre,
                            const float* LSE_pre, void* O, float* LSE_out, const StepAppend* app) {
  SmallStepParams p;
  std::memset(&p, 0, sizeof(p));
  p.B = d.batch;
  p.Hq = d.num_q_heads;
  p.Hkv = d.num_kv_heads;
  p.G = d.num_q_heads / d.num_kv_heads;
  p.S = d.block_len;
  p.scale_log2 = d.softmax_scale * SS_LOG2E;
  p.Q = static_cast<const __nv_bfloat16*>(Q);
  p.Kb = static_cast<const __nv_bfloat16*>(Kb);
  p.Vb = static_cast<const __nv_bfloat16*>(Vb);
  p.pre_o = O_pre;
  p.pre_lse = LSE_pre;
  p.out_o = static_cast<__nv_bfloat16*>(O);
  p.out_lse = LSE_out;
  if (app) {
    p.append = 1;
    p.cache = geom_of(d);
    p.lens = app->lens;
    p.Kc = static_cast<__nv_bfloat16*>(app->Kc);
    p.Vc = static_cast<__nv_bfloat16*>(app->Vc);
    p.status = app->status;
  }
  return p;
}
}  // namespace

cudaError_t launch_block_step_small(const fb_desc& d, const void* Q, const void* Kb, const void* Vb,
                                    const float* O_pre, const float* LSE_pre, void* O, float* LSE_out,
                                    cudaStream_t stream, const StepAppend* app) {
  const SmallStepParams p = step_params(d, Q, Kb, Vb, O_pre, LSE_pre, O, LSE_out, app);
  const int cpu = (p.S * p.G + SS_ROWS - 1) / SS_ROWS;
  const dim3 grid((unsigned)(p.B * p.Hkv * cpu));
  cudaError_t e;
  if (p.S <= 16)
    e = launch_pdl(block_step_small_kernel<16>, grid, dim3(SS_THREADS), 0, stream, p);
  else if (p.S <= 32)
    e = launch_pdl(block_step_small_kernel<32>, grid, dim3(SS_THREADS), 0, stream, p);
  else
    e = launch_pdl(block_step_small_kernel<64>, grid, dim3(SS_THREADS), 0, stream, p);
  note_launch();
  return e != cudaSuccess ? e : cudaGetLastError();
}

namespace {
template <int SP>
cudaError_t launch_rows(const SmallStepParams& p, dim3 grid, cudaStream_t stream) {
  static std::atomic<bool> configured[64];
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev >= 64 || !configured[dev].load(std::memory_order_acquire)) {
    e = cudaFuncSetAttribute(block_step_rows_kernel<SP>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)rows_smem_bytes<SP>());
    if (e != cudaSuccess) return e;
    if (dev < 64) configured[dev].store(true, std::memory_order_release);
  }
  return launch_pdl(block_step_rows_kernel<SP>, grid, dim3(SR_THREADS), rows_smem_bytes<SP>(), stream, p);
}
}  // namespace

cudaError_t launch_block_step_rows(const fb_desc& d, const void* Q, const void* Kb, const void* Vb,
                                   const float* O_pre, const float* LSE_pre, void* O, float* LSE_out,
                                   cudaStream_t stream, const StepAppend* app) {
  const SmallStepParams p = step_params(d, Q, Kb, Vb, O_pre, LSE_pre, O, LSE_out, app);
  const int cpu = (p.S * p.G + SR_ROWS - 1) / SR_ROWS;
  const dim3 grid((unsigned)(p.B * p.Hkv * cpu));
  cudaError_t e = p.S <= 16 ? launch_rows<16>(p, grid, stream)
                  : p.S <= 32 ? launch_rows<32>(p, grid, stream)
                              : launch_rows<64>(p, grid, stream);
  note_launch();
  return e != cudaSuccess ? e : cudaGetLastError();
}

}  // namespace fb
