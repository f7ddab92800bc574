// fb_step_small.cu -- the block step for short blocks on the CUDA cores.
//
// The in-block partial and the merge of the Core Mechanism ("FlashBlock:
// Attention Caching for Efficient Long-Context Block Diffusion", Technical
// Summary §2): for each query row of the active block, softmax attention over
// the block's own S keys (bidirectional), merged in log space with the cached
// block-external pair (O_pre, LSE_pre):
//     m = max(L_pre, L_in),  O = (e^{L_pre-m} O_pre + e^{L_in-m} O_in) / (e^{L_pre-m} + e^{L_in-m}).
//
// With a short block (S <= 64) and few query rows the step is pure latency:
// the tensor-core kernel runs one CTA per 128-row tile, i.e. a handful of SMs.
// Here one warp takes one query row and a CTA takes eight rows of one
// (b, kv head), so the rows spread over ~all SMs:
//  * the unit's K and V block rows go to shared memory once per CTA (rows
//    padded to 272 bytes, so a warp reading 32 different key rows at the same
//    column hits distinct banks);
//  * scores: lane k owns key k (and k + 32), a 128-term dot product against
//    the query row broadcast from shared memory;
//  * softmax over the lanes with warp shuffles, P kept in fp32;
//  * PV: lane l owns output dims 4l .. 4l+3, the S weights broadcast by
//    shuffle;
//  * merge and the bf16 store of the row (256 contiguous bytes per warp).
#include <cuda_bf16.h>
#include <math_constants.h>

#include "fb_internal.h"
#include "fb_ptx.cuh"

namespace fb {

namespace {

constexpr int SS_WARPS = 8;
constexpr int SS_ROWS_PER_CTA = SS_WARPS;  // query rows of one unit per CTA, one per warp
constexpr int SS_D = 128;
constexpr int SS_MAX_S = 64;
constexpr int SS_ROW_BYTES = SS_D * 2 + 16;  // padded K/V row in shared memory
constexpr float SS_LN2 = 0.6931471805599453f;

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
};

// acc[0..3] += the four bf16 pairs of a . b (one chain per pair)
__device__ __forceinline__ void dot8x4(const uint4& a, const uint4& b, float* acc) {
  const __nv_bfloat162* x = reinterpret_cast<const __nv_bfloat162*>(&a);
  const __nv_bfloat162* y = reinterpret_cast<const __nv_bfloat162*>(&b);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const float2 u = __bfloat1622float2(x[i]);
    const float2 v = __bfloat1622float2(y[i]);
    acc[i] = fmaf(u.x, v.x, fmaf(u.y, v.y, acc[i]));
  }
}

__device__ __forceinline__ void pv_fma(float w, const uint2& v, float4& acc) {
  const float2 v01 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&v.x));
  const float2 v23 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&v.y));
  acc.x = fmaf(w, v01.x, acc.x);
  acc.y = fmaf(w, v01.y, acc.y);
  acc.z = fmaf(w, v23.x, acc.z);
  acc.w = fmaf(w, v23.y, acc.w);
}

__device__ __forceinline__ void pv_step(float w, const uint8_t* vrow, float4& acc) {
  const uint2 v = *reinterpret_cast<const uint2*>(vrow);
  const float2 v01 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&v.x));
  const float2 v23 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&v.y));
  acc.x = fmaf(w, v01.x, acc.x);
  acc.y = fmaf(w, v01.y, acc.y);
  acc.z = fmaf(w, v23.x, acc.z);
  acc.w = fmaf(w, v23.y, acc.w);
}

__global__ void __launch_bounds__(SS_WARPS * 32) block_step_small_kernel(const SmallStepParams p) {
  __shared__ __align__(16) uint8_t sK[SS_MAX_S * SS_ROW_BYTES];
  __shared__ __align__(16) uint8_t sV[SS_MAX_S * SS_ROW_BYTES];
  __shared__ __align__(16) uint4 sQ[SS_WARPS][SS_D / 8];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int rows_unit = p.S * p.G;
  const int cpu = (rows_unit + SS_ROWS_PER_CTA - 1) / SS_ROWS_PER_CTA;  // CTAs per unit
  const int unit = blockIdx.x / cpu;
  const int b = unit / p.Hkv, kvh = unit % p.Hkv;
  const int pr = (blockIdx.x % cpu) * SS_ROWS_PER_CTA + warp;  // this warp's packed row
  const bool has_row = pr < rows_unit;
  const int t = has_row ? pr / p.G : 0, h = kvh * p.G + (has_row ? pr % p.G : 0);
  const size_t qrow = ((size_t)b * p.S + t) * p.Hq + h;

  pdl_wait();
  pdl_launch_dependents();

  // every global load of the CTA in flight at once: the unit's K and V block
  // rows (S x 16 chunks of 16 bytes), this warp's query row, its cached
  // output dims and LSE
  for (int i = threadIdx.x; i < p.S * (SS_D / 8); i += SS_WARPS * 32) {
    const int k = i >> 4, c = i & 15;
    const size_t src = (((size_t)b * p.S + k) * p.Hkv + kvh) * SS_D + c * 8;
    *reinterpret_cast<uint4*>(sK + k * SS_ROW_BYTES + c * 16) = *reinterpret_cast<const uint4*>(p.Kb + src);
    *reinterpret_cast<uint4*>(sV + k * SS_ROW_BYTES + c * 16) = *reinterpret_cast<const uint4*>(p.Vb + src);
  }
  float4 op = make_float4(0.f, 0.f, 0.f, 0.f);
  float lp = -CUDART_INF_F;
  if (has_row) {
    if (lane < 16) sQ[warp][lane] = *reinterpret_cast<const uint4*>(p.Q + qrow * SS_D + lane * 8);
    op = *reinterpret_cast<const float4*>(p.pre_o + qrow * SS_D + lane * 4);
    lp = p.pre_lse[((size_t)b * p.Hq + h) * p.S + t];
  }
  __syncthreads();
  if (!has_row) return;

  // scores of keys lane and lane + 32, in base 2 (four partial chains each);
  // the query row and the key row are read into registers first, so the 16
  // shared-memory loads of each are in flight together
  float s0 = -CUDART_INF_F, s1 = -CUDART_INF_F;
  {
    uint4 qv[SS_D / 8];
#pragma unroll
    for (int c = 0; c < SS_D / 8; ++c) qv[c] = sQ[warp][c];
    auto score = [&](int key) {
      uint4 kv[SS_D / 8];
      const uint8_t* kr = sK + key * SS_ROW_BYTES;
#pragma unroll
      for (int c = 0; c < SS_D / 8; ++c) kv[c] = *reinterpret_cast<const uint4*>(kr + c * 16);
      float a[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
      for (int c = 0; c < SS_D / 8; ++c) dot8x4(qv[c], kv[c], a);
      return ((a[0] + a[1]) + (a[2] + a[3])) * p.scale_log2;
    };
    if (lane < p.S) s0 = score(lane);
    if (lane + 32 < p.S) s1 = score(lane + 32);
  }
  float m = fmaxf(s0, s1);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
  const float p0 = exp2f(s0 - m), p1 = exp2f(s1 - m);  // 0 for missing keys (-inf)
  float l = p0 + p1;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) l += __shfl_xor_sync(0xffffffffu, l, o);
  // O_in (unnormalised): dims 4 lane .. 4 lane + 3, two accumulators
  float4 acc0 = make_float4(0.f, 0.f, 0.f, 0.f), acc1 = acc0;
  const uint8_t* vcol = sV + lane * 8;
  if (p.S == 32) {
    // the 32 V values of this lane's dims and the 32 weights first, then the FMAs
    uint2 vv[32];
    float ww[32];
#pragma unroll
    for (int k = 0; k < 32; ++k) {
      vv[k] = *reinterpret_cast<const uint2*>(vcol + k * SS_ROW_BYTES);
      ww[k] = __shfl_sync(0xffffffffu, p0, k);
    }
#pragma unroll
    for (int k = 0; k < 32; k += 2) {
      pv_fma(ww[k], vv[k], acc0);
      pv_fma(ww[k + 1], vv[k + 1], acc1);
    }
  } else {
    const int nk0 = min(p.S, 32);
#pragma unroll 8
    for (int k = 0; k < nk0; ++k) pv_step(__shfl_sync(0xffffffffu, p0, k), vcol + k * SS_ROW_BYTES, acc0);
#pragma unroll 8
    for (int k = 32; k < p.S; ++k) pv_step(__shfl_sync(0xffffffffu, p1, k - 32), vcol + k * SS_ROW_BYTES, acc1);
  }
  const float4 acc = make_float4(acc0.x + acc1.x, acc0.y + acc1.y, acc0.z + acc1.z, acc0.w + acc1.w);
  // merge equation in base 2 (the block always has keys, so l > 0)
  const float lin2 = m + log2f(l);
  const float lp2 = lp * 1.4426950408889634f;
  const float M = fmaxf(lp2, lin2);
  const float wp = exp2f(lp2 - M);  // 0 when the prefix is empty (lp = -inf)
  const float wi = exp2f(lin2 - M);
  const float inv_den = 1.f / (wp + wi);
  const float ao = exp2f(m - M) * inv_den;  // = wi / l / den
  const float ap = wp * inv_den;
  const float4 o = make_float4(fmaf(ap, op.x, ao * acc.x), fmaf(ap, op.y, ao * acc.y), fmaf(ap, op.z, ao * acc.z),
                               fmaf(ap, op.w, ao * acc.w));
  *reinterpret_cast<uint2*>(p.out_o + qrow * SS_D + lane * 4) =
      make_uint2(pack_bf16x2(o.x, o.y), pack_bf16x2(o.z, o.w));
  if (lane == 0 && p.out_lse) p.out_lse[((size_t)b * p.Hq + h) * p.S + t] = (M + log2f(wp + wi)) * SS_LN2;
}

}  // namespace

bool small_step_fits(const fb_desc& d, int num_sms) {
  const long long rows = (long long)d.batch * d.block_len * d.num_q_heads;
  const long long ctas = (long long)d.batch * d.num_kv_heads *
                         ((d.block_len * (d.num_q_heads / d.num_kv_heads) + SS_ROWS_PER_CTA - 1) / SS_ROWS_PER_CTA);
  // short blocks whose rows fill at most two waves of these CTAs
  return d.dtype == FB_BF16 && d.head_dim == SS_D && d.block_len <= SS_MAX_S && rows > 0 &&
         ctas <= 2LL * num_sms;
}

cudaError_t launch_block_step_small(const fb_desc& d, const void* Q, const void* Kb, const void* Vb,
                                    const float* O_pre, const float* LSE_pre, void* O, float* LSE_out,
                                    cudaStream_t stream) {
  SmallStepParams p;
  p.B = d.batch;
  p.Hq = d.num_q_heads;
  p.Hkv = d.num_kv_heads;
  p.G = d.num_q_heads / d.num_kv_heads;
  p.S = d.block_len;
  p.scale_log2 = d.softmax_scale * 1.4426950408889634f;
  p.Q = static_cast<const __nv_bfloat16*>(Q);
  p.Kb = static_cast<const __nv_bfloat16*>(Kb);
  p.Vb = static_cast<const __nv_bfloat16*>(Vb);
  p.pre_o = O_pre;
  p.pre_lse = LSE_pre;
  p.out_o = static_cast<__nv_bfloat16*>(O);
  p.out_lse = LSE_out;
  const int cpu = (p.S * p.G + SS_ROWS_PER_CTA - 1) / SS_ROWS_PER_CTA;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)(p.B * p.Hkv * cpu));
  cfg.blockDim = dim3(SS_WARPS * 32);
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  cudaError_t e = cudaLaunchKernelEx(&cfg, block_step_small_kernel, p);
  note_launch();
  return e != cudaSuccess ? e : cudaGetLastError();
}

}  // namespace fb
