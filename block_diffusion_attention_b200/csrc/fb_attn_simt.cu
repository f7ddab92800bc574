// fb_attn_simt.cu -- fp32 attention partials on the CUDA cores.
//
// The fp32 path keeps float32 inputs exact to about 1e-6 (the tensor cores
// have no fp32-input kind, and TF32 would not hold 1e-5).  One warp computes
// one query row (b, t, h): lanes take 32 keys at a time (each lane copies its
// key's K and V rows into shared memory with cp.async, all copies in flight
// at once), the row max and the row sum come from warp shuffles, and each
// lane accumulates D/32 output columns from the staged value rows.  Key sources, epilogues and the merge are those of the tensor-core
// kernel (the partial, the merge equation and the uncached pass of the Core
// Mechanism in "FlashBlock: Attention Caching for Efficient Long-Context
// Block Diffusion", Technical Summary §2).
#include <math_constants.h>

#include <atomic>

#include "fb_internal.h"
#include "fb_ptx.cuh"

namespace fb {

namespace {

constexpr int MAXD = 128;
constexpr int WARPS = 4;
constexpr int VROW = MAXD + 4;  // floats per staged key or value row (16-byte aligned, banks staggered)
// the key and the value rows of a chunk, per warp
constexpr size_t SIMT_SMEM = (size_t)2 * WARPS * 32 * VROW * sizeof(float);

struct SimtUnit {
  int n0;  // prefix keys
  int n1;  // block keys
  int L;
};

__device__ SimtUnit simt_unit(const AttnParams& p, int b, int kvh, bool rep) {
  const KeySource& s = p.src;
  SimtUnit u{0, 0, 0};
  if (s.has_prefix) {
    int L = s.prefix_lens[b];
    if (L < 0 || L > s.cap) {
      if (rep) report(p.dev_status, FB_ERR_BOUNDS);
      L = max(0, min(L, s.cap));
    }
    u.L = L;
    if (s.chunk_idx) {
      const int32_t* idx = s.chunk_idx + ((size_t)b * p.Hkv + kvh) * s.topk;
      const int nch = (L + s.chunk_size - 1) / s.chunk_size;
      int n = 0, prev = -1;
      for (int i = 0; i < s.topk; ++i) {
        const int c = idx[i];
        if (c < 0) break;
        if (c <= prev || c >= nch) {
          if (rep) report(p.dev_status, FB_ERR_BOUNDS);
          break;
        }
        n += min(s.chunk_size, L - c * s.chunk_size);
        prev = c;
      }
      u.n0 = n;
    } else {
      u.n0 = L;
    }
  }
  if (s.has_block) u.n1 = p.S;
  return u;
}

// Row offset (in elements) of key i of the unit, and which tensor it lives in.
__device__ __forceinline__ size_t simt_key_offset(const AttnParams& p, const SimtUnit& u, int b,
                                                  int kvh, int i, bool& in_block) {
  const KeySource& s = p.src;
  if (i >= u.n0) {
    in_block = true;
    return (((size_t)b * p.S + (i - u.n0)) * p.Hkv + kvh) * p.D;
  }
  in_block = false;
  int pos;
  if (s.chunk_idx) {
    const int slot = i / s.chunk_size;
    pos = s.chunk_idx[((size_t)b * p.Hkv + kvh) * s.topk + slot] * s.chunk_size + (i - slot * s.chunk_size);
  } else {
    pos = i;
  }
  if (s.paged) {
    const int page_size = 1 << s.page_shift;
    const int pi = pos >> s.page_shift;
    int pg = (pi < s.max_pages) ? s.block_table[(size_t)b * s.max_pages + pi] : -1;
    if (pg < 0 || pg >= s.num_pages) {
      report(p.dev_status, FB_ERR_BOUNDS);
      pg = 0;
    }
    return (((size_t)pg * page_size + (pos & (page_size - 1))) * p.Hkv + kvh) * p.D;
  }
  return (((size_t)b * s.cap + pos) * p.Hkv + kvh) * p.D;
}

__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}
__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

template <int EPI>
__global__ void __launch_bounds__(WARPS * 32)
    attn_simt_kernel(const AttnParams p, const float* __restrict__ Q, const float* __restrict__ Kp,
                     const float* __restrict__ Vp, const float* __restrict__ Kb,
                     const float* __restrict__ Vb) {
  // may start before the previous kernel in the stream has finished
  pdl_wait();
  pdl_launch_dependents();
  __shared__ float sq[WARPS][MAXD];
  extern __shared__ __align__(16) float simt_sv[];  // values [WARPS][32 keys][VROW], then keys alike
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int t = blockIdx.x * WARPS + warp;
  const int h = blockIdx.y;
  const int b = blockIdx.z;
  if (t >= p.S) return;
  const int kvh = h / p.G;
  if (p.unit_mask && p.unit_mask[b * p.Hkv + kvh] == 0) return;  // unit not refreshed: outputs kept
  const int D = p.D;
  const int nd = D >> 5;  // output columns per lane
  const size_t qrow = ((size_t)b * p.S + t) * p.Hq + h;
  for (int d = lane; d < D; d += 32) sq[warp][d] = Q[qrow * D + d];
  __syncwarp();

  const SimtUnit u = simt_unit(p, b, kvh, t == 0 && h == 0 && lane == 0);
  const int ntot = u.n0 + u.n1;
  float m = -CUDART_INF_F, l = 0.f;
  float o[MAXD / 32];
#pragma unroll
  for (int k = 0; k < MAXD / 32; ++k) o[k] = 0.f;

  for (int base = 0; base < ntot; base += 32) {
    const int i = base + lane;
    float z = -CUDART_INF_F;
    // this lane's key row (K and V share the layout): offset and tensor
    size_t off = 0;
    bool blk = false;
    float* sv = simt_sv + ((size_t)warp * 32 + lane) * VROW;  // this lane's key's value row
    float* sk = sv + (size_t)WARPS * 32 * VROW;                // and its key row
    if (i < ntot) {
      off = simt_key_offset(p, u, b, kvh, i, blk);
      // the key and value rows go to shared memory with all their copies in
      // flight at once (the value rows are read only after the dot products)
      const float* krow = (blk ? Kb : Kp) + off;
      const float* vrow = (blk ? Vb : Vp) + off;
      for (int d = 0; d < D; d += 4) cp_async16(smem_u32(sk + d), krow + d, 16u);
      for (int d = 0; d < D; d += 4) cp_async16(smem_u32(sv + d), vrow + d, 16u);
      cp_async_commit();
      cp_async_wait_all();  // (this lane's own rows: no other lane's copies needed)
      float acc = 0.f;
      for (int d = 0; d < D; d += 4) {
        const float4 kv = *reinterpret_cast<const float4*>(sk + d);
        acc = fmaf(sq[warp][d], kv.x, acc);
        acc = fmaf(sq[warp][d + 1], kv.y, acc);
        acc = fmaf(sq[warp][d + 2], kv.z, acc);
        acc = fmaf(sq[warp][d + 3], kv.w, acc);
      }
      z = acc * p.scale;
    }
    const float m_new = fmaxf(m, warp_max(z));
    const float alpha = (m == -CUDART_INF_F) ? 0.f : expf(m - m_new);
    const float pz = (i < ntot) ? expf(z - m_new) : 0.f;
    l = l * alpha + warp_sum(pz);
#pragma unroll
    for (int k = 0; k < MAXD / 32; ++k) o[k] *= alpha;
    const int nk = min(32, ntot - base);
    // the chunk's value rows, staged by their lanes, from shared memory
    __syncwarp();
    const float* svw = simt_sv + (size_t)warp * 32 * VROW;
#pragma unroll 8
    for (int jj = 0; jj < nk; ++jj) {
      const float pj = __shfl_sync(0xffffffffu, pz, jj);
#pragma unroll
      for (int k = 0; k < MAXD / 32; ++k)
        if (k < nd) o[k] = fmaf(pj, svw[jj * VROW + lane + 32 * k], o[k]);
    }
    __syncwarp();  // the rows may be written again by the next chunk
    m = m_new;
  }

  const bool empty = (ntot == 0) || !(l > 0.f);
  const float inv_l = empty ? 0.f : 1.f / l;
  const float lse = empty ? -CUDART_INF_F : m + logf(l);
  if (EPI == EPI_PARTIAL) {
    float* dst = p.out_o32 + qrow * D;
#pragma unroll
    for (int k = 0; k < MAXD / 32; ++k)
      if (k < nd) dst[lane + 32 * k] = o[k] * inv_l;
    if (lane == 0) p.out_lse[((size_t)b * p.Hq + h) * p.S + t] = lse;
  } else {
    float wp = 0.f, wi = 1.f, inv_den = 1.f, lse_out = lse;
    if (EPI == EPI_MERGE) {
      // merge equation: m = max(L_out, L_in); weights e^{L - m}
      const float lp = p.pre_lse[((size_t)b * p.Hq + h) * p.S + t];
      const float M = fmaxf(lp, lse);
      const float Ms = (M == -CUDART_INF_F) ? 0.f : M;
      wp = (lp == -CUDART_INF_F) ? 0.f : expf(lp - Ms);
      wi = empty ? 0.f : expf(lse - Ms);
      const float den = wp + wi;
      inv_den = den > 0.f ? 1.f / den : 0.f;
      lse_out = den > 0.f ? Ms + logf(den) : -CUDART_INF_F;
    }
    float* dst = reinterpret_cast<float*>(p.out_o) + qrow * D;
    const float* pre = (EPI == EPI_MERGE) ? p.pre_o + qrow * D : nullptr;
#pragma unroll
    for (int k = 0; k < MAXD / 32; ++k) {
      if (k < nd) {
        const float oin = o[k] * inv_l;
        dst[lane + 32 * k] = (EPI == EPI_MERGE) ? (wp * pre[lane + 32 * k] + wi * oin) * inv_den : oin;
      }
    }
    if (lane == 0 && p.out_lse) p.out_lse[((size_t)b * p.Hq + h) * p.S + t] = lse_out;
  }
}

}  // namespace

cudaError_t launch_attn_simt(const AttnParams& p, const float* Q, const float* Kp, const float* Vp,
                             const float* Kb, const float* Vb, cudaStream_t stream) {
  dim3 grid((p.S + WARPS - 1) / WARPS, p.Hq, p.B);
  void (*kern)(const AttnParams, const float*, const float*, const float*, const float*, const float*) =
      p.epi == EPI_PARTIAL ? attn_simt_kernel<EPI_PARTIAL>
      : p.epi == EPI_MERGE ? attn_simt_kernel<EPI_MERGE>
                           : attn_simt_kernel<EPI_NORM>;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  // (set once per device and kernel)
  static std::atomic<bool> configured[64][3];
  const int which = p.epi == EPI_PARTIAL ? 0 : p.epi == EPI_MERGE ? 1 : 2;
  if (dev >= 64 || !configured[dev][which].load(std::memory_order_acquire)) {
    e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)SIMT_SMEM);
    if (e != cudaSuccess) return e;
    if (dev < 64) configured[dev][which].store(true, std::memory_order_release);
  }
  e = launch_pdl(kern, grid, dim3(WARPS * 32), SIMT_SMEM, stream, p, Q, Kp, Vp, Kb, Vb);
  note_launch();
  return e != cudaSuccess ? e : cudaGetLastError();
}

}  // namespace fb
