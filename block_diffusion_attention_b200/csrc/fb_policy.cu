// fb_policy.cu -- refresh masks of the adaptive reuse strategies.
//
// "FlashBlock: Attention Caching for Efficient Long-Context Block Diffusion",
// Adaptive Reuse Strategies: instead of refreshing the cached block-external
// pair at fixed steps, a policy decides per step which work units recompute
// it.  Both policies here write a refresh mask [B, Hkv] (1 = recompute the
// unit's pair with this step's queries, 0 = keep the cached one) that the
// masked prefix pass consumes.
//
//  * Head-wise Selection: a (b, kv head) unit recomputes when the cosine
//    similarity of its queries now to the queries its cached pair was computed
//    with falls below gamma (the similarity is taken over the unit's S x G x D
//    query values).  A refreshed unit's queries become its new reference.
//  * Threshold-based Reuse: a sequence recomputes when the number M of block
//    tokens whose key or value moved by more than eps (max |change| over kv
//    heads and dims) since the previous step is at least tau.  The current
//    block K/V become the previous ones for the next step.
//
// Head-wise: one 8-CTA thread-block cluster per unit; each CTA reduces its
// slice of the unit to (q.r, |q|^2, |r|^2), every CTA reads the eight partials
// through distributed shared memory in rank order (so all take the same
// decision), and each copies its own slice into the reference when the unit
// refreshes.  Threshold: a wide pass (one warp per token) flags the tokens,
// counts them per CTA into the workspace and moves the block K/V into the
// previous-step buffers; a second pass sums the counts per sequence.
#include <cooperative_groups.h>
#include <cuda_bf16.h>
#include <math_constants.h>

#include "fb_internal.h"
#include "fb_ptx.cuh"

namespace cg = cooperative_groups;

namespace fb {

namespace {

constexpr int HW_CLUSTER = 8;
constexpr int HW_THREADS = 256;
constexpr int TH_TOKENS = 4;  // tokens (warps) per CTA of the threshold pass

// eight bf16 or four f32 values of one 16-byte vector, as floats
template <bool BF16>
__device__ __forceinline__ int unpack16(const uint4& v, float* f) {
  if (BF16) {
    const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&v);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const float2 x = __bfloat1622float2(h[i]);
      f[2 * i] = x.x;
      f[2 * i + 1] = x.y;
    }
    return 8;
  } else {
    f[0] = __uint_as_float(v.x);
    f[1] = __uint_as_float(v.y);
    f[2] = __uint_as_float(v.z);
    f[3] = __uint_as_float(v.w);
    return 4;
  }
}

template <bool BF16>
__global__ void __cluster_dims__(HW_CLUSTER, 1, 1) __launch_bounds__(HW_THREADS)
    headwise_mask_kernel(const uint4* __restrict__ Qnow, uint4* __restrict__ Qref, int S, int Hq, int Hkv,
                         int D, float gamma, int32_t* __restrict__ mask, float* __restrict__ sim_out) {
  // may start before the previous kernel in the stream has finished
  pdl_wait();
  pdl_launch_dependents();
  __shared__ float red[HW_THREADS / 32][3];
  __shared__ float part[3];
  cg::cluster_group cluster = cg::this_cluster();
  const int rank = (int)cluster.block_rank();
  const int unit = blockIdx.x / HW_CLUSTER;  // b * Hkv + kvh
  const int b = unit / Hkv, kvh = unit % Hkv;
  const int G = Hq / Hkv;
  constexpr int EPV = BF16 ? 8 : 4;           // elements per 16-byte vector
  const int vpt = G * D / EPV;                 // vectors of the unit per token
  const long long n = (long long)S * vpt;
  const long long v0 = n * rank / HW_CLUSTER, v1 = n * (rank + 1) / HW_CLUSTER;
  // vector v of the unit: token t = v / vpt, offset j = v % vpt inside the
  // token's G contiguous heads
  auto gidx = [&](long long v) -> size_t {
    const long long t = v / vpt;
    const long long j = v - t * vpt;
    return (size_t)(((long long)b * S + t) * Hq + (long long)kvh * G) * D / EPV + j;
  };
  float dot = 0.f, na = 0.f, nr = 0.f;
  for (long long v = v0 + threadIdx.x; v < v1; v += HW_THREADS) {
    const size_t g = gidx(v);
    float a[8], r[8];
    const uint4 va = Qnow[g];
    const uint4 vr = Qref[g];
    unpack16<BF16>(va, a);
    unpack16<BF16>(vr, r);
#pragma unroll
    for (int i = 0; i < EPV; ++i) {
      dot = fmaf(a[i], r[i], dot);
      na = fmaf(a[i], a[i], na);
      nr = fmaf(r[i], r[i], nr);
    }
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    dot += __shfl_xor_sync(0xffffffffu, dot, o);
    na += __shfl_xor_sync(0xffffffffu, na, o);
    nr += __shfl_xor_sync(0xffffffffu, nr, o);
  }
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (lane == 0) {
    red[warp][0] = dot;
    red[warp][1] = na;
    red[warp][2] = nr;
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    float s0 = 0.f, s1 = 0.f, s2 = 0.f;
    for (int w = 0; w < HW_THREADS / 32; ++w) {
      s0 += red[w][0];
      s1 += red[w][1];
      s2 += red[w][2];
    }
    part[0] = s0;
    part[1] = s1;
    part[2] = s2;
  }
  cluster.sync();
  // every CTA sums the cluster's partials in rank order: one decision
  float tdot = 0.f, tna = 0.f, tnr = 0.f;
  for (int r = 0; r < HW_CLUSTER; ++r) {
    const float* rp = cluster.map_shared_rank(part, r);
    tdot += rp[0];
    tna += rp[1];
    tnr += rp[2];
  }
  cluster.sync();  // no CTA leaves while another still reads its partials
  const float den = sqrtf(tna) * sqrtf(tnr);
  const float sim = den > 0.f ? tdot / den : 1.f;
  const bool refresh = !(sim >= gamma);  // a NaN similarity refreshes
  if (rank == 0 && threadIdx.x == 0) {
    mask[unit] = refresh ? 1 : 0;
    if (sim_out) sim_out[unit] = sim;
  }
  if (refresh)
    for (long long v = v0 + threadIdx.x; v < v1; v += HW_THREADS) {
      const size_t g = gidx(v);
      Qref[g] = Qnow[g];
    }
}

template <bool BF16>
__global__ void __launch_bounds__(TH_TOKENS * 32)
    threshold_flag_kernel(uint4* __restrict__ Kprev, uint4* __restrict__ Vprev, const uint4* __restrict__ Know,
                          const uint4* __restrict__ Vnow, int S, int vpt, float eps, int nslice,
                          int32_t* __restrict__ counts) {
  // may start before the previous kernel in the stream has finished
  pdl_wait();
  pdl_launch_dependents();
  __shared__ int flags[TH_TOKENS];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int slice = blockIdx.x, b = blockIdx.y;
  const int t = slice * TH_TOKENS + warp;
  int moved = 0;
  if (t < S) {
    const size_t base = ((size_t)b * S + t) * vpt;  // the token's Hkv x D values, contiguous
    for (int j = lane; j < vpt; j += 32) {
      const uint4 kn = Know[base + j], kp = Kprev[base + j];
      const uint4 vn = Vnow[base + j], vp = Vprev[base + j];
      float a[8], c[8];
      const int ne = unpack16<BF16>(kn, a);
      unpack16<BF16>(kp, c);
#pragma unroll
      for (int i = 0; i < 8; ++i)
        if (i < ne && fabsf(a[i] - c[i]) > eps) moved = 1;
      unpack16<BF16>(vn, a);
      unpack16<BF16>(vp, c);
#pragma unroll
      for (int i = 0; i < 8; ++i)
        if (i < ne && fabsf(a[i] - c[i]) > eps) moved = 1;
      Kprev[base + j] = kn;
      Vprev[base + j] = vn;
    }
    moved = __any_sync(0xffffffffu, moved);
  }
  if (lane == 0) flags[warp] = moved;
  __syncthreads();
  if (threadIdx.x == 0) {
    int c = 0;
    for (int w = 0; w < TH_TOKENS; ++w) c += flags[w];
    counts[(size_t)b * nslice + slice] = c;
  }
}

__global__ void threshold_decide_kernel(const int32_t* __restrict__ counts, int nslice, int Hkv, int32_t tau,
                                        int32_t* __restrict__ mask, int32_t* __restrict__ count_out) {
  // may start before the previous kernel in the stream has finished
  pdl_wait();
  pdl_launch_dependents();
  const int b = blockIdx.x;
  int c = 0;
  for (int i = threadIdx.x; i < nslice; i += 32) c += counts[(size_t)b * nslice + i];
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) c += __shfl_xor_sync(0xffffffffu, c, o);
  const int refresh = c >= tau ? 1 : 0;
  for (int k = threadIdx.x; k < Hkv; k += 32) mask[(size_t)b * Hkv + k] = refresh;
  if (threadIdx.x == 0 && count_out) count_out[b] = c;
}

}  // namespace

size_t threshold_ws_bytes(const fb_desc& d) {
  return (size_t)d.batch * ((d.block_len + TH_TOKENS - 1) / TH_TOKENS) * sizeof(int32_t);
}

cudaError_t launch_headwise_mask(const fb_desc& d, const void* Qnow, void* Qref, float gamma, int32_t* mask,
                                 float* sim, cudaStream_t stream) {
  const dim3 grid((unsigned)(d.batch * d.num_kv_heads * HW_CLUSTER));
  cudaError_t e = launch_pdl(d.dtype == FB_BF16 ? headwise_mask_kernel<true> : headwise_mask_kernel<false>, grid,
                             dim3(HW_THREADS), 0, stream, static_cast<const uint4*>(Qnow), static_cast<uint4*>(Qref),
                             d.block_len, d.num_q_heads, d.num_kv_heads, d.head_dim, gamma, mask, sim);
  note_launch();
  return e != cudaSuccess ? e : cudaGetLastError();
}

cudaError_t launch_threshold_mask(const fb_desc& d, void* Kprev, void* Vprev, const void* Know, const void* Vnow,
                                  float eps, int32_t tau, int32_t* mask, int32_t* count, int32_t* ws,
                                  cudaStream_t stream) {
  const int nslice = (d.block_len + TH_TOKENS - 1) / TH_TOKENS;
  const int epv = d.dtype == FB_BF16 ? 8 : 4;
  const int vpt = d.num_kv_heads * d.head_dim / epv;
  const dim3 grid((unsigned)nslice, (unsigned)d.batch);
  cudaError_t e =
      launch_pdl(d.dtype == FB_BF16 ? threshold_flag_kernel<true> : threshold_flag_kernel<false>, grid,
                 dim3(TH_TOKENS * 32), 0, stream, static_cast<uint4*>(Kprev), static_cast<uint4*>(Vprev),
                 static_cast<const uint4*>(Know), static_cast<const uint4*>(Vnow), d.block_len, vpt, eps, nslice, ws);
  note_launch();
  if (e == cudaSuccess) e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  e = launch_pdl(threshold_decide_kernel, dim3(d.batch), dim3(32), 0, stream, (const int32_t*)ws, nslice,
                 d.num_kv_heads, tau, mask, count);
  note_launch();
  return e != cudaSuccess ? e : cudaGetLastError();
}

}  // namespace fb
