// fb_aux.cu -- sparse-prefix chunk means and top-k selection, and the block
// append that grows the KV cache.
//
// Sparse prefix ("FlashBlock: Attention Caching for Efficient Long-Context
// Block Diffusion", Technical Summary §2, Adaptive Reuse Strategies,
// Compatibility with Sparse Attention): the prefix keys of each (b, kv head)
// are restricted to the top-k chunks by the score
//     qbar . kbar_c,
// qbar the mean query of the block over its tokens and the G heads of the
// group, kbar_c the mean key of chunk c over its valid rows.
// Append (Technical Summary §1: block diffusion keeps a KV cache of the blocks
// already generated, each block causal with respect to the earlier ones):
// a finalized block's K/V joins the prefix.
#include <cuda_bf16.h>
#include <math_constants.h>

#include <atomic>

#include "fb_attn_common.cuh"
#include "fb_internal.h"
#include "fb_ptx.cuh"

namespace fb {

namespace {

template <typename T>
__device__ __forceinline__ float to_f(T v);
template <>
__device__ __forceinline__ float to_f<float>(float v) { return v; }
template <>
__device__ __forceinline__ float to_f<__nv_bfloat16>(__nv_bfloat16 v) { return __bfloat162float(v); }

// grid (chunks, Hkv, B), block D threads: thread d averages column d.
// tail_rows == 0: chunk c0 + blockIdx.x of every sequence.  tail_rows > 0:
// the chunks holding sequence b's last tail_rows valid rows, [L_b - tail_rows,
// L_b), from its device length: chunk (max(L_b - tail_rows, 0) / chunk_size)
// + blockIdx.x, skipped when it starts at or past L_b.
template <typename T>
__global__ void chunk_means_kernel(const CacheGeom g, const int32_t* lens, int chunk_size,
                                   int c0, int tail_rows, int nch_total, const T* __restrict__ K,
                                   float* __restrict__ Kmean, int32_t* status) {
  // may start before the previous kernel in the stream has finished
  pdl_wait();
  pdl_launch_dependents();
  const int kvh = blockIdx.y;
  const int b = blockIdx.z;
  const int d = threadIdx.x;
  int L = lens[b];
  if (L < 0 || L > g.cap) {
    if (d == 0) report(status, FB_ERR_BOUNDS);
    L = max(0, min(L, g.cap));
  }
  int c = c0 + blockIdx.x;
  if (tail_rows > 0) {
    c = max(L - tail_rows, 0) / chunk_size + blockIdx.x;
    if (c * chunk_size >= L) return;  // (block-uniform)
  }
  const int lo = c * chunk_size;
  const int hi = min(lo + chunk_size, L);
  float acc = 0.f;
  for (int pos = lo; pos < hi; ++pos) {
    const long long off = cache_offset(g, b, pos, kvh);
    if (off < 0) {
      if (d == 0) report(status, FB_ERR_BOUNDS);
      continue;
    }
    acc += to_f<T>(K[off + d]);
  }
  const float mean = hi > lo ? acc / (float)(hi - lo) : 0.f;
  Kmean[(((size_t)b * g.Hkv + kvh) * nch_total + c) * g.D + d] = mean;
}

// One CTA of SEL_THREADS per (b, kv head); grid (Hkv, B).  The CTA
//   1. issues the loads of the first SEL_THREADS / 4 chunk means (four lanes
//      per chunk, a quarter of D each) into registers, so they are in flight
//      with the query loads,
//   2. sums the unit's S x G query rows per column (16-byte vectors, the row
//      groups added in a fixed order) into qbar,
//   3. scores every chunk, then ranks each chunk against all scores (rank =
//      chunks with a higher score, or an equal score and a lower index); the
//      chunks of rank below topk are the selected ones,
//   4. writes the selected chunks at their ascending-order positions
//      (select_from_scores).
// Dynamic shared memory: see sel_smem_bytes.
constexpr int SEL_THREADS = 512;
constexpr int SEL_PART_FLOATS = SEL_THREADS * 8;  // row-group sums of the query mean (16-bit inputs)

size_t sel_smem_bytes(int D, int nch_total) {
  // row-group sums, qbar, every score (padded to 4; the ranks later take its
  // place), every key (padded to 2), warp totals
  return (size_t)(SEL_PART_FLOATS + D + ((nch_total + 3) & ~3)) * sizeof(float) +
         (size_t)((nch_total + 1) & ~1) * 8 + (SEL_THREADS / 32) * sizeof(int);
}

// Adds the eight bf16 or four f32 values of a 16-byte vector to acc.
template <typename T>
__device__ __forceinline__ void add_vec16(const uint4& v, float* acc);
template <>
__device__ __forceinline__ void add_vec16<__nv_bfloat16>(const uint4& v, float* acc) {
  const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&v);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const float2 x = __bfloat1622float2(h[i]);
    acc[2 * i] += x.x;
    acc[2 * i + 1] += x.y;
  }
}
template <>
__device__ __forceinline__ void add_vec16<float>(const uint4& v, float* acc) {
  acc[0] += __uint_as_float(v.x);
  acc[1] += __uint_as_float(v.y);
  acc[2] += __uint_as_float(v.z);
  acc[3] += __uint_as_float(v.w);
}

// The selection order -- chunk a ranks above chunk b iff its score is higher,
// or equal with a lower index -- as one unsigned 64-bit key: the score's bits
// made monotonic (-0 taken as +0, so that equal scores compare equal), then
// the chunk index inverted; a chunk ranks above another iff its key is larger.
__device__ __forceinline__ unsigned long long rank_key(float sc, int c) {
  uint32_t u = __float_as_uint(sc + 0.f);
  u ^= (u >> 31) ? 0xffffffffu : 0x80000000u;
  return ((unsigned long long)u << 32) | (0xffffffffu - (uint32_t)c);
}

// Steps 3b and 4 of the selection, from the scores of the nch valid chunks in
// shared memory (key: nch 64-bit keys rounded up to an even count, rank: nch
// ints, which may take the scores' place, and wsum: SEL_THREADS / 32 ints of
// shared memory); writes the unit's topk list to out.
//   3b. rank of each chunk = the chunks that rank above it, counted by 1, 2
//       or 4 lanes per chunk (as many as keep all chunks in one pass of the
//       CTA where they can), two keys per shared-memory read; a chunk is
//       selected iff its rank is below topk (every chunk when there are at
//       most topk);
//   4.  the selected chunks at their ascending-order positions: within a warp
//       from a ballot, across warps from the warps' counts.
__device__ __forceinline__ void select_from_scores(const float* score, unsigned long long* key, int* rank, int* wsum,
                                                   int nch, int topk, int32_t* out) {
  if (nch > topk) {
    for (int c = threadIdx.x; c < ((nch + 1) & ~1); c += SEL_THREADS)
      key[c] = c < nch ? rank_key(score[c], c) : 0ull;  // the padding key ranks above nothing
    __syncthreads();
    const int lpc = nch <= SEL_THREADS / 4 ? 4 : (nch <= SEL_THREADS / 2 ? 2 : 1);  // lanes per chunk
    const int sub = threadIdx.x & (lpc - 1);
    const ulonglong2* k2 = reinterpret_cast<const ulonglong2*>(key);
    for (int base = 0; base < nch; base += SEL_THREADS / lpc) {
      const int c = base + threadIdx.x / lpc;
      const unsigned long long kc = key[min(c, nch - 1)];
      int better = 0;
      for (int o = sub; 2 * o < nch; o += lpc) {
        const ulonglong2 v = k2[o];
        better += (v.x > kc) + (v.y > kc);
      }
      if (lpc >= 2) better += __shfl_xor_sync(0xffffffffu, better, 1);
      if (lpc == 4) better += __shfl_xor_sync(0xffffffffu, better, 2);
      if (sub == 0 && c < nch) rank[c] = better;
    }
  } else {
    for (int c = threadIdx.x; c < nch; c += SEL_THREADS) rank[c] = 0;
  }
  __syncthreads();
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  int carry = 0;  // chunks selected in earlier passes
  for (int base = 0; base < nch; base += SEL_THREADS) {
    const int c = base + threadIdx.x;
    const bool sel = c < nch && rank[c] < topk;
    const unsigned bal = __ballot_sync(0xffffffffu, sel);
    if (lane == 0) wsum[warp] = __popc(bal);
    __syncthreads();
    int before = carry + __popc(bal & ((1u << lane) - 1u)), total = carry;
    for (int w2 = 0; w2 < SEL_THREADS / 32; ++w2) {
      const int v = wsum[w2];
      before += w2 < warp ? v : 0;
      total += v;
    }
    if (sel && before < topk) out[before] = c;
    carry = total;
    __syncthreads();  // wsum is written again by the next pass
  }
  for (int i = min(carry, topk) + threadIdx.x; i < topk; i += SEL_THREADS) out[i] = -1;
}

template <typename T>
__global__ void __launch_bounds__(SEL_THREADS)
    select_chunks_kernel(const CacheGeom g, const int32_t* lens, int chunk_size, int nch_total, int S, int Hq,
                         int topk, const T* __restrict__ Q, const float* __restrict__ Kmean,
                         int32_t* __restrict__ idx, int32_t* status) {
  // may start before the previous kernel in the stream has finished
  pdl_wait();
  pdl_launch_dependents();
  extern __shared__ float sm[];
  const int kvh = blockIdx.x;
  const int b = blockIdx.y;
  const int G = Hq / g.Hkv;
  const int D = g.D;
  float* rowsum = sm;                       // [rpi][D] row-group sums
  float* qbar = rowsum + SEL_PART_FLOATS;   // [D]
  float* score = qbar + D;                  // [nch_total rounded up to 4]; later the ranks
  unsigned long long* key =                 // [nch_total rounded up to 2], 16-byte aligned
      reinterpret_cast<unsigned long long*>(score + ((nch_total + 3) & ~3));
  int* rank = reinterpret_cast<int*>(score);  // (the scores are not read once the keys exist)
  int* wsum = reinterpret_cast<int*>(key + ((nch_total + 1) & ~1));  // [warps]
  // 1. the first pass's chunk means, loaded before anything else (rows below
  // nch_total always exist, whatever the prefix length), in flight with the
  // query loads.  Lane q4 of a chunk's four takes the float4s q4, q4 + 4, ...
  // of its mean row, so the four lanes read 64 contiguous bytes per step.
  const float* km = Kmean + ((size_t)b * g.Hkv + kvh) * nch_total * D;
  const int q4 = threadIdx.x & 3, dq = D / 4;
  constexpr int CPP = SEL_THREADS / 4;  // chunks per pass
  float4 kr[8];
  {
    const int c = threadIdx.x >> 2;
#pragma unroll
    for (int i = 0; i < 8; ++i)
      kr[i] = (c < nch_total && i < dq / 4) ? reinterpret_cast<const float4*>(km + (size_t)c * D)[4 * i + q4]
                                            : make_float4(0.f, 0.f, 0.f, 0.f);
  }
  int L = lens[b];
  if (L < 0 || L > g.cap) {
    if (threadIdx.x == 0) report(status, FB_ERR_BOUNDS);
    L = max(0, min(L, g.cap));
  }
  const int nch = (L + chunk_size - 1) / chunk_size;
  // 2. query mean over the S block tokens and the G heads of the group:
  // thread i takes vector i % vpr of rows i / vpr, + rpi, ...; the rpi
  // row-group sums of each column are then added in a fixed order
  constexpr int VEC = 16 / sizeof(T);
  const int vpr = D / VEC;                // vectors per row
  const int rpi = SEL_THREADS / vpr;      // rows per iteration
  const int rows = S * G;
  {
    const int vi = threadIdx.x % vpr, rg = threadIdx.x / vpr;
    if (rg < rpi) {
      float acc[VEC];
#pragma unroll
      for (int k = 0; k < VEC; ++k) acc[k] = 0.f;
#pragma unroll 8
      for (int rr = rg; rr < rows; rr += rpi) {
        const int t = rr / G, gg = rr - t * G;
        const uint4 v = *reinterpret_cast<const uint4*>(Q + (((size_t)b * S + t) * Hq + kvh * G + gg) * D + vi * VEC);
        add_vec16<T>(v, acc);
      }
#pragma unroll
      for (int k = 0; k < VEC; ++k) rowsum[rg * D + vi * VEC + k] = acc[k];
    }
  }
  __syncthreads();
  for (int d = threadIdx.x; d < D; d += SEL_THREADS) {
    float acc = 0.f;
    for (int w2 = 0; w2 < rpi; ++w2) acc += rowsum[w2 * D + d];
    qbar[d] = acc / (float)rows;
  }
  __syncthreads();
  // 3a. scores: four lanes per chunk, then two shuffles
  for (int base = 0; base < nch; base += CPP) {
    const int c = base + (threadIdx.x >> 2);
    const float4* qr = reinterpret_cast<const float4*>(qbar);
    const float4* kp = reinterpret_cast<const float4*>(km + (size_t)c * D);
    float acc = 0.f;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      if (i < dq / 4) {
        const float4 q = qr[4 * i + q4];
        const float4 k = base == 0 ? kr[i] : (c < nch ? kp[4 * i + q4] : make_float4(0.f, 0.f, 0.f, 0.f));
        acc = fmaf(q.x, k.x, fmaf(q.y, k.y, fmaf(q.z, k.z, fmaf(q.w, k.w, acc))));
      }
    }
    acc += __shfl_xor_sync(0xffffffffu, acc, 1);
    acc += __shfl_xor_sync(0xffffffffu, acc, 2);
    if (q4 == 0 && c < nch) score[c] = acc;
  }
  __syncthreads();
  select_from_scores(score, key, rank, wsum, nch, topk, idx + ((size_t)b * g.Hkv + kvh) * topk);
}

// The same selection with every input of the unit in shared memory first:
// warp 0 issues plain bulk copies of the unit's chunk means (one contiguous
// nch_total x D block) and of its S x G query rows (one copy of G contiguous
// heads per token), all completing on one mbarrier, so the unit's inputs
// (2 x 64 KB in the batched sparse workload) cross HBM in one round trip
// without the load/store unit.  Then
//   2. column sums of the query rows (16-byte vectors in up to 32 row
//      groups, added in a fixed order) into qbar,
//   3a. scores, eight lanes per chunk (four chunks per warp and step),
//   3b, 4. as in select_chunks_kernel.
// D = 128.  Used when sel_bulk_smem_bytes fits and both sources are 16-byte
// aligned.
constexpr int SELB_D = 128;
constexpr int SELB_GROUPS = 32;  // row groups of the column sums (at most)

size_t sel_bulk_smem_bytes(int rows, int nch_total, size_t esz) {
  // barrier (16), chunk means, query rows, row-group sums, qbar, every
  // score (padded to 4; the ranks later take its place), every key (padded
  // to 2), warp totals
  return 16 + (size_t)nch_total * SELB_D * 4 + (size_t)rows * SELB_D * esz +
         (size_t)(SELB_GROUPS * SELB_D + SELB_D + ((nch_total + 3) & ~3)) * sizeof(float) +
         (size_t)((nch_total + 1) & ~1) * 8 + (SEL_THREADS / 32) * sizeof(int);
}

template <typename T>
__global__ void __launch_bounds__(SEL_THREADS)
    select_chunks_bulk_kernel(const CacheGeom g, const int32_t* lens, int chunk_size, int nch_total, int S, int Hq,
                              int topk, const T* __restrict__ Q, const float* __restrict__ Kmean,
                              int32_t* __restrict__ idx, int32_t* status) {
  constexpr int D = SELB_D;
  extern __shared__ __align__(16) uint8_t selb_raw[];
  const int kvh = blockIdx.x;
  const int b = blockIdx.y;
  const int G = Hq / g.Hkv;
  const int rows = S * G;
  uint64_t* bar = reinterpret_cast<uint64_t*>(selb_raw);
  float* skm = reinterpret_cast<float*>(selb_raw + 16);      // [nch_total][D]
  T* sq = reinterpret_cast<T*>(skm + (size_t)nch_total * D);  // [rows][D]
  float* part = reinterpret_cast<float*>(sq + (size_t)rows * D);  // [SELB_GROUPS][D]
  float* qbar = part + SELB_GROUPS * D;                       // [D]
  float* score = qbar + D;                                    // [nch_total rounded up to 4]; later the ranks
  unsigned long long* key =                                   // [nch_total rounded up to 2]
      reinterpret_cast<unsigned long long*>(score + ((nch_total + 3) & ~3));
  int* rank = reinterpret_cast<int*>(score);                  // (scores are not read once the keys exist)
  int* wsum = reinterpret_cast<int*>(key + ((nch_total + 1) & ~1));  // [warps]
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    mbar_init(bar, 1);
    abort_flag = 0;
    fence_barrier_init();
  }
  __syncthreads();
  // may start before the previous kernel in the stream has finished
  pdl_wait();
  pdl_launch_dependents();
  const uint32_t qpiece = (uint32_t)(G * D * sizeof(T));
  if (threadIdx.x < 32) {
    // warp 0 issues the copies, the byte count first
    const uint32_t kbytes = (uint32_t)nch_total * D * 4;
    if (threadIdx.x == 0) {
      mbar_arrive_expect_tx(bar, kbytes + (uint32_t)S * qpiece);
      bulk_load(skm, Kmean + ((size_t)b * g.Hkv + kvh) * nch_total * D, kbytes, bar);
    }
    __syncwarp();
    for (int t = threadIdx.x; t < S; t += 32)
      bulk_load(sq + (size_t)t * G * D, Q + (((size_t)b * S + t) * Hq + (size_t)kvh * G) * D, qpiece, bar);
  }
  int L = lens[b];
  if (L < 0 || L > g.cap) {
    if (threadIdx.x == 0) report(status, FB_ERR_BOUNDS);
    L = max(0, min(L, g.cap));
  }
  const int nch = (L + chunk_size - 1) / chunk_size;
  if (!bounded_wait(bar, 0, &abort_flag, status, false)) {
    // the copies did not land in time (reported): wait once more, also
    // bounded, before the CTA's shared memory is given up
    bounded_wait(bar, 0, &abort_flag, nullptr, false);
    return;
  }
  // 2. query mean: thread i sums the 16-byte vector i % VPR of rows i / VPR,
  // + SEL_THREADS / VPR, ... (pairs of columns added as f32x2), then the row
  // groups are added in a fixed order
  {
    constexpr int VEC = 16 / sizeof(T);  // columns per vector
    constexpr int VPR = D / VEC;         // vectors per row
    static_assert(SEL_THREADS / VPR <= SELB_GROUPS, "row groups");
    const int vi = threadIdx.x % VPR;
    const int rg = threadIdx.x / VPR;
    float2 acc[VEC / 2];
#pragma unroll
    for (int k = 0; k < VEC / 2; ++k) acc[k] = make_float2(0.f, 0.f);
#pragma unroll 4
    for (int r = rg; r < rows; r += SEL_THREADS / VPR) {
      const uint4 v = *reinterpret_cast<const uint4*>(sq + (size_t)r * D + vi * VEC);
      const uint32_t w[4] = {v.x, v.y, v.z, v.w};
      if constexpr (VEC == 8) {
        // bf16 pair -> two floats: the low half shifted up, the high half masked
#pragma unroll
        for (int k = 0; k < 4; ++k)
          acc[k] = fadd2(acc[k], make_float2(__uint_as_float(w[k] << 16), __uint_as_float(w[k] & 0xffff0000u)));
      } else {
#pragma unroll
        for (int k = 0; k < 2; ++k)
          acc[k] = fadd2(acc[k], make_float2(__uint_as_float(w[2 * k]), __uint_as_float(w[2 * k + 1])));
      }
    }
    float* dst = part + rg * D + vi * VEC;
#pragma unroll
    for (int k = 0; k < VEC / 2; ++k) *reinterpret_cast<float2*>(dst + 2 * k) = acc[k];
  }
  __syncthreads();
  if (threadIdx.x < D) {
    constexpr int NG = SEL_THREADS / (D / (16 / sizeof(T)));  // row groups written
    float a4[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
    for (int w2 = 0; w2 < NG; ++w2) a4[w2 & 3] += part[w2 * D + threadIdx.x];
    qbar[threadIdx.x] = ((a4[0] + a4[1]) + (a4[2] + a4[3])) / (float)rows;
  }
  __syncthreads();
  // 3a. scores: eight lanes per chunk (lane l8 takes every eighth float4 of
  // the chunk's mean, starting at l8), four chunks per warp and pass
  {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int l8 = lane & 7;
    const float4* q4p = reinterpret_cast<const float4*>(qbar);
#pragma unroll 2
    for (int base = 0; base < nch; base += SEL_THREADS / 8) {
      const int c = base + warp * 4 + (lane >> 3);
      const float4* kp = reinterpret_cast<const float4*>(skm + (size_t)min(c, nch_total - 1) * D);
      float acc = 0.f;
#pragma unroll
      for (int i = 0; i < D / 32; ++i) {
        const float4 q = q4p[l8 + 8 * i];
        const float4 k = kp[l8 + 8 * i];
        acc = fmaf(q.x, k.x, fmaf(q.y, k.y, fmaf(q.z, k.z, fmaf(q.w, k.w, acc))));
      }
      acc += __shfl_xor_sync(0xffffffffu, acc, 1);
      acc += __shfl_xor_sync(0xffffffffu, acc, 2);
      acc += __shfl_xor_sync(0xffffffffu, acc, 4);
      if (l8 == 0 && c < nch) score[c] = acc;
    }
  }
  __syncthreads();
  select_from_scores(score, key, rank, wsum, nch, topk, idx + ((size_t)b * g.Hkv + kvh) * topk);
}

// One thread per 16-byte vector of the block's K and V.
template <typename T>
__global__ void kv_append_kernel(const CacheGeom g, const int32_t* lens, int S,
                                 const T* __restrict__ Kb, const T* __restrict__ Vb,
                                 T* __restrict__ Kc, T* __restrict__ Vc, int32_t* status) {
  // may start before the previous kernel in the stream has finished
  pdl_wait();
  pdl_launch_dependents();
  constexpr int VEC = 16 / sizeof(T);
  const long long nvec_row = g.D / VEC;
  const long long total = (long long)g.B * S * g.Hkv * nvec_row;
  for (long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x; i < total;
       i += (long long)gridDim.x * blockDim.x) {
    const int v = (int)(i % nvec_row);
    long long r = i / nvec_row;
    const int kvh = (int)(r % g.Hkv);
    r /= g.Hkv;
    const int t = (int)(r % S);
    const int b = (int)(r / S);
    const int L = lens[b];
    if (L < 0 || L + S > g.cap) {
      if (t == 0 && kvh == 0 && v == 0) report(status, FB_ERR_BOUNDS);
      continue;
    }
    const long long dst = cache_offset(g, b, L + t, kvh);
    if (dst < 0) {
      report(status, FB_ERR_BOUNDS);
      continue;
    }
    const size_t src = (((size_t)b * S + t) * g.Hkv + kvh) * g.D + (size_t)v * VEC;
    *reinterpret_cast<uint4*>(Kc + dst + v * VEC) = *reinterpret_cast<const uint4*>(Kb + src);
    *reinterpret_cast<uint4*>(Vc + dst + v * VEC) = *reinterpret_cast<const uint4*>(Vb + src);
  }
}

// grid (Hkv, B), block 32: the valid chunks that chunk_idx does not list, in
// ascending order, padded with -1.  Shared memory: one flag per chunk.
__global__ void complement_chunks_kernel(const CacheGeom g, const int32_t* lens, int chunk_size,
                                         int nch_total, int topk, const int32_t* __restrict__ idx,
                                         int32_t* __restrict__ comp, int comp_cap, int32_t* status) {
  // may start before the previous kernel in the stream has finished
  pdl_wait();
  pdl_launch_dependents();
  extern __shared__ int flag[];
  const int kvh = blockIdx.x, b = blockIdx.y;
  int L = lens[b];
  if (L < 0 || L > g.cap) {
    if (threadIdx.x == 0) report(status, FB_ERR_BOUNDS);
    L = max(0, min(L, g.cap));
  }
  const int nch = (L + chunk_size - 1) / chunk_size;
  for (int c = threadIdx.x; c < nch; c += blockDim.x) flag[c] = 0;
  __syncwarp();
  const int32_t* sel = idx + ((size_t)b * g.Hkv + kvh) * topk;
  for (int i = threadIdx.x; i < topk; i += blockDim.x) {
    const int c = sel[i];
    if (c >= 0 && c < nch) flag[c] = 1;
  }
  __syncwarp();
  if (threadIdx.x == 0) {
    int32_t* out = comp + ((size_t)b * g.Hkv + kvh) * comp_cap;
    int n = 0;
    for (int c = 0; c < nch; ++c) {
      if (flag[c]) continue;
      if (n < comp_cap) {
        out[n] = c;
      } else {
        report(status, FB_ERR_BOUNDS);
      }
      ++n;
    }
    for (; n < comp_cap; ++n) out[n] = -1;
  }
}

// One warp per query row: the merge equation of two partials (O, LSE) with
// m = max(L_a, L_b); rows where both are empty stay (0, -inf).
__global__ void merge_partials_kernel(int B, int S, int Hq, int D, const float* __restrict__ Oa,
                                      const float* __restrict__ La, const float* __restrict__ Ob,
                                      const float* __restrict__ Lb, float* Oo, float* Lo) {
  // may start before the previous kernel in the stream has finished
  pdl_wait();
  pdl_launch_dependents();
  const long long row = (long long)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  const long long nrows = (long long)B * S * Hq;
  if (row >= nrows) return;
  const int h = (int)(row % Hq);
  const long long bt = row / Hq;
  const int t = (int)(bt % S);
  const int b = (int)(bt / S);
  const size_t lrow = ((size_t)b * Hq + h) * S + t;
  const float la = La[lrow], lb = Lb[lrow];
  const float m = fmaxf(la, lb);
  const bool empty = (m == -CUDART_INF_F);
  const float wa = (empty || la == -CUDART_INF_F) ? 0.f : expf(la - m);
  const float wb = (empty || lb == -CUDART_INF_F) ? 0.f : expf(lb - m);
  const float den = wa + wb;
  const float inv = den > 0.f ? 1.f / den : 0.f;
  for (int d = lane * 4; d < D; d += 128) {
    const float4 a = *reinterpret_cast<const float4*>(Oa + row * D + d);
    const float4 c = *reinterpret_cast<const float4*>(Ob + row * D + d);
    float4 o;
    o.x = (wa * a.x + wb * c.x) * inv;
    o.y = (wa * a.y + wb * c.y) * inv;
    o.z = (wa * a.z + wb * c.z) * inv;
    o.w = (wa * a.w + wb * c.w) * inv;
    *reinterpret_cast<float4*>(Oo + row * D + d) = o;
  }
  __syncwarp();
  if (lane == 0) Lo[lrow] = empty ? -CUDART_INF_F : m + logf(den);
}

// Runs after the copy: advance each length by S when the block fitted.
__global__ void lens_advance_kernel(int32_t* lens, int B, int S, int cap) {
  // may start before the previous kernel in the stream has finished
  pdl_wait();
  pdl_launch_dependents();
  const int b = blockIdx.x * blockDim.x + threadIdx.x;
  if (b < B) {
    const int L = lens[b];
    if (L >= 0 && L + S <= cap) lens[b] = L + S;
  }
}

}  // namespace

cudaError_t launch_chunk_means(const fb_desc& d, const void* K, int c0, int c1, int tail_rows, float* Kmean,
                               int32_t* status, cudaStream_t stream) {
  const CacheGeom g = geom_of(d);
  const int nch_total = (g.cap + d.chunk_size - 1) / d.chunk_size;
  // tail mode: tail_rows rows straddle at most this many chunks
  const int nblk = tail_rows > 0 ? (tail_rows + d.chunk_size - 1) / d.chunk_size + 1 : c1 - c0;
  if (nblk <= 0) return cudaSuccess;
  dim3 grid(nblk, g.Hkv, g.B);
  cudaError_t e;
  if (d.dtype == FB_BF16)
    e = launch_pdl(chunk_means_kernel<__nv_bfloat16>, grid, dim3(g.D), 0, stream, g, d.prefix_lens, d.chunk_size,
                   c0, tail_rows, nch_total, static_cast<const __nv_bfloat16*>(K), Kmean, status);
  else
    e = launch_pdl(chunk_means_kernel<float>, grid, dim3(g.D), 0, stream, g, d.prefix_lens, d.chunk_size, c0,
                   tail_rows, nch_total, static_cast<const float*>(K), Kmean, status);
  note_launch();
  return e != cudaSuccess ? e : cudaGetLastError();
}

cudaError_t launch_select_chunks(const fb_desc& d, const void* Q, const float* Kmean, int32_t* idx,
                                 int32_t* status, cudaStream_t stream) {
  const CacheGeom g = geom_of(d);
  const int nch_total = (g.cap + d.chunk_size - 1) / d.chunk_size;
  dim3 grid(g.Hkv, g.B);
  cudaError_t e;
  // every input of a unit in shared memory, when it fits and the bulk copies'
  // 16-byte alignment holds
  const size_t esz = d.dtype == FB_BF16 ? 2 : 4;
  const int rows = d.block_len * (d.num_q_heads / g.Hkv);
  constexpr size_t BULK_SMEM_MAX = 220 * 1024;
  const size_t bulk_smem = sel_bulk_smem_bytes(rows, nch_total, esz);
  const size_t bulk_tx = (size_t)nch_total * SELB_D * 4 + (size_t)rows * SELB_D * esz;
  if (g.D == SELB_D && bulk_smem <= BULK_SMEM_MAX && bulk_tx < (1u << 20) &&
      (reinterpret_cast<uintptr_t>(Q) & 15) == 0 && (reinterpret_cast<uintptr_t>(Kmean) & 15) == 0) {
    int dev = 0;
    e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    // the shared-memory limit of the bulk kernels, raised once per device
    static std::atomic<bool> configured[64][2];
    const int which = d.dtype == FB_BF16 ? 0 : 1;
    void (*kb)(CacheGeom, const int32_t*, int, int, int, int, int, const __nv_bfloat16*, const float*, int32_t*,
               int32_t*) = select_chunks_bulk_kernel<__nv_bfloat16>;
    void (*kf)(CacheGeom, const int32_t*, int, int, int, int, int, const float*, const float*, int32_t*,
               int32_t*) = select_chunks_bulk_kernel<float>;
    if (dev >= 64 || !configured[dev][which].load(std::memory_order_acquire)) {
      e = which == 0 ? cudaFuncSetAttribute(kb, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)BULK_SMEM_MAX)
                     : cudaFuncSetAttribute(kf, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)BULK_SMEM_MAX);
      if (e != cudaSuccess) return e;
      if (dev < 64) configured[dev][which].store(true, std::memory_order_release);
    }
    if (which == 0)
      e = launch_pdl(kb, grid, dim3(SEL_THREADS), bulk_smem, stream, g, d.prefix_lens, d.chunk_size, nch_total,
                     d.block_len, d.num_q_heads, d.topk, static_cast<const __nv_bfloat16*>(Q), Kmean, idx, status);
    else
      e = launch_pdl(kf, grid, dim3(SEL_THREADS), bulk_smem, stream, g, d.prefix_lens, d.chunk_size, nch_total,
                     d.block_len, d.num_q_heads, d.topk, static_cast<const float*>(Q), Kmean, idx, status);
    note_launch();
    return e != cudaSuccess ? e : cudaGetLastError();
  }
  const size_t smem = sel_smem_bytes(g.D, nch_total);
  if (d.dtype == FB_BF16) {
    auto k = select_chunks_kernel<__nv_bfloat16>;
    if (smem > 48 * 1024) cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    e = launch_pdl(k, grid, dim3(SEL_THREADS), smem, stream, g, d.prefix_lens, d.chunk_size, nch_total,
                   d.block_len, d.num_q_heads, d.topk, static_cast<const __nv_bfloat16*>(Q), Kmean, idx, status);
  } else {
    auto k = select_chunks_kernel<float>;
    if (smem > 48 * 1024) cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    e = launch_pdl(k, grid, dim3(SEL_THREADS), smem, stream, g, d.prefix_lens, d.chunk_size, nch_total,
                   d.block_len, d.num_q_heads, d.topk, static_cast<const float*>(Q), Kmean, idx, status);
  }
  note_launch();
  return e != cudaSuccess ? e : cudaGetLastError();
}

cudaError_t launch_complement_chunks(const fb_desc& d, const int32_t* idx, int32_t* comp, int comp_cap,
                                     int32_t* status, cudaStream_t stream) {
  const CacheGeom g = geom_of(d);
  const int nch_total = (g.cap + d.chunk_size - 1) / d.chunk_size;
  dim3 grid(g.Hkv, g.B);
  const size_t smem = (size_t)nch_total * sizeof(int);
  if (smem > 48 * 1024)
    cudaFuncSetAttribute(complement_chunks_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  cudaError_t e = launch_pdl(complement_chunks_kernel, grid, dim3(32), smem, stream, g, d.prefix_lens,
                             d.chunk_size, nch_total, d.topk, idx, comp, comp_cap, status);
  note_launch();
  return e != cudaSuccess ? e : cudaGetLastError();
}

cudaError_t launch_merge_partials(const fb_desc& d, const float* Oa, const float* La, const float* Ob,
                                  const float* Lb, float* Oo, float* Lo, cudaStream_t stream) {
  const long long rows = (long long)d.batch * d.block_len * d.num_q_heads;
  const int warps = 8;
  cudaError_t e = launch_pdl(merge_partials_kernel, dim3((unsigned)((rows + warps - 1) / warps)), dim3(warps * 32),
                             0, stream, d.batch, d.block_len, d.num_q_heads, d.head_dim, Oa, La, Ob, Lb, Oo, Lo);
  note_launch();
  return e != cudaSuccess ? e : cudaGetLastError();
}

cudaError_t launch_kv_append(const fb_desc& d, const void* Kb, const void* Vb, void* Kc, void* Vc,
                             int32_t* lens_inout, int32_t* status, cudaStream_t stream) {
  const CacheGeom g = geom_of(d);
  const int32_t* lens = lens_inout ? lens_inout : d.prefix_lens;
  const int esz = d.dtype == FB_BF16 ? 2 : 4;
  const long long total = (long long)g.B * d.block_len * g.Hkv * (g.D * esz / 16);
  const int threads = 256;
  const long long want = (total + threads - 1) / threads;
  const int grid = (int)(want < 148 * 16 ? want : 148 * 16);
  cudaError_t e;
  if (d.dtype == FB_BF16)
    e = launch_pdl(kv_append_kernel<__nv_bfloat16>, dim3(grid), dim3(threads), 0, stream, g, lens, d.block_len,
                   static_cast<const __nv_bfloat16*>(Kb), static_cast<const __nv_bfloat16*>(Vb),
                   static_cast<__nv_bfloat16*>(Kc), static_cast<__nv_bfloat16*>(Vc), status);
  else
    e = launch_pdl(kv_append_kernel<float>, dim3(grid), dim3(threads), 0, stream, g, lens, d.block_len,
                   static_cast<const float*>(Kb), static_cast<const float*>(Vb), static_cast<float*>(Kc),
                   static_cast<float*>(Vc), status);
  note_launch();
  if (e == cudaSuccess) e = cudaGetLastError();
  if (e != cudaSuccess || !lens_inout) return e;
  // (waits for the append above to complete before it moves the lengths)
  return launch_lens_advance(d, lens_inout, stream);
}

cudaError_t launch_lens_advance(const fb_desc& d, int32_t* lens, cudaStream_t stream) {
  const CacheGeom g = geom_of(d);
  cudaError_t e = launch_pdl(lens_advance_kernel, dim3((g.B + 127) / 128), dim3(128), 0, stream, lens, g.B,
                             d.block_len, g.cap);
  note_launch();
  return e != cudaSuccess ? e : cudaGetLastError();
}

}  // namespace fb
