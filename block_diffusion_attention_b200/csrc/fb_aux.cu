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

#include "fb_internal.h"
#include "fb_ptx.cuh"

namespace fb {

namespace {

struct CacheGeom {
  int B, Hkv, D, cap, paged, page_shift, max_pages, num_pages;
  const int32_t* block_table;
};

CacheGeom geom_of(const fb_desc& d) {
  CacheGeom g;
  g.B = d.batch;
  g.Hkv = d.num_kv_heads;
  g.D = d.head_dim;
  g.paged = d.page_size > 0;
  g.page_shift = 0;
  if (g.paged)
    while ((1 << g.page_shift) < d.page_size) ++g.page_shift;
  g.max_pages = d.max_pages;
  g.num_pages = d.num_pages;
  g.cap = g.paged ? d.max_pages * d.page_size : d.kv_capacity;
  g.block_table = d.block_table;
  return g;
}

// Element offset of cache row `pos` of sequence b, kv head kvh; -1 if the row
// has no valid page.
__device__ __forceinline__ long long cache_offset(const CacheGeom& g, int b, int pos, int kvh) {
  if (g.paged) {
    const int pi = pos >> g.page_shift;
    if (pi >= g.max_pages) return -1;
    const int pg = g.block_table[(size_t)b * g.max_pages + pi];
    if (pg < 0 || pg >= g.num_pages) return -1;
    const int prow = pos & ((1 << g.page_shift) - 1);
    return (((long long)pg << g.page_shift) + prow) * g.Hkv * g.D + (long long)kvh * g.D;
  }
  return ((long long)b * g.cap + pos) * g.Hkv * g.D + (long long)kvh * g.D;
}

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

// grid (Hkv, B), block SEL_THREADS.  Dynamic shared memory:
// SEL_PART_FLOATS + D floats for the query mean, nch scores, nch flags.
constexpr int SEL_WARPS = 8, SEL_THREADS = SEL_WARPS * 32;
constexpr int SEL_PART_FLOATS = SEL_THREADS * 8;  // row-group sums of the query mean (16-bit inputs)

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
  // query mean over the S block tokens and the G heads of the group: the
  // unit's S x G rows of D values are read as 16-byte vectors, thread i taking
  // vector i % vpr of rows i / vpr, i / vpr + rpi, ...; the rpi row sums of
  // each column are then added in a fixed order
  constexpr int VEC = 16 / sizeof(T);
  const int vpr = g.D / VEC;                // vectors per row
  const int rpi = SEL_THREADS / vpr;        // rows per iteration
  float* part = sm;                         // [rpi][D] row-group sums
  float* qbar = sm + SEL_PART_FLOATS;       // [D]
  float* score = qbar + g.D;                // [nch_total]
  int* sel = reinterpret_cast<int*>(score + nch_total);
  int L = lens[b];
  if (L < 0 || L > g.cap) {
    if (threadIdx.x == 0) report(status, FB_ERR_BOUNDS);
    L = max(0, min(L, g.cap));
  }
  const int nch = (L + chunk_size - 1) / chunk_size;
  const int rows = S * G;
  {
    const int vi = threadIdx.x % vpr, r0 = threadIdx.x / vpr;
    if (r0 < rpi) {
      float acc[VEC];
#pragma unroll
      for (int k = 0; k < VEC; ++k) acc[k] = 0.f;
#pragma unroll 16
      for (int rr = r0; rr < rows; rr += rpi) {
        const int t = rr / G, gg = rr - t * G;
        const uint4 v =
            *reinterpret_cast<const uint4*>(Q + (((size_t)b * S + t) * Hq + kvh * G + gg) * g.D + vi * VEC);
        add_vec16<T>(v, acc);
      }
#pragma unroll
      for (int k = 0; k < VEC; ++k) part[r0 * g.D + vi * VEC + k] = acc[k];
    }
  }
  __syncthreads();
  for (int d = threadIdx.x; d < g.D; d += SEL_THREADS) {
    float acc = 0.f;
    for (int w2 = 0; w2 < rpi; ++w2) acc += part[w2 * g.D + d];
    qbar[d] = acc / (float)rows;
  }
  __syncthreads();
  // score of chunk c: four lanes per chunk, each over a quarter of D with
  // 16-byte loads (all independent), then two shuffles
  const float* km = Kmean + ((size_t)b * g.Hkv + kvh) * nch_total * g.D;
  // two chunks per lane group per pass, so a 128-chunk prefix needs one pass
  // with all of its loads in flight
  const int q4 = threadIdx.x & 3, dq = g.D / 4;
  constexpr int CPP = SEL_THREADS / 4;  // chunks per half-pass
  for (int base = 0; base < nch; base += 2 * CPP) {
    const int c0 = base + (threadIdx.x >> 2), c1 = c0 + CPP;
    float acc0 = 0.f, acc1 = 0.f;
    const float4* qr = reinterpret_cast<const float4*>(qbar + q4 * dq);
    const float4* kr0 = reinterpret_cast<const float4*>(km + (size_t)c0 * g.D + q4 * dq);
    const float4* kr1 = reinterpret_cast<const float4*>(km + (size_t)c1 * g.D + q4 * dq);
#pragma unroll 8
    for (int i = 0; i < dq / 4; ++i) {
      const float4 q = qr[i];
      const float4 k0 = c0 < nch ? kr0[i] : make_float4(0.f, 0.f, 0.f, 0.f);
      const float4 k1 = c1 < nch ? kr1[i] : make_float4(0.f, 0.f, 0.f, 0.f);
      acc0 = fmaf(q.x, k0.x, fmaf(q.y, k0.y, fmaf(q.z, k0.z, fmaf(q.w, k0.w, acc0))));
      acc1 = fmaf(q.x, k1.x, fmaf(q.y, k1.y, fmaf(q.z, k1.z, fmaf(q.w, k1.w, acc1))));
    }
    acc0 += __shfl_xor_sync(0xffffffffu, acc0, 1);
    acc0 += __shfl_xor_sync(0xffffffffu, acc0, 2);
    acc1 += __shfl_xor_sync(0xffffffffu, acc1, 1);
    acc1 += __shfl_xor_sync(0xffffffffu, acc1, 2);
    if (q4 == 0 && c0 < nch) score[c0] = acc0;
    if (q4 == 0 && c1 < nch) score[c1] = acc1;
  }
  __syncthreads();
  // rank = chunks that beat c (higher score, or equal score and lower index)
  for (int c = threadIdx.x; c < nch; c += SEL_THREADS) {
    const float sc = score[c];
    int better = 0;
    for (int c2 = 0; c2 < nch; ++c2) {
      const float s2 = score[c2];
      better += (s2 > sc) || (s2 == sc && c2 < c);
    }
    sel[c] = better < topk;
  }
  __syncthreads();
  // ascending chunk order: output slot = selected chunks before c
  int32_t* out = idx + ((size_t)b * g.Hkv + kvh) * topk;
  for (int c = threadIdx.x; c < nch; c += SEL_THREADS) {
    if (sel[c]) {
      int before = 0;
      for (int c2 = 0; c2 < c; ++c2) before += sel[c2];
      out[before] = c;
    }
  }
  const int nsel = min(topk, nch);
  for (int i = nsel + threadIdx.x; i < topk; i += SEL_THREADS) out[i] = -1;
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
  const size_t smem = (size_t)(SEL_PART_FLOATS + g.D + nch_total) * sizeof(float) + (size_t)nch_total * sizeof(int);
  dim3 grid(g.Hkv, g.B);
  cudaError_t e;
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
  e = launch_pdl(lens_advance_kernel, dim3((g.B + 127) / 128), dim3(128), 0, stream, lens_inout, g.B, d.block_len,
                 g.cap);
  note_launch();
  return e != cudaSuccess ? e : cudaGetLastError();
}

}  // namespace fb
