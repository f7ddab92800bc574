// fb_internal.h -- kernel parameter blocks and launchers shared between the
// C-ABI layer (fb_api.cu) and the kernel translation units.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "flashblock.h"

namespace fb {

// Output stage of the attention kernels.
enum Epilogue : int {
  EPI_PARTIAL = 0,  // normalised O (f32) + LSE: the cached pair, or one split's part
  EPI_MERGE = 1,    // merge with (O_pre, LSE_pre), write O in the input dtype + LSE
  EPI_NORM = 2,     // normalise, write O in the input dtype + LSE
};

// Where the keys of one (batch, kv head) work unit come from.  Virtual tile
// index j runs over the prefix tiles first, then the block tiles.
struct KeySource {
  int has_prefix;     // 1: prefix rows j < prefix_lens[b] take part
  int has_block;      // 1: all S block rows take part (after the prefix)
  int paged;          // prefix cache is a page pool
  int page_shift;     // log2(page_size) when paged
  int max_pages;      // columns of block_table
  int num_pages;      // pool pages
  int cap;            // rows per sequence (contiguous capacity or pages*page_size)
  const int32_t* block_table;
  const int32_t* prefix_lens;
  const int32_t* chunk_idx;  // sparse prefix list [B, Hkv, topk] or null
  int topk;
  int chunk_size;
};

struct AttnParams {
  int B, Hq, Hkv, G, S, D;
  int n_rt;      // row tiles per work unit (tensor-core path)
  int nsplit;    // key-range splits per unit (EPI_PARTIAL only)
  float scale;   // softmax scale (natural units)
  float scale_log2;  // scale * log2(e)
  int epi;
  int kv_stream_once;  // 1: prefix K/V is read once (evict-first L2 hint)
  const int32_t* unit_mask;  // [B, Hkv] or null: units with 0 are skipped (their outputs kept)
  // 1: the grid's CTAs are shared out among the units unit_mask selects
  // (active-unit split, EPI_PARTIAL only): CTA i writes its partial rows to
  // slot i of out_o32 ([grid][128][D]) and out_lse ([grid][128])
  int dyn;
  // Two-tile kernel with nsplit = 1 (any epilogue): the units from tail_u0 on
  // (the last, partial wave of CTAs) are split tail_k ways over their keys
  // (tail_k = 0: no such split).  CTA tail_u0 + i is split i % tail_k of
  // unit tail_u0 + i / tail_k; it writes its two tiles' partial rows to
  // slots 2 i and 2 i + 1 of tail_o ([slots][128][D], through the kernel's
  // second output map) and tail_lse ([slots][128]).
  int tail_u0, tail_k;
  float* tail_o;
  float* tail_lse;
  KeySource src;
  // Test builds only (FB_TEST_HOOKS): 1 = every CTA's K producer leaves the
  // load of its second key tile out, so the pipeline wait for it runs out
  // (the time-out path is then exercised).  Always 0 in the library proper.
  int test_skip_k1;
  // outputs
  float* out_o32;         // EPI_PARTIAL: [nsplit][B][S][Hq][D]
  float* out_lse;         // EPI_PARTIAL: [nsplit][B][Hq][S]; others: [B][Hq][S] or null
  void* out_o;            // EPI_MERGE / EPI_NORM: [B][S][Hq][D] in the input dtype
  const float* pre_o;     // EPI_MERGE inputs
  const float* pre_lse;
  int32_t* dev_status;
};

struct CombineParams {
  int B, Hq, S, D, nsplit;
  int G;                  // query heads per kv head (for unit_mask)
  const int32_t* unit_mask;  // [B, Hkv] or null: rows of units with 0 are left as they are
  int dyn;                // partials in the active-unit slot layout of AttnParams::dyn
  int grid, n_rt;         // (dyn) the attention launch's CTAs and query tiles per unit
  // tail_k > 0: merge only the tail units' rows, from the slot layout of
  // AttnParams::tail_o (tail_units units from tail_u0 on, npair tile pairs
  // per (b, kv head), Hkv kv heads)
  int tail_k, tail_u0, tail_units, npair, Hkv;
  // tail_k > 0 and not null: the cached pair joins the merge as one more
  // partial (the step's merge equation); then tail_k < 32
  const float* pre_o;     // [B][S][Hq][D]
  const float* pre_lse;   // [B][Hq][S] natural log
  const float* part_o;    // [nsplit][B][S][Hq][D]
  const float* part_lse;  // [nsplit][B][Hq][S]
  float* out_o32;         // f32 output (prefix pass) or null
  void* out_o;            // dtype output (full attention) or null
  int out_bf16;           // out_o element type: 1 bf16, 0 f32
  float* out_lse;         // [B][Hq][S] or null
};

// Tensor-core (bf16) path.
constexpr int TC_BM = 128;      // query rows per tile (TMEM lanes)
constexpr int TC_BN = 128;      // keys per tile
constexpr int TC_D = 128;       // head dim
constexpr int TC_SLOTS = 6;     // K/V ring: 32 KB slots (K and V of a tile take one each)
constexpr int TC_THREADS = 224; // 4 softmax warps, K/Q TMA warp, MMA warp, V TMA warp
constexpr int TC_MAX_SPLITS = 128;  // key-range splits per work unit
size_t tc_smem_bytes();
// Launch with programmatic stream serialization: the kernel may start while
// its predecessor in the stream finishes; it must call griddepcontrol.wait
// (pdl_wait) before reading anything that predecessor writes.
template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t stream,
                       Args... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, args...);
}

// ---- active-unit split plan (shared by the attention kernel and the combine)
// Every lane of the calling warp must take part (warp ballots over the mask).
__device__ __forceinline__ int active_count(const int32_t* mask, int nu) {
  const int lane = threadIdx.x & 31;
  int n = 0;
  for (int i0 = 0; i0 < nu; i0 += 32)
    n += __popc(__ballot_sync(0xffffffffu, i0 + lane < nu && mask[i0 + lane] != 0));
  return n;
}
// Number of active units before unit u.
__device__ __forceinline__ int active_rank(const int32_t* mask, int u) {
  const int lane = threadIdx.x & 31;
  int n = 0;
  for (int i0 = 0; i0 < u; i0 += 32)
    n += __popc(__ballot_sync(0xffffffffu, i0 + lane < u && mask[i0 + lane] != 0));
  return n;
}
// Index of the a-th active unit (0-based), or -1.
__device__ __forceinline__ int active_unit(const int32_t* mask, int nu, int a) {
  const int lane = threadIdx.x & 31;
  int base = 0;
  for (int i0 = 0; i0 < nu; i0 += 32) {
    unsigned m = __ballot_sync(0xffffffffu, i0 + lane < nu && mask[i0 + lane] != 0);
    const int c = __popc(m);
    if (a < base + c) {
      for (int k = a - base; k > 0; --k) m &= m - 1;  // drop the lower set bits
      return i0 + __ffs(m) - 1;
    }
    base += c;
  }
  return -1;
}
// Key splits per (active unit, query tile) when `grid` CTAs are shared out.
__device__ __forceinline__ int active_splits(int grid, int n_active, int n_rt) {
  if (n_active <= 0) return 1;
  const int ns = grid / (n_active * n_rt);
  return ns < 1 ? 1 : (ns > TC_MAX_SPLITS ? TC_MAX_SPLITS : ns);
}

// Geometry of a K/V cache (contiguous [B, cap, Hkv, D] or a page pool
// [num_pages, page, Hkv, D] addressed through block_table).
struct CacheGeom {
  int B, Hkv, D, cap, paged, page_shift, max_pages, num_pages;
  const int32_t* block_table;
};

inline CacheGeom geom_of(const fb_desc& d) {
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

// Block step of a short block on warp-level MMA (16 query rows per CTA, the
// tile in registers): usable when small_step_fits().
// With `app`, the step also writes the block's K/V into the cache rows
// [L_b, L_b + S) (the append of a block's last step; lens is not advanced).
struct StepAppend {
  const int32_t* lens;
  void* Kc;
  void* Vc;
  int32_t* status;
};
bool small_step_fits(const fb_desc& d, int num_sms);
cudaError_t launch_block_step_small(const fb_desc& d, const void* Q, const void* Kb, const void* Vb,
                                    const float* O_pre, const float* LSE_pre, void* O, float* LSE_out,
                                    cudaStream_t stream, const StepAppend* app = nullptr);
// The same on 64 query rows per CTA (16 per warp), for short blocks with more
// rows than small_step_fits() takes: usable when rows_step_fits().
bool rows_step_fits(const fb_desc& d);
cudaError_t launch_block_step_rows(const fb_desc& d, const void* Q, const void* Kb, const void* Vb,
                                   const float* O_pre, const float* LSE_pre, void* O, float* LSE_out,
                                   cudaStream_t stream, const StepAppend* app = nullptr);
// Advances lens[b] by S where the block fitted (after the append).
cudaError_t launch_lens_advance(const fb_desc& d, int32_t* lens, cudaStream_t stream);

cudaError_t launch_attn_tc(const AttnParams& p, const CUtensorMap& tmQ, const CUtensorMap& tmKp,
                           const CUtensorMap& tmVp, const CUtensorMap& tmKb, const CUtensorMap& tmVb,
                           const CUtensorMap& tmPre, const CUtensorMap& tmO, int grid, cudaStream_t stream);
cudaError_t launch_combine(const CombineParams& c, cudaStream_t stream);
// Two 128-row query tiles per CTA (tiles 2i and 2i + 1 of a unit; the grid is
// (b, kv head, tile pair, split) with the split fastest): for units of two or
// more query tiles.  No active-unit split (AttnParams::dyn must be 0).
// tmT: the tail slots' map (AttnParams::tail_o), or any map when tail_k = 0.
cudaError_t launch_attn_tc2(const AttnParams& p, const CUtensorMap& tmQ, const CUtensorMap& tmKp,
                            const CUtensorMap& tmVp, const CUtensorMap& tmKb, const CUtensorMap& tmVb,
                            const CUtensorMap& tmO, const CUtensorMap& tmT, int grid, cudaStream_t stream);

// CUDA-core (fp32) path.
cudaError_t launch_attn_simt(const AttnParams& p, const float* Q, const float* Kp,
                             const float* Vp, const float* Kb, const float* Vb,
                             cudaStream_t stream);

// Sparse prefix helpers and the cache append.
// Chunks [chunk_begin, chunk_end) of every sequence, or (tail_rows > 0) the
// chunks holding each sequence's last tail_rows valid rows by its device length.
cudaError_t launch_chunk_means(const fb_desc& d, const void* K, int chunk_begin, int chunk_end, int tail_rows,
                               float* Kmean, int32_t* dev_status, cudaStream_t stream);
cudaError_t launch_select_chunks(const fb_desc& d, const void* Q, const float* Kmean,
                                 int32_t* idx, int32_t* dev_status, cudaStream_t stream);
cudaError_t launch_complement_chunks(const fb_desc& d, const int32_t* idx, int32_t* comp, int comp_cap,
                                     int32_t* dev_status, cudaStream_t stream);
cudaError_t launch_merge_partials(const fb_desc& d, const float* Oa, const float* La, const float* Ob,
                                  const float* Lb, float* Oo, float* Lo, cudaStream_t stream);
cudaError_t launch_headwise_mask(const fb_desc& d, const void* Qnow, void* Qref, float gamma, int32_t* mask,
                                 float* sim, cudaStream_t stream);
cudaError_t launch_threshold_mask(const fb_desc& d, void* Kprev, void* Vprev, const void* Know, const void* Vnow,
                                  float eps, int32_t tau, int32_t* mask, int32_t* count, int32_t* ws,
                                  cudaStream_t stream);
size_t threshold_ws_bytes(const fb_desc& d);  // per-slice token counts of the threshold pass
cudaError_t launch_kv_append(const fb_desc& d, const void* Kb, const void* Vb, void* Kc, void* Vc,
                             int32_t* lens_inout, int32_t* dev_status, cudaStream_t stream);

// Count of kernels launched (process-wide).
void note_launch(int n = 1);

// First error wins; later ones are dropped.
__device__ __forceinline__ void report(int32_t* status, int code) {
  if (status) atomicCAS(status, 0, code);
}

}  // namespace fb
