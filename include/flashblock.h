/*
 * flashblock.h -- C ABI of libflashblock.so: cached block-diffusion attention
 * (FlashBlock) on NVIDIA B200 (sm_100a).
 *
 * The method ("FlashBlock: Attention Caching for Efficient Long-Context Block
 * Diffusion", Technical Summary §2 Methodology, Core Mechanism): at every
 * denoising step of the active block, softmax attention over
 * [finalized prefix ; block] splits into a block-external partial over the
 * prefix (A_out, L_out = log Z_out) and a block-internal partial over the block
 * (A_in, L_in).  The external pair is computed at a refresh step and reused on
 * later steps; each step merges it with a fresh internal partial by the
 * log-space merge equation
 *     A = (e^{L_out-m} A_out + e^{L_in-m} A_in) / (e^{L_out-m} + e^{L_in-m}),
 *     m = max(L_out, L_in).
 *
 * Conventions shared by every call
 * --------------------------------
 *  - Every tensor pointer is a DEVICE pointer, contiguous, 16-byte aligned,
 *    owned by the caller.  The library allocates no memory; scratch memory is
 *    the caller's `workspace` (size from fb_workspace_bytes()).
 *  - Layouts (row-major, innermost last):
 *      Q, O            [B, S, Hq, D]
 *      K/V cache       contiguous [B, kv_capacity, Hkv, D], or a page pool
 *                      [num_pages, page_size, Hkv, D] addressed through
 *                      block_table [B, max_pages] (int32, device)
 *      K/V block       [B, S, Hkv, D]
 *      O_pre           [B, S, Hq, D] float32
 *      LSE, LSE_pre    [B, Hq, S] float32, natural log of the unnormalised sum
 *      Kmean           [B, Hkv, ceil(capacity / chunk_size), D] float32
 *      chunk_idx       [B, Hkv, topk] int32, ascending, padded with -1
 *    Query head h reads KV head h / (Hq / Hkv).
 *  - dtype FB_BF16: Q, K, V, O are bfloat16 (tensor-core path, D = 128).
 *    dtype FB_FP32: Q, K, V, O are float32 (CUDA-core path, D in {32,64,96,128}).
 *    Accumulation is float32 in both.
 *  - Calls are asynchronous on `stream` (a cudaStream_t; NULL = legacy default
 *    stream) and deterministic: fixed split order, no floating-point atomics.
 *  - Errors: argument checks run on the host before anything is launched and
 *    return a non-zero fb_status synchronously.  Faults found on the device
 *    (an index out of range, a pipeline wait past its time limit) are written
 *    to *dev_status (device int32, nullable; the first error sticks, the
 *    caller zeroes it and reads it after synchronising).  The library never
 *    traps.
 *  - The library keeps no per-call state and is safe to call from several host
 *    threads; concurrent calls must not share output or workspace buffers.
 */
#ifndef FLASHBLOCK_H
#define FLASHBLOCK_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* 2: fb_block_step and fb_block_step_append take an optional workspace. */
#define FB_ABI_VERSION 2

/* Same type as cudaStream_t. */
typedef struct CUstream_st* fb_stream_t;

typedef enum fb_status {
  FB_OK = 0,
  FB_ERR_INVALID_ARG = 1,    /* null pointer, non-positive or inconsistent size */
  FB_ERR_UNSUPPORTED = 2,    /* valid but not implemented (head_dim, group size, dtype) */
  FB_ERR_ALIGNMENT = 3,      /* a tensor pointer is not 16-byte aligned */
  FB_ERR_WORKSPACE = 4,      /* workspace missing or smaller than fb_workspace_bytes() */
  FB_ERR_LAUNCH = 5,         /* no CUDA device, or the runtime refused a launch */
  FB_ERR_DEVICE_TIMEOUT = 6, /* device-side: a pipeline wait exceeded its time limit */
  FB_ERR_BOUNDS = 7          /* device-side: page, chunk or cache row out of range */
} fb_status;

typedef enum fb_dtype { FB_BF16 = 0, FB_FP32 = 1 } fb_dtype;

typedef struct fb_desc {
  int32_t batch;          /* B >= 1 */
  int32_t num_q_heads;    /* Hq >= 1 */
  int32_t num_kv_heads;   /* Hkv >= 1, Hq % Hkv == 0; bf16 needs G = Hq/Hkv a power of two <= 128 */
  int32_t head_dim;       /* D */
  int32_t block_len;      /* S >= 1: tokens of the active block */
  int32_t dtype;          /* fb_dtype */
  float softmax_scale;    /* > 0: logits are softmax_scale * (q . k) */
  int32_t kv_capacity;    /* contiguous cache: rows per sequence; paged: unused */
  int32_t page_size;      /* 0 = contiguous cache; else a power of two >= 64 */
  int32_t max_pages;      /* paged: columns of block_table */
  int32_t num_pages;      /* paged: pages in the pool */
  const int32_t* block_table; /* paged: device [B, max_pages]; else NULL */
  const int32_t* prefix_lens; /* device [B]: valid prefix rows L_b (0 allowed) */
  int32_t chunk_size;     /* sparse prefix: tokens per chunk, a multiple of 128; 0 if unused */
  int32_t topk;           /* sparse prefix: chunks kept per (b, kv head); 0 = dense prefix */
  int32_t num_splits;     /* prefix pass: key-range splits per work unit; 0 = library's choice */
} fb_desc;

/* Rows each sequence can hold: kv_capacity (contiguous) or max_pages*page_size (paged). */
int64_t fb_cache_rows(const fb_desc* d);

/* Bytes of device workspace that fb_prefix_partial and fb_full_reference_gpu
 * need for this descriptor on the current device (split-key partials:
 * splits x B x S x Hq x (D + 1) float32), and that lets fb_block_step split
 * the keys of a nearly empty last wave of CTAs (see there).  0 means no
 * workspace is needed. */
size_t fb_workspace_bytes(const fb_desc* d);

/* Block-external partial over the finalized prefix (the cached pair).
 * Core Mechanism: A_out and L_out = log Z_out over J_out, the tokens outside
 * the current block, here the prefix rows j < prefix_lens[b].  With
 * d->topk > 0 the key set of each (b, kv head) is the union of the chunks
 * listed in chunk_idx (the sparse prefix; see fb_select_chunks).
 * Q [B,S,Hq,D] (dtype); Kcache/Vcache (dtype; contiguous or paged);
 * chunk_idx [B,Hkv,topk] int32 or NULL when topk == 0.
 * Writes O_pre [B,S,Hq,D] float32 (normalised) and LSE_pre [B,Hq,S] float32;
 * an empty key set gives O_pre = 0, LSE_pre = -inf. */
fb_status fb_prefix_partial(const fb_desc* d, const void* Q, const void* Kcache,
                            const void* Vcache, const int32_t* chunk_idx,
                            float* O_pre, float* LSE_pre, void* workspace,
                            size_t workspace_bytes, int32_t* dev_status,
                            fb_stream_t stream);

/* One cached denoising step.  Core Mechanism: the block-internal partial of
 * Q over the block's own keys (bidirectional, no mask) merged in the same
 * kernel with the cached (O_pre, LSE_pre) by the merge equation.
 * Q [B,S,Hq,D], Kblk/Vblk [B,S,Hkv,D] (dtype).  Writes O [B,S,Hq,D] (dtype)
 * and, when LSE_out is not NULL, the merged LSE [B,Hq,S] float32.
 * workspace: optional (NULL, or fewer than fb_workspace_bytes(d) bytes, is
 * allowed).  With it, a long block (S > 64, bf16) whose one-CTA-per-unit grid
 * ends in a nearly empty wave splits the keys of that wave's units and merges
 * their partials with the cached pair in a second kernel (the same result up
 * to rounding); without it every unit keeps one CTA. */
fb_status fb_block_step(const fb_desc* d, const void* Q, const void* Kblk,
                        const void* Vblk, const float* O_pre, const float* LSE_pre,
                        void* O, float* LSE_out, void* workspace, size_t workspace_bytes,
                        int32_t* dev_status, fb_stream_t stream);

/* Uncached block diffusion (Technical Summary §1 Problem Statement): attention
 * of Q over [prefix rows j < L_b ; all S block rows] in one pass, no cached
 * partial.  The dense prefix is always used (topk is ignored).
 * Writes O [B,S,Hq,D] (dtype) and, when LSE_out is not NULL, LSE [B,Hq,S]. */
fb_status fb_full_reference_gpu(const fb_desc* d, const void* Q, const void* Kcache,
                                const void* Vcache, const void* Kblk, const void* Vblk,
                                void* O, float* LSE_out, void* workspace,
                                size_t workspace_bytes, int32_t* dev_status,
                                fb_stream_t stream);

/* Sparse prefix, step 1 (Adaptive Reuse Strategies, "Compatibility with
 * Sparse Attention": the selected keys are attended, the rest form J_out).
 * Mean key of chunks [chunk_begin, chunk_end) over their valid rows
 * j < prefix_lens[b]; chunks without a valid row get 0.  Call once for the
 * whole prefix and again for the chunks an append touched.
 * Kmean [B, Hkv, ceil(rows / chunk_size), D] float32. */
fb_status fb_chunk_means(const fb_desc* d, const void* Kcache, int32_t chunk_begin,
                         int32_t chunk_end, float* Kmean, int32_t* dev_status,
                         fb_stream_t stream);

/* Sparse prefix, step 1 after an append (Technical Summary §1: each finished
 * block joins the cache that later blocks attend to): the same means for the
 * chunks holding each sequence's last `rows` valid rows, j in
 * [max(L_b - rows, 0), L_b), with L_b = prefix_lens[b] read on the device.
 * Called with rows = S after fb_kv_append has advanced prefix_lens, it
 * refreshes exactly the chunks the append touched, with no host-side length,
 * so a block recorded once (in a CUDA graph, say) keeps the means current as
 * the sequence grows.  rows > 0.  Kmean as for fb_chunk_means. */
fb_status fb_chunk_means_tail(const fb_desc* d, const void* Kcache, int32_t rows, float* Kmean,
                              int32_t* dev_status, fb_stream_t stream);

/* Sparse prefix, step 2: per (b, kv head) score every valid chunk c by
 * qbar . Kmean[c], qbar the mean of Q over the S block tokens and the G query
 * heads of the group, and keep the top d->topk (ties to the lower index).
 * Writes chunk_idx [B,Hkv,topk] int32 in ascending chunk order, -1 padded. */
fb_status fb_select_chunks(const fb_desc* d, const void* Q, const float* Kmean,
                           int32_t* chunk_idx, int32_t* dev_status, fb_stream_t stream);

/* Residual reuse with sparse attention (Adaptive Reuse Strategies,
 * Compatibility with Sparse Attention: the unselected keys are the
 * block-external set whose contribution is cached).  For each (b, kv head),
 * the valid chunks (those holding a row j < prefix_lens[b]) that
 * chunk_idx [B,Hkv,d->topk] does not list, ascending, padded with -1, into
 * comp_idx [B,Hkv,comp_cap].  More than comp_cap of them records
 * FB_ERR_BOUNDS.  Pass comp_idx to fb_prefix_partial with topk = comp_cap to
 * get the residual partial. */
fb_status fb_complement_chunks(const fb_desc* d, const int32_t* chunk_idx, int32_t* comp_idx,
                               int32_t comp_cap, int32_t* dev_status, fb_stream_t stream);

/* The merge equation on two partials (Core Mechanism): with m = max(L_a, L_b),
 * O = (e^{L_a-m} O_a + e^{L_b-m} O_b) / (e^{L_a-m} + e^{L_b-m}) and
 * L = m + log(e^{L_a-m} + e^{L_b-m}); two empty partials give (0, -inf).
 * O_* [B,S,Hq,D] float32, LSE_* [B,Hq,S] float32; O_out/LSE_out may alias
 * an input. */
fb_status fb_merge_partials(const fb_desc* d, const float* O_a, const float* LSE_a,
                            const float* O_b, const float* LSE_b, float* O_out,
                            float* LSE_out, fb_stream_t stream);

/* ---- Adaptive reuse: refresh masks ("Adaptive Reuse Strategies") ----------
 * Instead of refreshing the cached block-external pair at fixed steps, a
 * policy decides at every step which work units recompute it.  A refresh
 * mask is device int32 [B, Hkv] (1 = recompute the (b, kv head) unit's pair
 * with this step's queries, 0 = keep the cached one); the policy calls below
 * write it and fb_prefix_partial_masked consumes it. */

/* Head-wise Selection: unit (b, kvh) refreshes when the cosine similarity of
 * its queries now (Q_now [B,S,Hq,D], heads kvh*G .. kvh*G+G-1) to the
 * reference queries (Q_ref, same layout: the queries the unit's cached pair
 * was computed with) is below gamma, i.e. sim < gamma; a NaN similarity
 * refreshes, and a unit whose two query sets are all zero has similarity 1.
 * The similarity is taken over the unit's S x G x D values, accumulated in
 * float32.  A refreshed unit's Q_now values are copied into Q_ref (which the
 * caller owns and keeps between steps).  gamma = +inf refreshes every unit
 * whatever Q_ref holds (use it on the first step of a block).  sim_out (device
 * float32 [B, Hkv]) may be NULL.  Q pointers 16-byte aligned.  Returns
 * FB_ERR_INVALID_ARG for a NaN gamma. */
fb_status fb_headwise_refresh_mask(const fb_desc* d, const void* Q_now, void* Q_ref, float gamma,
                                   int32_t* unit_mask, float* sim_out, fb_stream_t stream);

/* Threshold-based Reuse: sequence b refreshes (all its units) when M_b >= tau,
 * M_b the number of block tokens t whose key or value moved by more than eps
 * since the previous step: max over kv heads and dims of |K_now - K_prev| or
 * of |V_now - V_prev| above eps (differences taken in float32).  K/V blocks
 * [B,S,Hkv,D] in the descriptor's dtype, 16-byte aligned.  K_prev / V_prev
 * are state the caller owns: the call overwrites them with K_now / V_now, so
 * the next step compares with this one.  tau <= 0 refreshes every sequence
 * whatever K_prev / V_prev hold (use it on the first step of a block).
 * count_out (device int32 [B], M_b) may be NULL.  ws: device workspace of at
 * least fb_workspace_bytes(d) bytes (16-byte aligned; it may be the one the
 * prefix pass uses).  Returns FB_ERR_INVALID_ARG for a NaN eps. */
fb_status fb_threshold_refresh_mask(const fb_desc* d, void* K_prev, void* V_prev, const void* K_now,
                                    const void* V_now, float eps, int32_t tau, int32_t* unit_mask,
                                    int32_t* count_out, void* ws, size_t ws_bytes, fb_stream_t stream);

/* fb_prefix_partial restricted to the units a refresh mask selects: units
 * with unit_mask[b*Hkv + kvh] != 0 get (O_pre, LSE_pre) rows recomputed
 * exactly as fb_prefix_partial computes them; the rows of the other units are
 * not read or written (they keep the cached pair).  unit_mask: device int32
 * [B, Hkv], read on the device (no host synchronisation).  Other arguments,
 * workspace rule and errors as for fb_prefix_partial. */
fb_status fb_prefix_partial_masked(const fb_desc* d, const void* Q, const void* Kcache,
                                   const void* Vcache, const int32_t* chunk_idx,
                                   const int32_t* unit_mask, float* O_pre, float* LSE_pre, void* ws,
                                   size_t ws_bytes, int32_t* dev_status, fb_stream_t stream);

/* Block end (Technical Summary §1: the KV cache of finished blocks, which
 * later blocks attend to causally): copy the finalized block's K/V [B,S,Hkv,D] into cache rows
 * [L_b, L_b + S) (contiguous or paged).  When lens_inout is not NULL
 * (device [B]), it is read for L_b and then advanced by S.  A block that does
 * not fit records FB_ERR_BOUNDS in dev_status and is not written. */
fb_status fb_kv_append(const fb_desc* d, const void* Kblk, const void* Vblk,
                       void* Kcache, void* Vcache, int32_t* lens_inout,
                       int32_t* dev_status, fb_stream_t stream);

/* The last denoising step of a block, with the block's append: the same
 * results as fb_block_step followed by fb_kv_append(d, Kblk, Vblk, Kcache,
 * Vcache, lens_inout, ...) (Core Mechanism: the step's output; Technical
 * Summary §1: the finished block joins the cache).  For short blocks (S <= 64,
 * bf16) it is one kernel -- the step kernel also writes the block's K/V rows
 * into the cache rows [L_b, L_b + S) -- plus the length update when
 * lens_inout is not NULL; other shapes run the two calls.  Arguments, layouts
 * and errors as for those two calls. */
fb_status fb_block_step_append(const fb_desc* d, const void* Q, const void* Kblk, const void* Vblk,
                               const float* O_pre, const float* LSE_pre, void* O, float* LSE_out,
                               void* Kcache, void* Vcache, int32_t* lens_inout, void* workspace,
                               size_t workspace_bytes, int32_t* dev_status, fb_stream_t stream);

/* Bytes of the static scratch array behind fb_prefix_partial_noalloc. */
#define FB_NOALLOC_SCRATCH_BYTES ((size_t)16 << 20)

/* fb_prefix_partial for callers that cannot allocate device memory: an
 * embedding whose memory planner hands out one fixed device arena at start-up
 * and forbids allocator calls afterwards, a plug-in host that gives its
 * plug-ins no allocator, or a latency-critical serving loop that cannot afford
 * the device-wide synchronisation a cudaMalloc or cudaFree may cause.  No
 * counterpart in the paper: it is a deployment variant of the prefix pass.
 * Same arguments and results as fb_prefix_partial without the workspace: the
 * split-key partials go to a FB_NOALLOC_SCRATCH_BYTES array inside the
 * library's device image, present on every GPU that loads the library until
 * the process exits.
 *  - Allocates nothing and calls no allocating routine.
 *  - Returns FB_ERR_WORKSPACE (nothing launched) when this call's partials
 *    need more than FB_NOALLOC_SCRATCH_BYTES (fb_workspace_bytes() says how
 *    much a descriptor needs; long single sequences fit, e.g. 9.5 MB at
 *    B = 1, S = 32, Hq = 32, 128K prefix).
 *  - The first call on each device looks up the array's device address with
 *    that device current; make that first call before any stream capture.
 *    The lookup is repeated when the device's context has changed (after a
 *    device reset), so the call after a reset is a first call again.
 *  - All calls share the one array, which keeps the last call's contents
 *    (nothing in it needs to start at zero).  Calls that can overlap on the
 *    GPU (other streams, other host threads) race on it: serialise them. */
fb_status fb_prefix_partial_noalloc(const fb_desc* d, const void* Q, const void* Kcache,
                                    const void* Vcache, const int32_t* chunk_idx,
                                    float* O_pre, float* LSE_pre, int32_t* dev_status,
                                    fb_stream_t stream);

/* Human-readable name of a status code (static storage). */
const char* fb_status_string(fb_status s);

/* Number of kernels this library has launched in this process. */
uint64_t fb_launch_count(void);

/* FB_ABI_VERSION of the loaded library. */
int32_t fb_abi_version(void);

#ifdef __cplusplus
}
#endif

#endif /* FLASHBLOCK_H */
