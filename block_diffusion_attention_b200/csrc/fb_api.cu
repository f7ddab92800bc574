// fb_api.cu -- the extern "C" entry points of libflashblock.so: argument
// checks, work decomposition (query-row tiles, key-range splits), TMA tensor
// maps and kernel dispatch.  See include/flashblock.h for the contract.
#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <algorithm>
#include <atomic>
#include <cmath>
#include <cstring>
#include <mutex>

#include "fb_internal.h"

namespace fb {

static std::atomic<uint64_t> g_launches{0};
void note_launch(int n) { g_launches.fetch_add((uint64_t)n, std::memory_order_relaxed); }

#ifdef FB_TEST_HOOKS
static std::atomic<int> g_test_skip_k1{0};
#endif

namespace {

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(ptr);
  });
  return fn;
}

// 4-D tensor map, innermost dimension first, 128-byte swizzle (bf16 unless
// `f32` is set).
bool make_map(CUtensorMap* m, const void* base, const uint64_t dims[4], const uint64_t strides_bytes[3],
              const uint32_t box[4], bool f32 = false) {
  auto fn = encode_fn();
  if (!fn) return false;
  cuuint64_t gd[4] = {dims[0], dims[1], dims[2], dims[3]};
  cuuint64_t gs[3] = {strides_bytes[0], strides_bytes[1], strides_bytes[2]};
  cuuint32_t bx[4] = {box[0], box[1], box[2], box[3]};
  cuuint32_t es[4] = {1, 1, 1, 1};
  CUresult r = fn(m, f32 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT32 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4,
                  const_cast<void*>(base), gd, gs, bx, es,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// SM count of the current device, cached per device (host threads may call
// concurrently: each entry is written once with the same value, atomically).
int device_sms() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 148;
  static std::atomic<int> cache[64];
  if (dev >= 0 && dev < 64) {
    const int c = cache[dev].load(std::memory_order_relaxed);
    if (c > 0) return c;
  }
  int n = 0;
  if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) n = 148;
  if (dev >= 0 && dev < 64) cache[dev].store(n, std::memory_order_relaxed);
  return n;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
bool pow2(int x) { return x > 0 && (x & (x - 1)) == 0; }
int log2i(int x) {
  int s = 0;
  while ((1 << s) < x) ++s;
  return s;
}

int64_t cache_rows(const fb_desc& d) {
  return d.page_size > 0 ? (int64_t)d.max_pages * d.page_size : (int64_t)d.kv_capacity;
}

fb_status check_desc(const fb_desc* d) {
  if (!d) return FB_ERR_INVALID_ARG;
  if (d->batch <= 0 || d->num_q_heads <= 0 || d->num_kv_heads <= 0 || d->head_dim <= 0 ||
      d->block_len <= 0)
    return FB_ERR_INVALID_ARG;
  if (d->num_q_heads % d->num_kv_heads) return FB_ERR_INVALID_ARG;
  if (!(d->softmax_scale > 0.f) || !std::isfinite(d->softmax_scale)) return FB_ERR_INVALID_ARG;
  if (d->dtype == FB_BF16) {
    if (d->head_dim != TC_D) return FB_ERR_UNSUPPORTED;
    const int G = d->num_q_heads / d->num_kv_heads;
    if (!pow2(G) || G > TC_BM) return FB_ERR_UNSUPPORTED;
  } else if (d->dtype == FB_FP32) {
    if (d->head_dim % 32 || d->head_dim > 128) return FB_ERR_UNSUPPORTED;
  } else {
    return FB_ERR_UNSUPPORTED;
  }
  return FB_OK;
}

fb_status check_cache(const fb_desc* d) {
  if (!d->prefix_lens || (reinterpret_cast<uintptr_t>(d->prefix_lens) & 3u)) return FB_ERR_INVALID_ARG;
  if (d->page_size > 0) {
    if (!pow2(d->page_size) || d->page_size < 64) return FB_ERR_UNSUPPORTED;
    if (!d->block_table || d->max_pages <= 0 || d->num_pages <= 0) return FB_ERR_INVALID_ARG;
    if (cache_rows(*d) > (int64_t)1 << 30) return FB_ERR_UNSUPPORTED;
  } else {
    if (d->page_size < 0 || d->kv_capacity < 0) return FB_ERR_INVALID_ARG;
  }
  return FB_OK;
}

fb_status check_sparse(const fb_desc* d, const int32_t* chunk_idx) {
  if (d->topk < 0) return FB_ERR_INVALID_ARG;
  if (d->topk == 0) return FB_OK;
  if (!chunk_idx) return FB_ERR_INVALID_ARG;
  if (d->chunk_size <= 0 || d->chunk_size % TC_BN) return FB_ERR_UNSUPPORTED;
  return FB_OK;
}

KeySource key_source(const fb_desc& d, bool prefix, bool block, const int32_t* chunk_idx) {
  KeySource s;
  std::memset(&s, 0, sizeof(s));
  s.has_prefix = prefix;
  s.has_block = block;
  if (prefix) {
    s.paged = d.page_size > 0;
    s.page_shift = s.paged ? log2i(d.page_size) : 0;
    s.max_pages = d.max_pages;
    s.num_pages = d.num_pages;
    s.cap = (int)cache_rows(d);
    s.block_table = d.block_table;
    s.prefix_lens = d.prefix_lens;
    s.chunk_idx = (d.topk > 0) ? chunk_idx : nullptr;
    s.topk = d.topk;
    s.chunk_size = d.chunk_size;
  }
  return s;
}

AttnParams base_params(const fb_desc& d) {
  AttnParams p;
  std::memset(&p, 0, sizeof(p));
  p.B = d.batch;
  p.Hq = d.num_q_heads;
  p.Hkv = d.num_kv_heads;
  p.G = d.num_q_heads / d.num_kv_heads;
  p.S = d.block_len;
  p.D = d.head_dim;
  p.n_rt = (d.block_len * p.G + TC_BM - 1) / TC_BM;
  p.nsplit = 1;
  p.scale = d.softmax_scale;
  p.scale_log2 = d.softmax_scale * 1.4426950408889634f;
  p.kv_stream_once = (p.n_rt == 1);  // one query tile per unit: each K/V byte is read once
#ifdef FB_TEST_HOOKS
  p.test_skip_k1 = g_test_skip_k1.load(std::memory_order_relaxed);
#endif
  return p;
}

// Query tiles (128 packed rows) of one (b, kv head) unit.
int row_tiles(const fb_desc& d) {
  const int G = d.num_q_heads / d.num_kv_heads;
  return (d.block_len * G + TC_BM - 1) / TC_BM;
}

// Units of two or more query tiles run on the two-tile kernel: one CTA per
// pair of tiles, each K/V tile loaded once for both.
bool use_pairs(const fb_desc& d) { return d.dtype == FB_BF16 && row_tiles(d) >= 2; }

// CTAs of one key split: (b, kv head, query tile) or (b, kv head, tile pair).
long long cta_units(const fb_desc& d) {
  const int rt = row_tiles(d);
  return (long long)d.batch * d.num_kv_heads * (use_pairs(d) ? (rt + 1) / 2 : rt);
}

// Tail split of the two-tile kernel.  Unsplit, the grid's last wave can be
// nearly empty: 760 tile pairs at the video shape are five full waves of 148
// and one of 20, so a sixth of the pass runs on 20 SMs.  Where that last wave
// holds at most half the SMs, its units can be split k ways over their keys
// instead (k about SMs / tail units, at least 3 key tiles per split, at most
// 31 splits, so that the combine holds them and the step's cached pair in
// one warp), into slots the combine merges, while the other units keep one
// CTA each.  tail_splits gives that k (0: no tail split).
long long tail_splits(long long units, long long slots, long long est_tiles) {
  const long long tail = units % slots;
  if (units <= slots || tail == 0 || 2 * tail > slots) return 0;
  const long long k = std::min<long long>(slots / tail, std::min<long long>(est_tiles / 3, 31));
  return k >= 2 ? k : 0;
}

// Key-range splits of the prefix pass.  Cost model in key-tile times: every
// wave of CTAs costs its longest split plus a fixed per-CTA overhead (set-up,
// pipeline fill, epilogue ~ 3 tiles), and splitting adds a combine pass
// (~ 2 tiles).  Splits keep at least 3 tiles each.
int choose_splits(const fb_desc& d, long long est_tiles) {
  if (d.dtype != FB_BF16) return 1;
  const long long units = cta_units(d);
  long long max_ns = est_tiles / 3;
  if (max_ns < 1) max_ns = 1;
  if (max_ns > TC_MAX_SPLITS) max_ns = TC_MAX_SPLITS;
  if (d.num_splits > 0)
    return (int)std::min<long long>(std::min<long long>(d.num_splits, TC_MAX_SPLITS), std::max<long long>(est_tiles, 1));
  const long long slots = device_sms();
  // Four or more waves of CTAs without splitting: a split would only add
  // the combine, whose partials (f32, one set per split) are large next to
  // the work per wave (video shape: 3.10 ms with five splits, 2.93 ms with
  // none).
  if (units >= 4 * slots) return 1;
  int best = 1;
  double best_cost = 1e30;
  for (long long ns = 1; ns <= max_ns; ++ns) {
    const long long waves = (units * ns + slots - 1) / slots;
    const double per_split = std::ceil((double)est_tiles / (double)ns);
    const double cost = (double)waves * (per_split + 3.0) + (ns > 1 ? 2.0 : 0.0);
    if (cost < best_cost - 1e-9) {
      best_cost = cost;
      best = (int)ns;
    }
  }
  // One-tile units (an HBM-streaming pass): the fewest splits whose cost is
  // within 7 % of the best.  The model counts work per SM, but such a pass
  // gains nothing from more CTAs once HBM is saturated, and every split adds
  // partials to combine (128K dense prefix, 8 kv heads: 17 splits 92.2 us,
  // 18 splits 97.2 us, 16 splits 92.2-94.1 us, 15 splits 95.9-97.4 us).
  // Not for two-tile units, which are bound by the tensor pipe and the
  // softmax: one wave of 128 unsplit CTAs on 148 SMs (uncached pass, 16
  // sequences, 32K dense prefix) took 504 us against 457 us for 8 splits.
  for (long long ns = 1; ns < best && !use_pairs(d); ++ns) {
    const long long waves = (units * ns + slots - 1) / slots;
    const double cost = (double)waves * (std::ceil((double)est_tiles / (double)ns) + 3.0) + (ns > 1 ? 2.0 : 0.0);
    if (cost <= 1.07 * best_cost) {
      best = (int)ns;
      best_cost = cost;
      break;
    }
  }
  // One split with the tail split (see tail_plan) where that is cheaper: the
  // full waves of unsplit units, then the tail units' splits, then the combine.
  if (use_pairs(d)) {
    const long long k = tail_splits(units, slots, est_tiles);
    if (k > 0) {
      const double cost = (double)(units / slots) * ((double)est_tiles + 3.0) +
                          (std::ceil((double)est_tiles / (double)k) + 3.0) + 2.0;
      if (cost < best_cost - 1e-9) return 1;
    }
  }
  return best;
}

long long prefix_tiles_estimate(const fb_desc& d) {
  if (d.topk > 0) return (long long)d.topk * ((d.chunk_size + TC_BN - 1) / TC_BN);
  return (cache_rows(d) + TC_BN - 1) / TC_BN;
}

// The masked prefix pass shares its grid out among the selected units (one
// slot of 128 partial rows per CTA) when the full pass fills at most two
// waves: there, dropping units would not shorten the pass.
bool use_active_split(const fb_desc& d, long long grid) { return grid <= 2LL * device_sms(); }

size_t active_split_bytes(long long grid) { return (size_t)grid * TC_BM * (TC_D + 1) * sizeof(float); }

size_t split_bytes(const fb_desc& d, int ns) {
  if (ns <= 1) return 0;
  const size_t rows = (size_t)d.batch * d.block_len * d.num_q_heads;
  return (size_t)ns * rows * (size_t)(d.head_dim + 1) * sizeof(float);
}

// The tail split of a pass planned with one split (choose_splits), where it
// applies: two-tile units, no explicit split count.
struct TailPlan {
  int u0 = 0;     // first tail unit
  int units = 0;  // tail units
  int k = 0;      // splits per tail unit (0: no tail split)
};

TailPlan tail_plan(const fb_desc& d, int ns, long long est_tiles) {
  TailPlan t;
  if (ns != 1 || !use_pairs(d) || d.num_splits > 0) return t;
  const long long units = cta_units(d);
  const long long slots = device_sms();
  const long long k = tail_splits(units, slots, est_tiles);
  if (k == 0) return t;
  t.u0 = (int)(units - units % slots);
  t.units = (int)(units % slots);
  t.k = (int)k;
  return t;
}

// The tail split of the tensor-core step (two-tile units, S > 64): one CTA
// per unit otherwise, so where its cost model (full waves, then the tail's
// splits, then the combine) beats the plain grid.
TailPlan step_tail_plan(const fb_desc& d) {
  TailPlan t;
  if (d.dtype != FB_BF16 || small_step_fits(d, device_sms()) || rows_step_fits(d) || !use_pairs(d)) return t;
  const long long units = cta_units(d);
  const long long slots = device_sms();
  const long long est = (d.block_len + TC_BN - 1) / TC_BN;
  const long long k = tail_splits(units, slots, est);
  if (k == 0) return t;
  const double plain = (double)((units + slots - 1) / slots) * ((double)est + 3.0);
  const double split = (double)(units / slots) * ((double)est + 3.0) + (std::ceil((double)est / (double)k) + 3.0) + 2.0;
  if (split >= plain) return t;
  t.u0 = (int)(units - units % slots);
  t.units = (int)(units % slots);
  t.k = (int)k;
  return t;
}

// Slots of the tail splits: (tail unit, split, tile) x 128 rows x (D + 1) f32.
size_t tail_bytes(const TailPlan& t) {
  return (size_t)t.units * t.k * 2 * TC_BM * (TC_D + 1) * sizeof(float);
}

fb_status from_cuda(cudaError_t e) { return e == cudaSuccess ? FB_OK : FB_ERR_LAUNCH; }

struct Maps {
  CUtensorMap q, kp, vp, kb, vb;
};

bool q_map(CUtensorMap* m, const fb_desc& d, const void* Q) {
  const int G = d.num_q_heads / d.num_kv_heads;
  const uint64_t D = d.head_dim, Hq = d.num_q_heads, S = d.block_len, B = d.batch;
  const uint64_t dims[4] = {D, Hq, S, B};
  const uint64_t str[3] = {D * 2, Hq * D * 2, S * Hq * D * 2};
  const uint32_t box[4] = {64, (uint32_t)G, (uint32_t)(TC_BM / G), 1};
  return make_map(m, Q, dims, str, box);
}

// Cached O_pre [B, S, Hq, D] f32 in the packed query-row order of a tile:
// 32-float column blocks (128 B) of G heads x 128/G tokens; also the map the
// prefix pass stores its partials through,
// `outer` sequences of that layout (B, or splits x B for the split partials).
bool pre_map(CUtensorMap* m, const fb_desc& d, const float* O_pre, int outer = 0) {
  const int G = d.num_q_heads / d.num_kv_heads;
  const uint64_t D = d.head_dim, Hq = d.num_q_heads, S = d.block_len;
  const uint64_t B = outer > 0 ? (uint64_t)outer : (uint64_t)d.batch;
  const uint64_t dims[4] = {D, Hq, S, B};
  const uint64_t str[3] = {D * 4, Hq * D * 4, S * Hq * D * 4};
  const uint32_t box[4] = {32, (uint32_t)G, (uint32_t)(TC_BM / G), 1};
  return make_map(m, O_pre, dims, str, box, true);
}

// Active-unit split partials: `slots` blocks of 128 packed rows x D f32, in
// the same 32-float column boxes as pre_map.
bool slot_map(CUtensorMap* m, const fb_desc& d, const float* base, int slots) {
  const int G = d.num_q_heads / d.num_kv_heads;
  const uint64_t D = d.head_dim;
  const uint64_t dims[4] = {D, (uint64_t)G, (uint64_t)(TC_BM / G), (uint64_t)slots};
  const uint64_t str[3] = {D * 4, (uint64_t)G * D * 4, (uint64_t)TC_BM * D * 4};
  const uint32_t box[4] = {32, (uint32_t)G, (uint32_t)(TC_BM / G), 1};
  return make_map(m, base, dims, str, box, true);
}

// The two-tile kernel with the tail split tp (its slots at the start of ws),
// then the combine of the tail rows into the outputs (and, for the step, the
// cached pair) that c names.
fb_status run_tail_split(AttnParams p, const TailPlan& tp, const fb_desc& d, void* ws, const CUtensorMap& q,
                         const CUtensorMap& kp, const CUtensorMap& vp, const CUtensorMap& kb,
                         const CUtensorMap& vb, const CUtensorMap& tm_out, CombineParams c, cudaStream_t s) {
  const int slots = tp.units * tp.k * 2;
  float* tail_o = static_cast<float*>(ws);
  float* tail_l = tail_o + (size_t)slots * TC_BM * TC_D;
  p.nsplit = 1;
  p.tail_u0 = tp.u0;
  p.tail_k = tp.k;
  p.tail_o = tail_o;
  p.tail_lse = tail_l;
  CUtensorMap tm_tail;
  if (!slot_map(&tm_tail, d, tail_o, slots)) return FB_ERR_LAUNCH;
  const cudaError_t e = launch_attn_tc2(p, q, kp, vp, kb, vb, tm_out, tm_tail, tp.u0 + tp.units * tp.k, s);
  if (e != cudaSuccess) return from_cuda(e);
  c.B = d.batch;
  c.Hq = d.num_q_heads;
  c.S = d.block_len;
  c.D = d.head_dim;
  c.G = p.G;
  c.part_o = tail_o;
  c.part_lse = tail_l;
  c.tail_k = tp.k;
  c.tail_u0 = tp.u0;
  c.tail_units = tp.units;
  c.npair = (p.n_rt + 1) / 2;
  c.Hkv = d.num_kv_heads;
  return from_cuda(launch_combine(c, s));
}

bool block_map(CUtensorMap* m, const fb_desc& d, const void* X) {
  const uint64_t D = d.head_dim, H = d.num_kv_heads, S = d.block_len, B = d.batch;
  const uint64_t dims[4] = {D, H, S, B};
  const uint64_t str[3] = {D * 2, H * D * 2, S * H * D * 2};
  const uint32_t box[4] = {64, 1, TC_BN, 1};
  return make_map(m, X, dims, str, box);
}

bool cache_map(CUtensorMap* m, const fb_desc& d, const void* X) {
  const uint64_t D = d.head_dim, H = d.num_kv_heads;
  if (d.page_size > 0) {
    const uint64_t P = d.page_size, N = d.num_pages;
    const uint64_t dims[4] = {D, H, P, N};
    const uint64_t str[3] = {D * 2, H * D * 2, P * H * D * 2};
    const uint32_t box[4] = {64, 1, (uint32_t)(d.page_size < TC_BN ? d.page_size : TC_BN), 1};
    return make_map(m, X, dims, str, box);
  }
  const uint64_t cap = d.kv_capacity > 0 ? (uint64_t)d.kv_capacity : 1, B = d.batch;
  const uint64_t dims[4] = {D, H, cap, B};
  const uint64_t str[3] = {D * 2, H * D * 2, cap * H * D * 2};
  const uint32_t box[4] = {64, 1, TC_BN, 1};
  return make_map(m, X, dims, str, box);
}

}  // namespace
}  // namespace fb

using namespace fb;

extern "C" {

int64_t fb_cache_rows(const fb_desc* d) { return d ? cache_rows(*d) : -1; }

size_t fb_workspace_bytes(const fb_desc* d) {
  if (check_desc(d) != FB_OK) return 0;
  const int ns_pre = choose_splits(*d, prefix_tiles_estimate(*d));
  fb_desc dense = *d;
  dense.topk = 0;
  const long long est_full = prefix_tiles_estimate(dense) + (d->block_len + TC_BN - 1) / TC_BN;
  const int ns_full = choose_splits(dense, est_full);
  size_t need = split_bytes(*d, ns_pre);
  need = std::max(need, tail_bytes(tail_plan(*d, ns_pre, prefix_tiles_estimate(*d))));
  need = std::max(need, split_bytes(*d, ns_full));
  need = std::max(need, tail_bytes(tail_plan(dense, ns_full, est_full)));
  need = std::max(need, tail_bytes(step_tail_plan(*d)));
  need = std::max(need, threshold_ws_bytes(*d));
  if (d->dtype == FB_BF16 && !use_pairs(*d)) {
    // the masked prefix pass's active-unit slots
    const long long grid = cta_units(*d) * ns_pre;
    if (use_active_split(*d, grid)) need = std::max(need, active_split_bytes(grid));
  }
  return need;
}

}  // extern "C"

namespace {

fb_status prefix_partial(const fb_desc* d, const void* Q, const void* Kc, const void* Vc,
                         const int32_t* chunk_idx, const int32_t* unit_mask, float* O_pre, float* LSE_pre,
                         void* ws, size_t ws_bytes, int32_t* dev_status, fb_stream_t stream) {
  fb_status st = check_desc(d);
  if (st != FB_OK) return st;
  if ((st = check_cache(d)) != FB_OK) return st;
  if ((st = check_sparse(d, chunk_idx)) != FB_OK) return st;
  if (!Q || !Kc || !Vc || !O_pre || !LSE_pre) return FB_ERR_INVALID_ARG;
  if (!aligned16(Q) || !aligned16(Kc) || !aligned16(Vc) || !aligned16(O_pre) ||
      (reinterpret_cast<uintptr_t>(LSE_pre) & 3u))
    return FB_ERR_ALIGNMENT;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  AttnParams p = base_params(*d);
  p.src = key_source(*d, true, false, chunk_idx);
  p.epi = EPI_PARTIAL;
  p.dev_status = dev_status;
  p.unit_mask = unit_mask;
  if (d->dtype == FB_FP32) {
    p.out_o32 = O_pre;
    p.out_lse = LSE_pre;
    return from_cuda(launch_attn_simt(p, static_cast<const float*>(Q), static_cast<const float*>(Kc),
                                      static_cast<const float*>(Vc), nullptr, nullptr, s));
  }
  const int ns = choose_splits(*d, prefix_tiles_estimate(*d));
  const bool pairs = use_pairs(*d);
  const long long grid = cta_units(*d) * ns;
  const bool active = unit_mask != nullptr && !pairs && use_active_split(*d, grid);
  const size_t need = active ? active_split_bytes(grid) : split_bytes(*d, ns);
  if (need > 0 && (!ws || ws_bytes < need || !aligned16(ws))) return FB_ERR_WORKSPACE;
  Maps m;
  if (!q_map(&m.q, *d, Q) || !cache_map(&m.kp, *d, Kc) || !cache_map(&m.vp, *d, Vc))
    return FB_ERR_LAUNCH;
  if (active) {
    // partials in per-CTA slots, merged per active unit by the combine
    float* part_o = static_cast<float*>(ws);
    float* part_l = part_o + (size_t)grid * TC_BM * TC_D;
    p.dyn = 1;
    p.out_o32 = part_o;
    p.out_lse = part_l;
    CUtensorMap tm_out;
    if (!slot_map(&tm_out, *d, part_o, (int)grid)) return FB_ERR_LAUNCH;
    cudaError_t e = launch_attn_tc(p, m.q, m.kp, m.vp, m.kp, m.vp, m.q, tm_out, (int)grid, s);
    if (e != cudaSuccess) return from_cuda(e);
    CombineParams c;
    std::memset(&c, 0, sizeof(c));
    c.B = d->batch;
    c.Hq = d->num_q_heads;
    c.S = d->block_len;
    c.D = d->head_dim;
    c.part_o = part_o;
    c.part_lse = part_l;
    c.out_o32 = O_pre;
    c.out_lse = LSE_pre;
    c.G = p.G;
    c.unit_mask = unit_mask;
    c.dyn = 1;
    c.grid = (int)grid;
    c.n_rt = p.n_rt;
    return from_cuda(launch_combine(c, s));
  }
  // the tail split where the workspace holds its slots (else the plain plan)
  const TailPlan tp = pairs ? tail_plan(*d, ns, prefix_tiles_estimate(*d)) : TailPlan{};
  if (tp.k > 0 && ws && ws_bytes >= tail_bytes(tp) && aligned16(ws)) {
    p.out_o32 = O_pre;
    p.out_lse = LSE_pre;
    p.kv_stream_once = (p.n_rt <= 2);
    CUtensorMap tm_out;
    if (!pre_map(&tm_out, *d, O_pre, d->batch)) return FB_ERR_LAUNCH;
    CombineParams c;
    std::memset(&c, 0, sizeof(c));
    c.out_o32 = O_pre;
    c.out_lse = LSE_pre;
    c.unit_mask = unit_mask;
    return run_tail_split(p, tp, *d, ws, m.q, m.kp, m.vp, m.kp, m.vp, tm_out, c, s);
  }
  p.nsplit = ns;
  float* part_o = O_pre;
  float* part_l = LSE_pre;
  if (ns > 1) {
    part_o = static_cast<float*>(ws);
    part_l = part_o + (size_t)ns * d->batch * d->block_len * d->num_q_heads * d->head_dim;
  }
  p.out_o32 = part_o;
  p.out_lse = part_l;
  CUtensorMap tm_out;
  if (!pre_map(&tm_out, *d, part_o, d->batch * ns)) return FB_ERR_LAUNCH;
  cudaError_t e;
  if (pairs) {
    p.kv_stream_once = (p.n_rt <= 2);  // one tile pair per unit: each K/V byte is read once
    e = launch_attn_tc2(p, m.q, m.kp, m.vp, m.kp, m.vp, tm_out, tm_out, (int)grid, s);
  } else {
    e = launch_attn_tc(p, m.q, m.kp, m.vp, m.kp, m.vp, m.q, tm_out, (int)grid, s);
  }
  if (e != cudaSuccess || ns == 1) return from_cuda(e);
  CombineParams c;
  std::memset(&c, 0, sizeof(c));
  c.B = d->batch;
  c.Hq = d->num_q_heads;
  c.S = d->block_len;
  c.D = d->head_dim;
  c.nsplit = ns;
  c.part_o = part_o;
  c.part_lse = part_l;
  c.out_o32 = O_pre;
  c.out_lse = LSE_pre;
  c.G = p.G;
  c.unit_mask = unit_mask;
  return from_cuda(launch_combine(c, s));
}

}  // namespace

extern "C" {

fb_status fb_prefix_partial(const fb_desc* d, const void* Q, const void* Kc, const void* Vc,
                            const int32_t* chunk_idx, float* O_pre, float* LSE_pre, void* ws,
                            size_t ws_bytes, int32_t* dev_status, fb_stream_t stream) {
  return prefix_partial(d, Q, Kc, Vc, chunk_idx, nullptr, O_pre, LSE_pre, ws, ws_bytes, dev_status, stream);
}

fb_status fb_prefix_partial_masked(const fb_desc* d, const void* Q, const void* Kc, const void* Vc,
                                   const int32_t* chunk_idx, const int32_t* unit_mask, float* O_pre,
                                   float* LSE_pre, void* ws, size_t ws_bytes, int32_t* dev_status,
                                   fb_stream_t stream) {
  if (!unit_mask) return FB_ERR_INVALID_ARG;
  if (reinterpret_cast<uintptr_t>(unit_mask) & 3u) return FB_ERR_ALIGNMENT;
  return prefix_partial(d, Q, Kc, Vc, chunk_idx, unit_mask, O_pre, LSE_pre, ws, ws_bytes, dev_status, stream);
}

fb_status fb_headwise_refresh_mask(const fb_desc* d, const void* Q_now, void* Q_ref, float gamma,
                                   int32_t* unit_mask, float* sim_out, fb_stream_t stream) {
  fb_status st = check_desc(d);
  if (st != FB_OK) return st;
  if (!Q_now || !Q_ref || !unit_mask || std::isnan(gamma)) return FB_ERR_INVALID_ARG;
  if (!aligned16(Q_now) || !aligned16(Q_ref) || (reinterpret_cast<uintptr_t>(unit_mask) & 3u) ||
      (reinterpret_cast<uintptr_t>(sim_out) & 3u))
    return FB_ERR_ALIGNMENT;
  return from_cuda(launch_headwise_mask(*d, Q_now, Q_ref, gamma, unit_mask, sim_out,
                                        reinterpret_cast<cudaStream_t>(stream)));
}

fb_status fb_threshold_refresh_mask(const fb_desc* d, void* K_prev, void* V_prev, const void* K_now,
                                    const void* V_now, float eps, int32_t tau, int32_t* unit_mask,
                                    int32_t* count_out, void* ws, size_t ws_bytes, fb_stream_t stream) {
  fb_status st = check_desc(d);
  if (st != FB_OK) return st;
  if (!K_prev || !V_prev || !K_now || !V_now || !unit_mask || std::isnan(eps)) return FB_ERR_INVALID_ARG;
  if (!aligned16(K_prev) || !aligned16(V_prev) || !aligned16(K_now) || !aligned16(V_now) ||
      (reinterpret_cast<uintptr_t>(unit_mask) & 3u) || (reinterpret_cast<uintptr_t>(count_out) & 3u))
    return FB_ERR_ALIGNMENT;
  if (!ws || ws_bytes < threshold_ws_bytes(*d) || !aligned16(ws)) return FB_ERR_WORKSPACE;
  return from_cuda(launch_threshold_mask(*d, K_prev, V_prev, K_now, V_now, eps, tau, unit_mask, count_out,
                                         static_cast<int32_t*>(ws), reinterpret_cast<cudaStream_t>(stream)));
}

fb_status fb_block_step(const fb_desc* d, const void* Q, const void* Kb, const void* Vb,
                        const float* O_pre, const float* LSE_pre, void* O, float* LSE_out, void* ws,
                        size_t ws_bytes, int32_t* dev_status, fb_stream_t stream) {
  fb_status st = check_desc(d);
  if (st != FB_OK) return st;
  if (!Q || !Kb || !Vb || !O_pre || !LSE_pre || !O) return FB_ERR_INVALID_ARG;
  if (!aligned16(Q) || !aligned16(Kb) || !aligned16(Vb) || !aligned16(O_pre) || !aligned16(O) ||
      (reinterpret_cast<uintptr_t>(LSE_pre) & 3u) || (reinterpret_cast<uintptr_t>(LSE_out) & 3u))
    return FB_ERR_ALIGNMENT;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  AttnParams p = base_params(*d);
  p.src = key_source(*d, false, true, nullptr);
  p.epi = EPI_MERGE;
  p.pre_o = O_pre;
  p.pre_lse = LSE_pre;
  p.out_o = O;
  p.out_lse = LSE_out;
  p.dev_status = dev_status;
  if (d->dtype == FB_FP32)
    return from_cuda(launch_attn_simt(p, static_cast<const float*>(Q), nullptr, nullptr,
                                      static_cast<const float*>(Kb), static_cast<const float*>(Vb), s));
  if (small_step_fits(*d, device_sms()))
    return from_cuda(launch_block_step_small(*d, Q, Kb, Vb, O_pre, LSE_pre, O, LSE_out, s));
  if (rows_step_fits(*d))
    return from_cuda(launch_block_step_rows(*d, Q, Kb, Vb, O_pre, LSE_pre, O, LSE_out, s));
  Maps m;
  CUtensorMap tm_pre, tm_out;
  if (!q_map(&m.q, *d, Q) || !block_map(&m.kb, *d, Kb) || !block_map(&m.vb, *d, Vb) ||
      !pre_map(&tm_pre, *d, O_pre) || !q_map(&tm_out, *d, O))
    return FB_ERR_LAUNCH;
  const long long grid = cta_units(*d);
  if (use_pairs(*d)) {
    p.kv_stream_once = (p.n_rt <= 2);
    // the tail split (see tail_plan) where the workspace holds its slots:
    // the combine merges the tail's key splits and the cached pair
    const TailPlan tp = step_tail_plan(*d);
    if (tp.k > 0 && ws && ws_bytes >= tail_bytes(tp) && aligned16(ws)) {
      CombineParams c;
      std::memset(&c, 0, sizeof(c));
      c.out_o = O;
      c.out_bf16 = 1;
      c.out_lse = LSE_out;
      c.pre_o = O_pre;
      c.pre_lse = LSE_pre;
      return run_tail_split(p, tp, *d, ws, m.q, m.kb, m.vb, m.kb, m.vb, tm_out, c, s);
    }
    return from_cuda(launch_attn_tc2(p, m.q, m.kb, m.vb, m.kb, m.vb, tm_out, tm_out, (int)grid, s));
  }
  return from_cuda(launch_attn_tc(p, m.q, m.kb, m.vb, m.kb, m.vb, tm_pre, tm_out, (int)grid, s));
}

fb_status fb_block_step_append(const fb_desc* d, const void* Q, const void* Kb, const void* Vb,
                               const float* O_pre, const float* LSE_pre, void* O, float* LSE_out, void* Kc,
                               void* Vc, int32_t* lens_inout, void* ws, size_t ws_bytes, int32_t* dev_status,
                               fb_stream_t stream) {
  fb_status st = check_desc(d);
  if (st != FB_OK) return st;
  if (!Q || !Kb || !Vb || !O_pre || !LSE_pre || !O || !Kc || !Vc) return FB_ERR_INVALID_ARG;
  if (!d->prefix_lens && !lens_inout) return FB_ERR_INVALID_ARG;
  if (d->page_size > 0) {
    if (!pow2(d->page_size) || !d->block_table || d->max_pages <= 0 || d->num_pages <= 0)
      return FB_ERR_INVALID_ARG;
  } else if (d->kv_capacity <= 0) {
    return FB_ERR_INVALID_ARG;
  }
  if (!aligned16(Q) || !aligned16(Kb) || !aligned16(Vb) || !aligned16(O_pre) || !aligned16(O) ||
      !aligned16(Kc) || !aligned16(Vc) || (reinterpret_cast<uintptr_t>(LSE_pre) & 3u) ||
      (reinterpret_cast<uintptr_t>(LSE_out) & 3u))
    return FB_ERR_ALIGNMENT;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  const bool small = small_step_fits(*d, device_sms());
  if (small || rows_step_fits(*d)) {
    // one kernel: the step, and the unit's first CTA writes the block's rows
    const StepAppend app{lens_inout ? lens_inout : d->prefix_lens, Kc, Vc, dev_status};
    cudaError_t e = small ? launch_block_step_small(*d, Q, Kb, Vb, O_pre, LSE_pre, O, LSE_out, s, &app)
                          : launch_block_step_rows(*d, Q, Kb, Vb, O_pre, LSE_pre, O, LSE_out, s, &app);
    if (e != cudaSuccess || !lens_inout) return from_cuda(e);
    return from_cuda(launch_lens_advance(*d, lens_inout, s));
  }
  // other shapes: the step, then the append
  st = fb_block_step(d, Q, Kb, Vb, O_pre, LSE_pre, O, LSE_out, ws, ws_bytes, dev_status, stream);
  if (st != FB_OK) return st;
  return fb_kv_append(d, Kb, Vb, Kc, Vc, lens_inout, dev_status, stream);
}

fb_status fb_full_reference_gpu(const fb_desc* d, const void* Q, const void* Kc, const void* Vc,
                                const void* Kb, const void* Vb, void* O, float* LSE_out, void* ws,
                                size_t ws_bytes, int32_t* dev_status, fb_stream_t stream) {
  fb_status st = check_desc(d);
  if (st != FB_OK) return st;
  if ((st = check_cache(d)) != FB_OK) return st;
  if (!Q || !Kc || !Vc || !Kb || !Vb || !O) return FB_ERR_INVALID_ARG;
  if (!aligned16(Q) || !aligned16(Kc) || !aligned16(Vc) || !aligned16(Kb) || !aligned16(Vb) ||
      !aligned16(O) || (reinterpret_cast<uintptr_t>(LSE_out) & 3u))
    return FB_ERR_ALIGNMENT;
  fb_desc dense = *d;
  dense.topk = 0;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  AttnParams p = base_params(dense);
  p.src = key_source(dense, true, true, nullptr);
  p.dev_status = dev_status;
  if (d->dtype == FB_FP32) {
    p.epi = EPI_NORM;
    p.out_o = O;
    p.out_lse = LSE_out;
    return from_cuda(launch_attn_simt(p, static_cast<const float*>(Q), static_cast<const float*>(Kc),
                                      static_cast<const float*>(Vc), static_cast<const float*>(Kb),
                                      static_cast<const float*>(Vb), s));
  }
  const long long est = prefix_tiles_estimate(dense) + (d->block_len + TC_BN - 1) / TC_BN;
  const int ns = choose_splits(dense, est);
  const size_t need = split_bytes(dense, ns);
  if (need > 0 && (!ws || ws_bytes < need || !aligned16(ws))) return FB_ERR_WORKSPACE;
  Maps m;
  if (!q_map(&m.q, dense, Q) || !cache_map(&m.kp, dense, Kc) || !cache_map(&m.vp, dense, Vc) ||
      !block_map(&m.kb, dense, Kb) || !block_map(&m.vb, dense, Vb))
    return FB_ERR_LAUNCH;
  const long long units = cta_units(dense);
  const bool pairs = use_pairs(dense);
  if (pairs) p.kv_stream_once = (p.n_rt <= 2);
  if (ns == 1) {
    p.epi = EPI_NORM;
    p.out_o = O;
    p.out_lse = LSE_out;
    CUtensorMap tm_out;
    if (!q_map(&tm_out, dense, O)) return FB_ERR_LAUNCH;
    // the tail split (see tail_plan) where the workspace holds its slots
    const TailPlan tp = pairs ? tail_plan(dense, ns, est) : TailPlan{};
    if (tp.k > 0 && ws && ws_bytes >= tail_bytes(tp) && aligned16(ws)) {
      CombineParams c;
      std::memset(&c, 0, sizeof(c));
      c.out_o = O;
      c.out_bf16 = 1;
      c.out_lse = LSE_out;
      return run_tail_split(p, tp, dense, ws, m.q, m.kp, m.vp, m.kb, m.vb, tm_out, c, s);
    }
    if (pairs) return from_cuda(launch_attn_tc2(p, m.q, m.kp, m.vp, m.kb, m.vb, tm_out, tm_out, (int)units, s));
    return from_cuda(launch_attn_tc(p, m.q, m.kp, m.vp, m.kb, m.vb, m.q, tm_out, (int)units, s));
  }
  p.epi = EPI_PARTIAL;
  p.nsplit = ns;
  float* part_o = static_cast<float*>(ws);
  float* part_l = part_o + (size_t)ns * d->batch * d->block_len * d->num_q_heads * d->head_dim;
  p.out_o32 = part_o;
  p.out_lse = part_l;
  CUtensorMap tm_out;
  if (!pre_map(&tm_out, dense, part_o, d->batch * ns)) return FB_ERR_LAUNCH;
  cudaError_t e = pairs ? launch_attn_tc2(p, m.q, m.kp, m.vp, m.kb, m.vb, tm_out, tm_out, (int)(units * ns), s)
                        : launch_attn_tc(p, m.q, m.kp, m.vp, m.kb, m.vb, m.q, tm_out, (int)(units * ns), s);
  if (e != cudaSuccess) return from_cuda(e);
  CombineParams c;
  std::memset(&c, 0, sizeof(c));
  c.B = d->batch;
  c.Hq = d->num_q_heads;
  c.S = d->block_len;
  c.D = d->head_dim;
  c.nsplit = ns;
  c.part_o = part_o;
  c.part_lse = part_l;
  c.out_o = O;
  c.out_bf16 = 1;
  c.out_lse = LSE_out;
  return from_cuda(launch_combine(c, s));
}

fb_status fb_chunk_means(const fb_desc* d, const void* Kc, int32_t c0, int32_t c1, float* Kmean,
                         int32_t* dev_status, fb_stream_t stream) {
  fb_status st = check_desc(d);
  if (st != FB_OK) return st;
  if ((st = check_cache(d)) != FB_OK) return st;
  if (!Kc || !Kmean) return FB_ERR_INVALID_ARG;
  if (d->chunk_size <= 0) return FB_ERR_INVALID_ARG;
  const int64_t nch = (cache_rows(*d) + d->chunk_size - 1) / d->chunk_size;
  if (c0 < 0 || c1 < c0 || c1 > nch) return FB_ERR_INVALID_ARG;
  if (!aligned16(Kc) || !aligned16(Kmean)) return FB_ERR_ALIGNMENT;
  return from_cuda(launch_chunk_means(*d, Kc, c0, c1, 0, Kmean, dev_status,
                                      reinterpret_cast<cudaStream_t>(stream)));
}

fb_status fb_chunk_means_tail(const fb_desc* d, const void* Kc, int32_t rows, float* Kmean,
                              int32_t* dev_status, fb_stream_t stream) {
  fb_status st = check_desc(d);
  if (st != FB_OK) return st;
  if ((st = check_cache(d)) != FB_OK) return st;
  if (!Kc || !Kmean || rows <= 0) return FB_ERR_INVALID_ARG;
  if (d->chunk_size <= 0) return FB_ERR_INVALID_ARG;
  if (!aligned16(Kc) || !aligned16(Kmean)) return FB_ERR_ALIGNMENT;
  const int64_t rows_cap = std::min<int64_t>(rows, cache_rows(*d));
  return from_cuda(launch_chunk_means(*d, Kc, 0, 0, (int)std::max<int64_t>(rows_cap, 1), Kmean, dev_status,
                                      reinterpret_cast<cudaStream_t>(stream)));
}

fb_status fb_select_chunks(const fb_desc* d, const void* Q, const float* Kmean, int32_t* chunk_idx,
                           int32_t* dev_status, fb_stream_t stream) {
  fb_status st = check_desc(d);
  if (st != FB_OK) return st;
  if ((st = check_cache(d)) != FB_OK) return st;
  if (!Q || !Kmean || !chunk_idx) return FB_ERR_INVALID_ARG;
  if (d->chunk_size <= 0 || d->topk <= 0) return FB_ERR_INVALID_ARG;
  const int64_t nch = (cache_rows(*d) + d->chunk_size - 1) / d->chunk_size;
  if (nch > 16384) return FB_ERR_UNSUPPORTED;  // scores + flags stay within shared memory
  if (!aligned16(Q) || !aligned16(Kmean) || (reinterpret_cast<uintptr_t>(chunk_idx) & 3u))
    return FB_ERR_ALIGNMENT;
  return from_cuda(launch_select_chunks(*d, Q, Kmean, chunk_idx, dev_status,
                                        reinterpret_cast<cudaStream_t>(stream)));
}

fb_status fb_kv_append(const fb_desc* d, const void* Kb, const void* Vb, void* Kc, void* Vc,
                       int32_t* lens_inout, int32_t* dev_status, fb_stream_t stream) {
  fb_status st = check_desc(d);
  if (st != FB_OK) return st;
  if (!d->prefix_lens && !lens_inout) return FB_ERR_INVALID_ARG;
  if (d->page_size > 0) {
    if (!pow2(d->page_size) || !d->block_table || d->max_pages <= 0 || d->num_pages <= 0)
      return FB_ERR_INVALID_ARG;
  } else if (d->kv_capacity <= 0) {
    return FB_ERR_INVALID_ARG;
  }
  if (!Kb || !Vb || !Kc || !Vc) return FB_ERR_INVALID_ARG;
  if (!aligned16(Kb) || !aligned16(Vb) || !aligned16(Kc) || !aligned16(Vc)) return FB_ERR_ALIGNMENT;
  return from_cuda(launch_kv_append(*d, Kb, Vb, Kc, Vc, lens_inout, dev_status,
                                    reinterpret_cast<cudaStream_t>(stream)));
}

fb_status fb_complement_chunks(const fb_desc* d, const int32_t* chunk_idx, int32_t* comp_idx,
                               int32_t comp_cap, int32_t* dev_status, fb_stream_t stream) {
  fb_status st = check_desc(d);
  if (st != FB_OK) return st;
  if ((st = check_cache(d)) != FB_OK) return st;
  if (!chunk_idx || !comp_idx || d->chunk_size <= 0 || d->topk <= 0 || comp_cap <= 0) return FB_ERR_INVALID_ARG;
  const int64_t nch = (cache_rows(*d) + d->chunk_size - 1) / d->chunk_size;
  if (nch > 16384) return FB_ERR_UNSUPPORTED;
  if ((reinterpret_cast<uintptr_t>(chunk_idx) & 3u) || (reinterpret_cast<uintptr_t>(comp_idx) & 3u))
    return FB_ERR_ALIGNMENT;
  return from_cuda(launch_complement_chunks(*d, chunk_idx, comp_idx, comp_cap, dev_status,
                                            reinterpret_cast<cudaStream_t>(stream)));
}

fb_status fb_merge_partials(const fb_desc* d, const float* O_a, const float* LSE_a, const float* O_b,
                            const float* LSE_b, float* O_out, float* LSE_out, fb_stream_t stream) {
  fb_status st = check_desc(d);
  if (st != FB_OK) return st;
  if (!O_a || !LSE_a || !O_b || !LSE_b || !O_out || !LSE_out) return FB_ERR_INVALID_ARG;
  if (d->head_dim % 4) return FB_ERR_UNSUPPORTED;
  if (!aligned16(O_a) || !aligned16(O_b) || !aligned16(O_out) || (reinterpret_cast<uintptr_t>(LSE_a) & 3u) ||
      (reinterpret_cast<uintptr_t>(LSE_b) & 3u) || (reinterpret_cast<uintptr_t>(LSE_out) & 3u))
    return FB_ERR_ALIGNMENT;
  return from_cuda(launch_merge_partials(*d, O_a, LSE_a, O_b, LSE_b, O_out, LSE_out,
                                         reinterpret_cast<cudaStream_t>(stream)));
}

const char* fb_status_string(fb_status s) {
  switch (s) {
    case FB_OK: return "FB_OK";
    case FB_ERR_INVALID_ARG: return "FB_ERR_INVALID_ARG";
    case FB_ERR_UNSUPPORTED: return "FB_ERR_UNSUPPORTED";
    case FB_ERR_ALIGNMENT: return "FB_ERR_ALIGNMENT";
    case FB_ERR_WORKSPACE: return "FB_ERR_WORKSPACE";
    case FB_ERR_LAUNCH: return "FB_ERR_LAUNCH";
    case FB_ERR_DEVICE_TIMEOUT: return "FB_ERR_DEVICE_TIMEOUT";
    case FB_ERR_BOUNDS: return "FB_ERR_BOUNDS";
  }
  return "FB_ERR_UNKNOWN";
}

uint64_t fb_launch_count(void) { return g_launches.load(std::memory_order_relaxed); }

int32_t fb_abi_version(void) { return FB_ABI_VERSION; }

#ifdef FB_TEST_HOOKS
// Test builds only (libflashblock_testhooks.so): 1 = the attention kernels'
// K producers leave the load of their second key tile out, so the wait for it
// runs out (these builds bound every wait by a short FB_WAIT_LIMIT_NS).
void fb_test_set_skip_k1(int32_t on) { g_test_skip_k1.store(on ? 1 : 0, std::memory_order_relaxed); }
#endif

}  // extern "C"
