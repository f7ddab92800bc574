// fb_attn_common.cuh -- device helpers shared by the tensor-core attention
// kernels (one query tile per CTA in fb_attn_tc.cu, two in fb_attn_tc2.cu):
// tile geometry, the bounded mbarrier wait, the key tiles of a work unit
// (dense or sparse prefix, in-block keys) and their TMA loads.
#pragma once

#include <cuda.h>
#include <stdint.h>

#include "fb_internal.h"
#include "fb_ptx.cuh"

namespace fb {

constexpr int BM = TC_BM, BN = TC_BN, HD = TC_D;
static_assert(BM == BN && BN == HD, "square 128 tiles");
constexpr uint32_t Q_BYTES = BM * HD * 2;       // 32 KB: one query tile
constexpr uint32_t SLOT_BYTES = BN * HD * 2;    // 32 KB: one K or one V tile
constexpr uint32_t HALF_BYTES = BN * 128;       // one 64-column half of a tile
constexpr float RESCALE_LOG2 = 8.0f;   // rescale O only when the row max grows by > 2^8
#ifndef FB_WAIT_LIMIT_NS
#define FB_WAIT_LIMIT_NS 1000000000ull
#endif
constexpr uint64_t WAIT_LIMIT_NS = FB_WAIT_LIMIT_NS;  // bound of every pipeline wait
constexpr float LN2 = 0.6931471805599453f;

// Waits for the phase of `bar` with the given parity, for at most
// WAIT_LIMIT_NS.  On expiry it sets the CTA's abort flag, records
// FB_ERR_DEVICE_TIMEOUT and returns false; with honour_abort it also gives up
// as soon as another thread of the CTA has set the flag.
__device__ __forceinline__ bool bounded_wait(uint64_t* bar, uint32_t parity, volatile int* abort_flag,
                                             int32_t* status, bool honour_abort = true) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = global_timer_ns();
  for (;;) {
    // each try sleeps until the phase completes or 1 ms passes
    if (mbar_try_wait(bar, parity)) return true;
    if (honour_abort && *abort_flag) return false;
    if (global_timer_ns() - t0 > WAIT_LIMIT_NS) {
      *abort_flag = 1;
      report(status, FB_ERR_DEVICE_TIMEOUT);
      return false;
    }
  }
}

struct UnitTiles {
  int n0;  // prefix tiles
  int n1;  // block tiles
  int L;   // valid prefix rows
};

// Number of key tiles of one (b, kv head) work unit.  A sparse chunk list must
// be ascending and inside the valid prefix; the first entry that is not ends
// the list (and is reported).
__device__ inline UnitTiles unit_tiles(const AttnParams& p, int b, int kvh, bool rep) {
  const KeySource& s = p.src;
  UnitTiles u{0, 0, 0};
  if (s.has_prefix) {
    int L = s.prefix_lens[b];
    if (L < 0 || L > s.cap) {
      if (rep) report(p.dev_status, FB_ERR_BOUNDS);
      L = max(0, min(L, s.cap));
    }
    u.L = L;
    if (s.chunk_idx) {
      // 32 list entries per step, one per lane (the calling warp is
      // converged): the list ends at its first entry that is -1, not above
      // its predecessor or past the valid prefix (the last two are reported)
      const int32_t* idx = s.chunk_idx + ((size_t)b * p.Hkv + kvh) * s.topk;
      const int nch = (L + s.chunk_size - 1) / s.chunk_size;
      const int lane = threadIdx.x & 31;
      int n = 0, prev = -1;
      for (int i0 = 0; i0 < s.topk; i0 += 32) {
        const int i = i0 + lane;
        const int c = i < s.topk ? idx[i] : -1;
        int cp = __shfl_up_sync(0xffffffffu, c, 1);
        if (lane == 0) cp = prev;
        const bool bad = c >= 0 && (c <= cp || c >= nch);
        // (every lane takes part in both ballots)
        const unsigned stops = __ballot_sync(0xffffffffu, c < 0 || bad);
        const unsigned bads = __ballot_sync(0xffffffffu, bad);
        const int first = stops ? __ffs(stops) - 1 : 32;  // entries below it are valid
        if (rep && first < 32 && ((bads >> first) & 1u)) report(p.dev_status, FB_ERR_BOUNDS);
        int tiles = 0;
        if (lane < first) {
          const int lo = c * s.chunk_size;
          tiles = (min(lo + s.chunk_size, L) - lo + BN - 1) / BN;
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) tiles += __shfl_xor_sync(0xffffffffu, tiles, o);
        n += tiles;
        if (stops) break;
        prev = __shfl_sync(0xffffffffu, c, 31);
      }
      u.n0 = n;
    } else {
      u.n0 = (L + BN - 1) / BN;
    }
  }
  if (s.has_block) u.n1 = (p.S + BN - 1) / BN;
  return u;
}

struct Tile {
  int seg;     // 0 prefix, 1 block
  int row;     // logical row of the first key (cache position or block position)
  int nvalid;  // keys of this tile that take part (>= 1)
};

// `clist`: the unit's sparse chunk list (global memory or a shared-memory
// copy), or null for a dense prefix.
__device__ __forceinline__ Tile tile_at(const AttnParams& p, const UnitTiles& u, const int32_t* clist, int j) {
  Tile t;
  const KeySource& s = p.src;
  if (j < u.n0) {
    t.seg = 0;
    if (clist) {
      const int tpc = s.chunk_size / BN;
      const int slot = j / tpc;
      const int c = clist[slot];
      t.row = c * s.chunk_size + (j - slot * tpc) * BN;
    } else {
      t.row = j * BN;
    }
    t.nvalid = min(BN, u.L - t.row);
  } else {
    t.seg = 1;
    t.row = (j - u.n0) * BN;
    t.nvalid = min(BN, p.S - t.row);
  }
  return t;
}

// Loads one K or V tile (both 64-dim halves) of the given tile into `dst`.
__device__ __forceinline__ void load_kv_tile(uint8_t* dst, const CUtensorMap* prefix_map,
                                             const CUtensorMap* block_map, uint64_t* bar,
                                             const AttnParams& p, const UnitTiles& u,
                                             const Tile& t, int b, int kvh, uint64_t policy) {
  const KeySource& s = p.src;
  if (t.seg == 1) {
#pragma unroll
    for (int h = 0; h < 2; ++h) tma_load_4d(dst + h * HALF_BYTES, block_map, bar, h * 64, kvh, t.row, b);
    return;
  }
  if (!s.paged) {
#pragma unroll
    for (int h = 0; h < 2; ++h)
      tma_load_4d_hint(dst + h * HALF_BYTES, prefix_map, bar, h * 64, kvh, t.row, b, policy);
    return;
  }
  const int page_size = 1 << s.page_shift;
  const int box = page_size < BN ? page_size : BN;
  for (int sub = 0; sub < BN / box; ++sub) {
    const int r = t.row + sub * box;
    const int pi = r >> s.page_shift;
    int pg = (pi < s.max_pages) ? s.block_table[(size_t)b * s.max_pages + pi] : -1;
    if (pg < 0 || pg >= s.num_pages) {
      // rows past the prefix may sit on unmapped pages: read page 0 instead
      // (those keys are masked); inside the prefix it is an error.
      if (r < u.L) report(p.dev_status, FB_ERR_BOUNDS);
      pg = 0;
    }
    const int prow = r & (page_size - 1);
#pragma unroll
    for (int h = 0; h < 2; ++h)
      tma_load_4d_hint(dst + h * HALF_BYTES + sub * box * 128, prefix_map, bar, h * 64, kvh, prow, pg,
                       policy);
  }
}

}  // namespace fb
