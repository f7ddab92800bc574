// fb_attn_tc.cu -- bf16 attention partials on the sm_100a tensor cores.
//
// One CTA computes one (batch b, kv head, 128-row query tile, key-range split)
// work item of softmax attention, the partial (A, L = log Z) of the Core
// Mechanism of "FlashBlock: Attention Caching for Efficient Long-Context
// Block Diffusion" (Technical Summary §2).  The same kernel serves the three
// uses of the method:
//   * the block-external partial over the finalized prefix (EPI_PARTIAL),
//   * the block-internal partial fused with the merge equation (EPI_MERGE),
//   * the uncached full attention over [prefix ; block] (EPI_NORM, or
//     EPI_PARTIAL splits combined by combine_kernel).
//
// Query rows are GQA-packed: the 128 rows of a tile are (token, group head)
// pairs of one kv head, so each K/V tile that TMA brings in is used by all G
// query heads of the group.
//
// Warp roles (192 threads):
//   warps 0-3  softmax: thread r owns query row r (TMEM lane r); online softmax
//              in fp32 with base-2 exponentials, P to shared memory as bf16,
//              lazy rescaling of the TMEM accumulator, epilogue;
//   warp 4     TMA producer: Q once, then K and V tiles into a 2-stage ring;
//   warp 5     TMEM owner and MMA issuer: S = Q K^T and O += P V with
//              tcgen05.mma (M = 128, N = 128, K = 16 per instruction).
//
// TMEM: S at columns [0, 128), O at [128, 256).
// Shared memory (1024-byte aligned, 128-byte swizzle everywhere):
//   Q [2 halves of 64 dims][128 rows][128 B]                 32 KB
//   per stage: K [2][128 keys][128 B], V [2][128 keys][128 B]  64 KB
//   P [2 halves of 64 keys][128 rows][128 B]                 32 KB
//
// Every mbarrier wait is bounded in time; on expiry the CTA records
// FB_ERR_DEVICE_TIMEOUT, drains its own copies and MMAs, frees TMEM and exits.
#include <cuda_bf16.h>
#include <math_constants.h>

#include "fb_internal.h"
#include "fb_ptx.cuh"

namespace fb {

namespace {

constexpr int BM = TC_BM, BN = TC_BN, HD = TC_D, NST = TC_STAGES;
constexpr uint32_t Q_BYTES = BM * HD * 2;       // 32 KB
constexpr uint32_t KV_TILE_BYTES = BN * HD * 2; // 32 KB (K or V)
constexpr uint32_t HALF_BYTES = BN * 128;       // one 64-column half of a tile
constexpr uint32_t P_BYTES = BM * BN * 2;       // 32 KB
constexpr uint32_t OFF_Q = 0;
constexpr uint32_t OFF_KV = OFF_Q + Q_BYTES;
constexpr uint32_t OFF_P = OFF_KV + NST * 2 * KV_TILE_BYTES;
constexpr uint32_t OFF_BAR = OFF_P + P_BYTES;
constexpr int NUM_BARS = 1 + 3 * NST + 5;
constexpr uint32_t SMEM_BYTES = OFF_BAR + 256 + 1024;  // + alignment slack
constexpr uint32_t TMEM_COLS = 256;
constexpr uint32_t TMEM_S = 0, TMEM_O = 128;
constexpr float RESCALE_LOG2 = 8.0f;   // rescale O only when the row max grows by > 2^8
constexpr uint64_t WAIT_LIMIT_NS = 1000000000ull;
constexpr float LN2 = 0.6931471805599453f;

static_assert(NUM_BARS * 8 + 8 <= 256, "barrier area");
static_assert(SMEM_BYTES <= 232448, "shared memory");

struct Shared {
  uint64_t* q_full;
  uint64_t* k_full;
  uint64_t* v_full;
  uint64_t* empty;
  uint64_t* s_full;
  uint64_t* s_free;
  uint64_t* p_full;
  uint64_t* o_done;
  uint64_t* drain;
  uint32_t* tmem_slot;
  volatile int* abort_flag;
};

__device__ __forceinline__ bool wait_bar(uint64_t* bar, uint32_t parity, const Shared& sh,
                                         int32_t* status, bool honour_abort = true) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = global_timer_ns();
  for (uint32_t n = 1;; ++n) {
    if (mbar_try_wait(bar, parity)) return true;
    if ((n & 63u) == 0) {
      if (honour_abort && *sh.abort_flag) return false;
      if (global_timer_ns() - t0 > WAIT_LIMIT_NS) {
        *sh.abort_flag = 1;
        report(status, FB_ERR_DEVICE_TIMEOUT);
        return false;
      }
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
__device__ UnitTiles unit_tiles(const AttnParams& p, int b, int kvh, bool rep) {
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
        const int lo = c * s.chunk_size;
        const int hi = min(lo + s.chunk_size, L);
        n += (hi - lo + BN - 1) / BN;
        prev = c;
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

__device__ __forceinline__ Tile tile_at(const AttnParams& p, const UnitTiles& u, int b, int kvh,
                                        int j) {
  Tile t;
  const KeySource& s = p.src;
  if (j < u.n0) {
    t.seg = 0;
    if (s.chunk_idx) {
      const int tpc = s.chunk_size / BN;
      const int slot = j / tpc;
      const int c = s.chunk_idx[((size_t)b * p.Hkv + kvh) * s.topk + slot];
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
                                             const Tile& t, int b, int kvh) {
  const KeySource& s = p.src;
  if (t.seg == 1) {
#pragma unroll
    for (int h = 0; h < 2; ++h) tma_load_4d(dst + h * HALF_BYTES, block_map, bar, h * 64, kvh, t.row, b);
    return;
  }
  if (!s.paged) {
#pragma unroll
    for (int h = 0; h < 2; ++h) tma_load_4d(dst + h * HALF_BYTES, prefix_map, bar, h * 64, kvh, t.row, b);
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
      tma_load_4d(dst + h * HALF_BYTES + sub * box * 128, prefix_map, bar, h * 64, kvh, prow, pg);
  }
}

template <int EPI>
__global__ void __launch_bounds__(TC_THREADS, 1)
    attn_tc_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmKp,
                   const __grid_constant__ CUtensorMap tmVp, const __grid_constant__ CUtensorMap tmKb,
                   const __grid_constant__ CUtensorMap tmVb, const AttnParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  uint8_t* sQ = smem + OFF_Q;
  uint8_t* sKV = smem + OFF_KV;
  uint8_t* sP = smem + OFF_P;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + OFF_BAR);
  Shared sh;
  sh.q_full = bars;
  sh.k_full = bars + 1;
  sh.v_full = sh.k_full + NST;
  sh.empty = sh.v_full + NST;
  sh.s_full = sh.empty + NST;
  sh.s_free = sh.s_full + 1;
  sh.p_full = sh.s_free + 1;
  sh.o_done = sh.p_full + 1;
  sh.drain = sh.o_done + 1;
  sh.tmem_slot = reinterpret_cast<uint32_t*>(sh.drain + 1);
  sh.abort_flag = reinterpret_cast<volatile int*>(sh.tmem_slot + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  int bid = blockIdx.x;
  const int split = bid % p.nsplit;
  bid /= p.nsplit;
  const int rt = bid % p.n_rt;
  bid /= p.n_rt;
  const int kvh = bid % p.Hkv;
  const int b = bid / p.Hkv;

  if (threadIdx.x == 0) {
    mbar_init(sh.q_full, 1);
    for (int i = 0; i < NST; ++i) {
      mbar_init(&sh.k_full[i], 1);
      mbar_init(&sh.v_full[i], 1);
      mbar_init(&sh.empty[i], 1);
    }
    mbar_init(sh.s_full, 1);
    mbar_init(sh.s_free, 128);
    mbar_init(sh.p_full, 4);
    mbar_init(sh.o_done, 1);
    mbar_init(sh.drain, 1);
    *sh.abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 5) {
    tmem_alloc(sh.tmem_slot, TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before_sync();
  __syncthreads();
  tc_fence_after_sync();
  const uint32_t tmem = *sh.tmem_slot;

  const UnitTiles u = unit_tiles(p, b, kvh, threadIdx.x == 0);
  const int ntot = u.n0 + u.n1;
  const int j0 = (int)(((long long)split * ntot) / p.nsplit);
  const int j1 = (int)(((long long)(split + 1) * ntot) / p.nsplit);
  const int nt = j1 - j0;
  int32_t* status = p.dev_status;

  if (warp == 4) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      tma_prefetch_map(&tmQ);
      tma_prefetch_map(&tmKp);
      tma_prefetch_map(&tmVp);
      mbar_arrive_expect_tx(sh.q_full, Q_BYTES);
      const int t0 = rt * (BM / p.G);
      tma_load_4d(sQ, &tmQ, sh.q_full, 0, kvh * p.G, t0, b);
      tma_load_4d(sQ + BM * 128, &tmQ, sh.q_full, 64, kvh * p.G, t0, b);
      int issued = 0;
      for (int jj = 0; jj < nt; ++jj) {
        const int st = jj % NST;
        const uint32_t use = jj / NST;
        if (!wait_bar(&sh.empty[st], (use & 1) ^ 1, sh, status)) break;
        const Tile t = tile_at(p, u, b, kvh, j0 + jj);
        uint8_t* dK = sKV + st * 2 * KV_TILE_BYTES;
        uint8_t* dV = dK + KV_TILE_BYTES;
        mbar_arrive_expect_tx(&sh.k_full[st], KV_TILE_BYTES);
        load_kv_tile(dK, &tmKp, &tmKb, &sh.k_full[st], p, u, t, b, kvh);
        mbar_arrive_expect_tx(&sh.v_full[st], KV_TILE_BYTES);
        load_kv_tile(dV, &tmVp, &tmVb, &sh.v_full[st], p, u, t, b, kvh);
        issued = jj + 1;
      }
      // After an abort, let the copies in flight land before the CTA exits.
      if (*sh.abort_flag) {
        wait_bar(sh.q_full, 0, sh, nullptr, false);
        for (int jj = max(0, issued - NST); jj < issued; ++jj) {
          const int st = jj % NST;
          const uint32_t use = jj / NST;
          wait_bar(&sh.k_full[st], use & 1, sh, nullptr, false);
          wait_bar(&sh.v_full[st], use & 1, sh, nullptr, false);
        }
      }
    }
  } else if (warp == 5) {
    // --------------------------------------------------------------- MMA issuer
    constexpr uint32_t IDESC_QK = idesc_bf16_f32(BM, BN, false, false);
    constexpr uint32_t IDESC_PV = idesc_bf16_f32(BM, HD, false, true);
    const uint32_t tS = tmem + TMEM_S;
    const uint32_t tO = tmem + TMEM_O;
    const uint32_t aQ = smem_u32(sQ);
    const uint32_t aP = smem_u32(sP);
    auto issue_qk = [&](int st) {
      const uint32_t aK = smem_u32(sKV + st * 2 * KV_TILE_BYTES);
#pragma unroll
      for (int kk = 0; kk < HD / 16; ++kk) {
        const uint32_t off = (kk >> 2) * HALF_BYTES + (kk & 3) * 32;
        umma_bf16_ss(tS, sw128_desc(aQ + off, 16, 1024), sw128_desc(aK + off, 16, 1024), IDESC_QK,
                     kk > 0);
      }
    };
    auto issue_pv = [&](int st, bool acc) {
      const uint32_t aV = smem_u32(sKV + st * 2 * KV_TILE_BYTES + KV_TILE_BYTES);
#pragma unroll
      for (int kk = 0; kk < BN / 16; ++kk) {
        const uint32_t offp = (kk >> 2) * (BM * 128) + (kk & 3) * 32;
        umma_bf16_ss(tO, sw128_desc(aP + offp, 16, 1024),
                     sw128_desc(aV + kk * 16 * 128, HALF_BYTES, 1024), IDESC_PV,
                     (acc || kk > 0) ? 1u : 0u);
      }
    };
    bool ok = wait_bar(sh.q_full, 0, sh, status);
    if (ok && nt > 0) {
      ok = wait_bar(&sh.k_full[0], 0, sh, status);
      if (ok) {
        tc_fence_after_sync();
        if (lane == 0) {
          issue_qk(0);
          tc_commit(sh.s_full);
        }
        __syncwarp();
      }
      for (int jj = 0; ok && jj < nt; ++jj) {
        const int st = jj % NST;
        const uint32_t use = jj / NST;
        if (jj + 1 < nt) {
          const int st1 = (jj + 1) % NST;
          const uint32_t use1 = (jj + 1) / NST;
          if (!(ok = wait_bar(&sh.k_full[st1], use1 & 1, sh, status))) break;
          if (!(ok = wait_bar(sh.s_free, jj & 1, sh, status))) break;
          tc_fence_after_sync();
          if (lane == 0) {
            issue_qk(st1);
            tc_commit(sh.s_full);
          }
          __syncwarp();
        }
        if (!(ok = wait_bar(&sh.v_full[st], use & 1, sh, status))) break;
        const Tile t = tile_at(p, u, b, kvh, j0 + jj);
        if (t.seg == 0 && t.nvalid < BN) {
          // Cache rows past the prefix may hold anything (even NaN); P is 0
          // there but 0 * NaN is not, so clear those V rows.
          uint8_t* dV = sKV + st * 2 * KV_TILE_BYTES + KV_TILE_BYTES;
          const int nrow = BN - t.nvalid;
          for (int i = lane; i < nrow * 16; i += 32) {
            const int r = t.nvalid + (i >> 4);
            const int h = (i >> 3) & 1;
            const int c = i & 7;
            *reinterpret_cast<uint4*>(dV + h * HALF_BYTES + r * 128 + c * 16) = make_uint4(0, 0, 0, 0);
          }
          fence_proxy_async_smem();
        }
        __syncwarp();
        if (!(ok = wait_bar(sh.p_full, jj & 1, sh, status))) break;
        tc_fence_after_sync();
        if (lane == 0) {
          issue_pv(st, jj > 0);
          tc_commit(sh.o_done);
          tc_commit(&sh.empty[st]);
        }
        __syncwarp();
      }
    }
    // Drain every MMA this thread issued before TMEM can be released.
    if (lane == 0) tc_commit(sh.drain);
    __syncwarp();
    wait_bar(sh.drain, 0, sh, nullptr, false);
  } else {
    // ------------------------------------------------------ softmax + epilogue
    const int r = warp * 32 + lane;  // query row of this thread = TMEM lane
    const uint32_t lane_off = (uint32_t)(warp * 32) << 16;
    const uint32_t tS = tmem + TMEM_S + lane_off;
    const uint32_t tO = tmem + TMEM_O + lane_off;
    const uint32_t p_row = smem_u32(sP) + r * 128;
    const float c2 = p.scale_log2;
    float m_run = -CUDART_INF_F;
    float l_run = 0.f;
    bool ok = true;
    for (int jj = 0; jj < nt; ++jj) {
      if (!(ok = wait_bar(sh.s_full, jj & 1, sh, status))) break;
      tc_fence_after_sync();
      uint32_t sv[BN];
#pragma unroll
      for (int c = 0; c < BN / 32; ++c)
        tmem_ld_32x32(tS + c * 32, *reinterpret_cast<uint32_t(*)[32]>(&sv[c * 32]));
      tmem_ld_wait();
      tc_fence_before_sync();
      mbar_arrive(sh.s_free);

      const Tile t = tile_at(p, u, b, kvh, j0 + jj);
      float s[BN];
      float mx = -CUDART_INF_F;
#pragma unroll
      for (int c = 0; c < BN; ++c) {
        s[c] = (c < t.nvalid) ? __uint_as_float(sv[c]) : -CUDART_INF_F;
        mx = fmaxf(mx, s[c]);
      }
      const float mt = mx * c2;
      const bool need = mt > m_run + RESCALE_LOG2;
      const float m_new = need ? mt : m_run;
      const float alpha = ex2_approx(m_run - m_new);  // 0 when m_run = -inf
      const float m_use = (m_new == -CUDART_INF_F) ? 0.f : m_new;
      float l0 = 0.f, l1 = 0.f, l2 = 0.f, l3 = 0.f;
#pragma unroll
      for (int c = 0; c < BN; c += 4) {
        s[c] = ex2_approx(fmaf(s[c], c2, -m_use));
        s[c + 1] = ex2_approx(fmaf(s[c + 1], c2, -m_use));
        s[c + 2] = ex2_approx(fmaf(s[c + 2], c2, -m_use));
        s[c + 3] = ex2_approx(fmaf(s[c + 3], c2, -m_use));
        l0 += s[c];
        l1 += s[c + 1];
        l2 += s[c + 2];
        l3 += s[c + 3];
      }
      l_run = l_run * alpha + ((l0 + l1) + (l2 + l3));
      m_run = m_new;

      if (jj > 0) {
        // PV of the previous tile must be done: P is single-buffered and O
        // may be rescaled below.
        if (!(ok = wait_bar(sh.o_done, (jj - 1) & 1, sh, status))) break;
        tc_fence_after_sync();
        if (__any_sync(0xffffffffu, need)) {
#pragma unroll
          for (int c = 0; c < HD / 32; ++c) {
            uint32_t ov[32];
            tmem_ld_32x32(tO + c * 32, ov);
            tmem_ld_wait();
#pragma unroll
            for (int i = 0; i < 32; ++i) ov[i] = __float_as_uint(__uint_as_float(ov[i]) * alpha);
            tmem_st_32x32(tO + c * 32, ov);
          }
          tmem_st_wait();
        }
      }
      // P (bf16) into the K-major, 128-byte-swizzled A-operand layout.
#pragma unroll
      for (int c = 0; c < BN; c += 8) {
        const int half = c >> 6;
        const int chunk = (c & 63) >> 3;
        const uint32_t addr = p_row + half * (BM * 128) + ((chunk ^ (r & 7)) << 4);
        st_shared_v4(addr, pack_bf16x2(s[c], s[c + 1]), pack_bf16x2(s[c + 2], s[c + 3]),
                     pack_bf16x2(s[c + 4], s[c + 5]), pack_bf16x2(s[c + 6], s[c + 7]));
      }
      fence_proxy_async_smem();
      tc_fence_before_sync();
      __syncwarp();
      if (lane == 0) mbar_arrive(sh.p_full);
    }
    if (ok && nt > 0) {
      ok = wait_bar(sh.o_done, (nt - 1) & 1, sh, status);
      tc_fence_after_sync();
    }
    // ---------------------------------------------------------------- epilogue
    const int pr = rt * BM + r;
    const int tok = pr / p.G;
    const int h = kvh * p.G + (pr - tok * p.G);
    const bool row_ok = ok && tok < p.S;
    const bool empty = (nt == 0) || !(l_run > 0.f);
    const float inv_l = empty ? 0.f : 1.f / l_run;
    const float lse2 = empty ? -CUDART_INF_F : m_run + log2f(l_run);  // log2 of Z
    if (EPI == EPI_PARTIAL) {
      const size_t orow = (((size_t)split * p.B + b) * p.S + tok) * p.Hq + h;
      float* dst = p.out_o32 + orow * HD;
#pragma unroll
      for (int c = 0; c < HD / 32; ++c) {
        uint32_t ov[32];
        if (nt > 0) {
          tmem_ld_32x32(tO + c * 32, ov);
          tmem_ld_wait();
        } else {
#pragma unroll
          for (int i = 0; i < 32; ++i) ov[i] = 0u;
        }
        if (row_ok) {
#pragma unroll
          for (int i = 0; i < 32; i += 4) {
            float4 v = make_float4(__uint_as_float(ov[i]) * inv_l, __uint_as_float(ov[i + 1]) * inv_l,
                                   __uint_as_float(ov[i + 2]) * inv_l, __uint_as_float(ov[i + 3]) * inv_l);
            *reinterpret_cast<float4*>(dst + c * 32 + i) = v;
          }
        }
      }
      if (row_ok)
        p.out_lse[(((size_t)split * p.B + b) * p.Hq + h) * p.S + tok] = lse2 * LN2;
    } else {
      const size_t orow = ((size_t)b * p.S + tok) * p.Hq + h;
      float wp = 0.f, wo = inv_l, inv_den = 1.f, lse_out2 = lse2;
      if (EPI == EPI_MERGE) {
        // merge equation in base 2: weights e^{L - m} become 2^{L2 - M}
        const float lp2 = row_ok ? p.pre_lse[((size_t)b * p.Hq + h) * p.S + tok] * 1.4426950408889634f
                                 : -CUDART_INF_F;
        const float M = fmaxf(lp2, lse2);
        const float Ms = (M == -CUDART_INF_F) ? 0.f : M;
        wp = ex2_approx(lp2 - Ms);
        const float wi = ex2_approx(lse2 - Ms);
        const float den = wp + wi;
        inv_den = den > 0.f ? 1.f / den : 0.f;
        wo = empty ? 0.f : ex2_approx(m_run - Ms);  // = wi / l_run
        lse_out2 = den > 0.f ? Ms + log2f(den) : -CUDART_INF_F;
      }
      __nv_bfloat16* dst = reinterpret_cast<__nv_bfloat16*>(p.out_o) + orow * HD;
      const float* pre = (EPI == EPI_MERGE) ? p.pre_o + orow * HD : nullptr;
#pragma unroll
      for (int c = 0; c < HD / 32; ++c) {
        uint32_t ov[32];
        tmem_ld_32x32(tO + c * 32, ov);
        tmem_ld_wait();
        if (row_ok) {
          float o[32];
#pragma unroll
          for (int i = 0; i < 32; ++i) o[i] = __uint_as_float(ov[i]) * wo;
          if (EPI == EPI_MERGE) {
#pragma unroll
            for (int i = 0; i < 32; i += 4) {
              const float4 q = *reinterpret_cast<const float4*>(pre + c * 32 + i);
              o[i] = (o[i] + wp * q.x) * inv_den;
              o[i + 1] = (o[i + 1] + wp * q.y) * inv_den;
              o[i + 2] = (o[i + 2] + wp * q.z) * inv_den;
              o[i + 3] = (o[i + 3] + wp * q.w) * inv_den;
            }
          }
#pragma unroll
          for (int i = 0; i < 32; i += 8) {
            uint4 v = make_uint4(pack_bf16x2(o[i], o[i + 1]), pack_bf16x2(o[i + 2], o[i + 3]),
                                 pack_bf16x2(o[i + 4], o[i + 5]), pack_bf16x2(o[i + 6], o[i + 7]));
            *reinterpret_cast<uint4*>(dst + c * 32 + i) = v;
          }
        }
      }
      if (row_ok && p.out_lse) p.out_lse[((size_t)b * p.Hq + h) * p.S + tok] = lse_out2 * LN2;
    }
  }

  tc_fence_before_sync();
  __syncthreads();
  if (warp == 5) {
    tc_fence_after_sync();
    tmem_dealloc(tmem, TMEM_COLS);
  }
}

// Log-space merge of the split-key partials of one query row (the merge
// equation applied across splits, in a fixed order).  One warp per row.
__global__ void combine_kernel(const CombineParams c) {
  const int warps = blockDim.x >> 5;
  const long long row = (long long)blockIdx.x * warps + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  const long long nrows = (long long)c.B * c.S * c.Hq;
  if (row >= nrows) return;
  const int h = (int)(row % c.Hq);
  const long long bt = row / c.Hq;
  const int t = (int)(bt % c.S);
  const int b = (int)(bt / c.S);
  const size_t split_stride_o = (size_t)nrows * c.D;
  const size_t split_stride_l = (size_t)c.B * c.Hq * c.S;
  const size_t lrow = ((size_t)b * c.Hq + h) * c.S + t;
  float M = -CUDART_INF_F;
  for (int s = 0; s < c.nsplit; ++s) M = fmaxf(M, c.part_lse[s * split_stride_l + lrow]);
  const bool empty = (M == -CUDART_INF_F);
  float den = 0.f;
  for (int d0 = lane * 4; d0 < c.D; d0 += 128) {
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    den = 0.f;
    if (!empty) {
      for (int s = 0; s < c.nsplit; ++s) {
        const float ls = c.part_lse[s * split_stride_l + lrow];
        const float w = (ls == -CUDART_INF_F) ? 0.f : expf(ls - M);
        den += w;
        const float4 v = *reinterpret_cast<const float4*>(c.part_o + s * split_stride_o + row * c.D + d0);
        acc.x += w * v.x;
        acc.y += w * v.y;
        acc.z += w * v.z;
        acc.w += w * v.w;
      }
      const float inv = 1.f / den;
      acc.x *= inv;
      acc.y *= inv;
      acc.z *= inv;
      acc.w *= inv;
    }
    if (c.out_o32) {
      *reinterpret_cast<float4*>(c.out_o32 + row * c.D + d0) = acc;
    } else if (c.out_bf16) {
      uint2 v = make_uint2(pack_bf16x2(acc.x, acc.y), pack_bf16x2(acc.z, acc.w));
      *reinterpret_cast<uint2*>(reinterpret_cast<__nv_bfloat16*>(c.out_o) + row * c.D + d0) = v;
    } else {
      *reinterpret_cast<float4*>(reinterpret_cast<float*>(c.out_o) + row * c.D + d0) = acc;
    }
  }
  if (lane == 0 && c.out_lse) {
    if (empty) {
      c.out_lse[lrow] = -CUDART_INF_F;
    } else {
      float dd = 0.f;
      for (int s = 0; s < c.nsplit; ++s) {
        const float ls = c.part_lse[s * split_stride_l + lrow];
        dd += (ls == -CUDART_INF_F) ? 0.f : expf(ls - M);
      }
      c.out_lse[lrow] = M + logf(dd);
    }
  }
}

}  // namespace

size_t tc_smem_bytes() { return SMEM_BYTES; }

cudaError_t launch_attn_tc(const AttnParams& p, const CUtensorMap& tmQ, const CUtensorMap& tmKp,
                           const CUtensorMap& tmVp, const CUtensorMap& tmKb,
                           const CUtensorMap& tmVb, int grid, cudaStream_t stream) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  static bool configured[64][3] = {};
  void (*kern)(CUtensorMap, CUtensorMap, CUtensorMap, CUtensorMap, CUtensorMap, AttnParams);
  switch (p.epi) {
    case EPI_PARTIAL: kern = attn_tc_kernel<EPI_PARTIAL>; break;
    case EPI_MERGE: kern = attn_tc_kernel<EPI_MERGE>; break;
    default: kern = attn_tc_kernel<EPI_NORM>; break;
  }
  if (dev < 64 && !configured[dev][p.epi]) {
    e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)SMEM_BYTES);
    if (e != cudaSuccess) return e;
    configured[dev][p.epi] = true;
  }
  kern<<<grid, TC_THREADS, SMEM_BYTES, stream>>>(tmQ, tmKp, tmVp, tmKb, tmVb, p);
  note_launch();
  return cudaGetLastError();
}

cudaError_t launch_combine(const CombineParams& c, cudaStream_t stream) {
  const long long rows = (long long)c.B * c.S * c.Hq;
  const int warps = 8;
  const long long grid = (rows + warps - 1) / warps;
  combine_kernel<<<(unsigned)grid, warps * 32, 0, stream>>>(c);
  note_launch();
  return cudaGetLastError();
}

}  // namespace fb
