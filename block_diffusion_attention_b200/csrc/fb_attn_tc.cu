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
// Warp roles (224 threads):
//   warps 0-3  softmax: thread r owns query row r (TMEM lane r); copies its Q
//              row into tensor memory, then online softmax in fp32 with
//              base-2 exponentials (a quarter of them on the FMA pipe), P
//              written back into tensor memory as bf16 pairs, lazy rescaling
//              of the accumulator, epilogue (output tile staged in shared
//              memory, written by TMA stores);
//   warp 4     TMA producer of Q (once) and the K tiles, warp 6 of the V
//              tiles, into a ring of six 32 KB shared-memory slots (tile j's
//              K takes an even slot, its V an odd one): each producer refills
//              its own slots as soon as they are consumed, so a K load never
//              waits behind the release of a V slot;
//   warp 5     TMEM owner and MMA issuer: the whole warp runs the issue loop
//              (warp-uniform tile indices and descriptors) and one elected
//              lane issues the tcgen05.mma: S = Q K^T (A = Q from tensor
//              memory, B = K from shared memory) and O += P V (A = P from
//              tensor memory, B = V from shared memory), M = 128, N = 128,
//              K = 16.
//
// TMEM (512 columns): S double-buffered at columns [0, 128) and [128, 256) --
// tile j's P overwrites the first 64 columns of its own S buffer -- the O
// accumulator at [256, 384) and Q at [384, 448).  QK^T of tile j + 1
// therefore overlaps the softmax of tile j, and a K slot is released as soon
// as its QK^T is done.
// Shared memory (1024-byte aligned, 128-byte swizzle everywhere):
//   Q     [2 halves of 64 dims][128 rows][128 B]        32 KB
//   ring  6 x [2 halves][128 keys][128 B]              192 KB
//
// A refresh mask can leave units out (their CTAs return after the
// prologue), or share the grid out among the selected units only (the
// active-unit split; see AttnParams::dyn).
//
// Every mbarrier wait is bounded in time; on expiry the CTA records
// FB_ERR_DEVICE_TIMEOUT, drains its own copies and MMAs, frees TMEM and exits.
#include <cuda_bf16.h>
#include <math_constants.h>

#include <atomic>

#include "fb_attn_common.cuh"
#include "fb_internal.h"
#include "fb_ptx.cuh"

namespace fb {

namespace {

constexpr int NSLOT = TC_SLOTS;
constexpr uint32_t OFF_Q = 0;
constexpr uint32_t OFF_RING = OFF_Q + Q_BYTES;
constexpr uint32_t OFF_BAR = OFF_RING + NSLOT * SLOT_BYTES;
constexpr int NUM_BARS = 1 + 2 * NSLOT + 2 + 2 + 5;
constexpr uint32_t PRE_BYTES = BM * HD * 4;      // 64 KB: O_pre rows of a tile (f32)
constexpr int PRE_SLOT = NSLOT - 2;             // O_pre prefetch uses the last two ring slots
constexpr uint32_t SMEM_BYTES = OFF_BAR + 256 + 1024;  // + alignment slack
constexpr uint32_t TMEM_COLS = 512;
constexpr uint32_t TMEM_S0 = 0, TMEM_O = 256;           // S buffers at 0 and 128
constexpr uint32_t TMEM_Q = 384;                        // Q (bf16 pairs), 64 columns

static_assert(NUM_BARS * 8 + 8 <= 256, "barrier area");
static_assert(SMEM_BYTES <= 232448, "shared memory");

struct Shared {
  uint64_t* q_full;
  uint64_t* full;    // [NSLOT] ring slot loaded
  uint64_t* empty;   // [NSLOT] ring slot consumed
  uint64_t* s_full;  // [2] S buffer written by QK^T
  uint64_t* p_full;  // [2] P written into that S buffer (and O rescaled)
  uint64_t* o_done;  // [2] PV(j) finished: barrier j % 2
  uint64_t* drain;
  uint64_t* pre_full; // O_pre rows prefetched (merge epilogue of short units)
  uint64_t* q_tmem;   // Q copied into tensor memory by the softmax warps
  uint32_t* tmem_slot;
  volatile int* abort_flag;
};

__device__ __forceinline__ bool wait_bar(uint64_t* bar, uint32_t parity, const Shared& sh,
                                         int32_t* status, bool honour_abort = true) {
  return bounded_wait(bar, parity, sh.abort_flag, status, honour_abort);
}

// wait_bar for a whole warp: every lane waits, then the warp agrees on the
// outcome (a time-out seen by one lane ends the wait for all), so the warp
// collectives that follow never meet a split warp.
__device__ __forceinline__ bool wait_bar_warp(uint64_t* bar, uint32_t parity, const Shared& sh,
                                              int32_t* status) {
  return __all_sync(0xffffffffu, wait_bar(bar, parity, sh, status));
}

// Ring slot sequence: tile j uses slot item 2j for K and 2j + 1 for V.
__device__ __forceinline__ int slot_of(int item) { return item % NSLOT; }
__device__ __forceinline__ uint32_t use_of(int item) { return (uint32_t)(item / NSLOT); }

template <int EPI>
__global__ void __launch_bounds__(TC_THREADS, 1)
    attn_tc_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmKp,
                   const __grid_constant__ CUtensorMap tmVp, const __grid_constant__ CUtensorMap tmKb,
                   const __grid_constant__ CUtensorMap tmVb, const __grid_constant__ CUtensorMap tmPre,
                   const __grid_constant__ CUtensorMap tmO, const AttnParams p) {
  constexpr int NC = BN;  // key columns of a tile
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  uint8_t* sQ = smem + OFF_Q;
  uint8_t* sRing = smem + OFF_RING;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + OFF_BAR);
  Shared sh;
  sh.q_full = bars;
  sh.full = bars + 1;
  sh.empty = sh.full + NSLOT;
  sh.s_full = sh.empty + NSLOT;
  sh.p_full = sh.s_full + 2;
  sh.o_done = sh.p_full + 2;
  sh.drain = sh.o_done + 2;
  sh.pre_full = sh.drain + 1;
  sh.q_tmem = sh.pre_full + 1;
  sh.tmem_slot = reinterpret_cast<uint32_t*>(sh.q_tmem + 1);
  sh.abort_flag = reinterpret_cast<volatile int*>(sh.tmem_slot + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;


  if (threadIdx.x == 0) {
    mbar_init(sh.q_full, 1);
    for (int i = 0; i < NSLOT; ++i) {
      mbar_init(&sh.full[i], 1);
      mbar_init(&sh.empty[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&sh.s_full[i], 1);
      mbar_init(&sh.p_full[i], 4);
    }
    mbar_init(&sh.o_done[0], 1);
    mbar_init(&sh.o_done[1], 1);
    mbar_init(sh.drain, 1);
    mbar_init(sh.pre_full, 1);
    mbar_init(sh.q_tmem, 4);
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
  if (warp == 4 && lane == 0) {
    // tensor maps are kernel parameters: fetch them while the previous kernel finishes
    tma_prefetch_map(&tmQ);
    tma_prefetch_map(&tmKp);
    tma_prefetch_map(&tmVp);
    tma_prefetch_map(&tmKb);
    tma_prefetch_map(&tmVb);
    tma_prefetch_map(&tmPre);
    tma_prefetch_map(&tmO);
  }
  // This CTA's (b, kv head, query tile, key split) from its grid index, and
  // the key-tile count of a unit that has no prefix (the in-block step):
  // kernel parameters only, so they are worked out while the previous kernel
  // finishes.
  int b = 0, kvh = 0, rt = 0, split = 0, nsplit = p.nsplit;
  if (!p.dyn) {
    unsigned bid = blockIdx.x;
    split = (int)(bid % (unsigned)nsplit);
    bid /= (unsigned)nsplit;
    rt = (int)(bid % (unsigned)p.n_rt);
    bid /= (unsigned)p.n_rt;
    kvh = (int)(bid % (unsigned)p.Hkv);
    b = (int)(bid / (unsigned)p.Hkv);
  }
  UnitTiles u = p.src.has_prefix ? UnitTiles{0, 0, 0} : unit_tiles(p, b, kvh, false);

  // Everything above touches no global memory; from here on inputs may come
  // from the previous kernel in the stream.
  pdl_wait();
  pdl_launch_dependents();

  // A unit the refresh mask leaves out keeps its cached outputs: no work.  In
  // the active-unit split the grid is shared out among the selected units
  // only.  The mask, the prefix lengths and the chunk lists may be written by
  // the previous kernel, so they are read after the dependency wait.
  bool skip;
  if (p.dyn) {
    const int na = active_count(p.unit_mask, p.B * p.Hkv);
    nsplit = active_splits(gridDim.x, na, p.n_rt);
    const int a = blockIdx.x / (p.n_rt * nsplit);
    const int un = a < na ? active_unit(p.unit_mask, p.B * p.Hkv, a) : -1;
    skip = un < 0;
    b = skip ? 0 : un / p.Hkv;
    kvh = skip ? 0 : un % p.Hkv;
    rt = (blockIdx.x / nsplit) % p.n_rt;
    split = blockIdx.x % nsplit;
  } else {
    skip = p.unit_mask != nullptr && p.unit_mask[b * p.Hkv + kvh] == 0;
  }
  if (skip)
    u = UnitTiles{0, 0, 0};
  else if (p.src.has_prefix)
    u = unit_tiles(p, b, kvh, threadIdx.x == 0);
  // the unit's sparse chunk list (read through the L1 cache)
  const int32_t* clist =
      p.src.chunk_idx ? p.src.chunk_idx + ((size_t)b * p.Hkv + kvh) * p.src.topk : nullptr;
  const int ntot = u.n0 + u.n1;
  // split * ntot < 2^7 * 2^23: 32-bit arithmetic is exact
  const int j0 = (int)(((unsigned)split * (unsigned)ntot) / (unsigned)nsplit);
  const int j1 = (int)(((unsigned)(split + 1) * (unsigned)ntot) / (unsigned)nsplit);
  const int nt = j1 - j0;
  int32_t* status = p.dev_status;
  // The merge epilogue of a unit with at most two key tiles leaves the last
  // two ring slots free: the cached O_pre rows are prefetched into them.
  const bool pre_smem = (EPI == EPI_MERGE) && nt <= 2;

  if (skip) {
    // nothing to load, multiply or write
  } else if (warp == 4 || warp == 6) {
    // ----------------------------------------------------------- TMA producers
    if (lane == 0) {
      const int kv = warp == 6 ? 1 : 0;  // this producer's items: 2 jj + kv
      const uint64_t policy = p.kv_stream_once ? l2_policy_evict_first() : l2_policy_evict_normal();
      const int t0 = rt * (BM / p.G);
      if (kv == 0) {
        mbar_arrive_expect_tx(sh.q_full, Q_BYTES);
        tma_load_4d(sQ, &tmQ, sh.q_full, 0, kvh * p.G, t0, b);
        tma_load_4d(sQ + BM * 128, &tmQ, sh.q_full, 64, kvh * p.G, t0, b);
      }
      if (kv == 0 && pre_smem) {
        // [4 column blocks of 32 floats][128 rows][128 B], 128-byte swizzle
        mbar_arrive_expect_tx(sh.pre_full, PRE_BYTES);
#pragma unroll
        for (int c = 0; c < 4; ++c)
          tma_load_4d(sRing + PRE_SLOT * SLOT_BYTES + c * (BM * 128), &tmPre, sh.pre_full, c * 32, kvh * p.G,
                      t0, b);
      }
      int issued = 0;  // tiles whose item this producer has issued
      for (int jj = 0; jj < nt; ++jj) {
        const Tile t = tile_at(p, u, clist, j0 + jj);
        const int item = 2 * jj + kv;
        const int sl = slot_of(item);
        if (!wait_bar(&sh.empty[sl], (use_of(item) & 1) ^ 1, sh, status)) break;
        issued = jj + 1;
#ifdef FB_TEST_HOOKS
        if (p.test_skip_k1 && kv == 0 && jj == 1) continue;  // never loaded: its wait runs out
#endif
        mbar_arrive_expect_tx(&sh.full[sl], SLOT_BYTES);
        load_kv_tile(sRing + sl * SLOT_BYTES, kv ? &tmVp : &tmKp, kv ? &tmVb : &tmKb, &sh.full[sl], p, u, t, b,
                     kvh, policy);
      }
      // After an abort, let the copies in flight land before the CTA exits
      // (this producer's own: its last NSLOT / 2 items at most).
      if (*sh.abort_flag) {
        if (kv == 0) wait_bar(sh.q_full, 0, sh, nullptr, false);
        if (kv == 0 && pre_smem) wait_bar(sh.pre_full, 0, sh, nullptr, false);
        for (int jj = max(0, issued - NSLOT / 2); jj < issued; ++jj) {
#ifdef FB_TEST_HOOKS
          if (p.test_skip_k1 && kv == 0 && jj == 1) continue;
#endif
          const int item = 2 * jj + kv;
          wait_bar(&sh.full[slot_of(item)], use_of(item) & 1, sh, nullptr, false);
        }
      }
    }
  } else if (warp == 5) {
    // --------------------------------------------------------------- MMA issuer
    constexpr uint32_t IDESC_PV = idesc_bf16_f32(BM, HD, false, true);
    constexpr uint32_t IDESC_QK_FULL = idesc_bf16_f32(BM, NC, false, false);
    const uint32_t tO = tmem + TMEM_O;
    // Shared-memory descriptors: built once; an operand at byte offset `off`
    // from its base is the base descriptor plus off >> 4 (start-address field).
    const uint64_t dK = sw128_desc(smem_u32(sRing), 16, 1024);
    const uint64_t dV = sw128_desc(smem_u32(sRing), HALF_BYTES, 1024);
    // The whole warp runs the issue loop, so tile indices, descriptors and
    // tensor-memory addresses are warp-uniform values; one elected lane issues
    // each group of tcgen05.mma and its commits.
    const bool leader = elect_one_sync();
    // A tile with fewer valid keys runs N = (valid keys rounded up to 16) for
    // QK^T and as many 16-key steps of PV: no work on empty columns.
    auto issue_qk = [&](int jj, int nvalid) {
      const uint32_t idesc =
          nvalid >= NC ? IDESC_QK_FULL : idesc_bf16_f32(BM, min(NC, (nvalid + 15) & ~15), false, false);
      const uint64_t dk = dK + ((slot_of(2 * jj) * SLOT_BYTES) >> 4);
      const uint32_t tS = tmem + TMEM_S0 + (uint32_t)(jj & 1) * BN;
      // A = Q from tensor memory (16 dims = 8 packed columns per step), B = K
      // from shared memory: only K crosses the shared-memory read port
      if (leader) {
#pragma unroll
        for (int kk = 0; kk < HD / 16; ++kk) {
          const uint32_t off = ((kk >> 2) * HALF_BYTES + (kk & 3) * 32) >> 4;
          umma_bf16_ts(tS, tmem + TMEM_Q + kk * 8, dk + off, idesc, kk > 0);
        }
      }
    };
    auto issue_pv = [&](int jj, int nvalid) {
      const uint64_t dv = dV + ((slot_of(2 * jj + 1) * SLOT_BYTES) >> 4);
      const uint32_t tP = tmem + TMEM_S0 + (uint32_t)(jj & 1) * BN;  // P (bf16 pairs) over S
      const int ksteps = (nvalid + 15) >> 4;
      if (leader) {
#pragma unroll
        for (int kk = 0; kk < NC / 16; ++kk)
          if (kk < ksteps)
            umma_bf16_ts(tO, tP + kk * 8, dv + ((kk * 16 * 128) >> 4), IDESC_PV, (jj > 0 || kk > 0) ? 1u : 0u);
      }
    };
    // Per tile j: QK^T(j + 1) as soon as K(j + 1) has landed (the tensor pipe
    // then works while the softmax of tile j runs), then V(j) is waited for
    // and its tail rows cleared, so that the work between "P of tile j is
    // ready" and the PV(j) issue is one barrier test.  (This warp shares its
    // scheduler with a softmax warp, so every instruction on that path
    // delays the tensor pipe.)
    bool ok = wait_bar_warp(sh.q_tmem, 0, sh, status);
    if (ok && nt > 0) {
      Tile tc = tile_at(p, u, clist, j0);
      ok = wait_bar_warp(&sh.full[slot_of(0)], 0, sh, status);
      if (ok) {
        tc_fence_after_sync();
        issue_qk(0, tc.nvalid);
        if (leader) {
          tc_commit(&sh.s_full[0]);
          tc_commit(&sh.empty[slot_of(0)]);
        }
      }
      for (int jj = 0; ok && jj < nt; ++jj) {
        Tile tn = tc;
        if (jj + 1 < nt) {
          tn = tile_at(p, u, clist, j0 + jj + 1);
          const int ik = 2 * (jj + 1);
          if (!(ok = wait_bar_warp(&sh.full[slot_of(ik)], use_of(ik) & 1, sh, status))) break;
          tc_fence_after_sync();
          issue_qk(jj + 1, tn.nvalid);
          if (leader) {
            tc_commit(&sh.s_full[(jj + 1) & 1]);
            tc_commit(&sh.empty[slot_of(ik)]);
          }
        }
        const int iv = 2 * jj + 1;
        if (!(ok = wait_bar_warp(&sh.full[slot_of(iv)], use_of(iv) & 1, sh, status))) break;
        if (tc.seg == 0 && (tc.nvalid & 15)) {
          // Cache rows past the prefix may hold anything (even NaN); P is 0
          // there but 0 * NaN is not, so clear the V rows up to the next
          // 16-key step that PV reads (at most 15 rows, once per unit), the
          // warp's lanes sharing the 16-byte stores.
          uint8_t* dVs = sRing + slot_of(iv) * SLOT_BYTES;
          const int nrow = ((tc.nvalid + 15) & ~15) - tc.nvalid;
          for (int i = lane; i < nrow * 16; i += 32) {
            const int r = tc.nvalid + (i >> 4);
            const int h = (i >> 3) & 1;
            const int c = i & 7;
            *reinterpret_cast<uint4*>(dVs + h * HALF_BYTES + r * 128 + c * 16) = make_uint4(0, 0, 0, 0);
          }
          fence_proxy_async_smem();
          __syncwarp();
        }
        if (!(ok = wait_bar_warp(&sh.p_full[jj & 1], (jj >> 1) & 1, sh, status))) break;
        tc_fence_after_sync();
        issue_pv(jj, tc.nvalid);
        if (leader) {
          tc_commit(&sh.o_done[jj & 1]);
          tc_commit(&sh.empty[slot_of(iv)]);
        }
        tc = tn;
      }
    }
    // Drain every MMA this warp issued before TMEM can be released (a drain
    // that runs out of time is recorded too, unless an error already is).
    if (leader) tc_commit(sh.drain);
    __syncwarp();
    wait_bar(sh.drain, 0, sh, status, false);
  } else {
    // ------------------------------------------------------ softmax + epilogue
    const int r = warp * 32 + lane;  // query row of this thread = TMEM lane
    const uint32_t lane_off = (uint32_t)(warp * 32) << 16;
    const uint32_t tO = tmem + TMEM_O + lane_off;
    const float c2 = p.scale_log2;
    const int pr = rt * BM + r;
    const int tok = pr / p.G;
    const int h = kvh * p.G + (pr - tok * p.G);
    // cached LSE of this row, read before the key loop so its latency hides
    const float lp_nat = (EPI == EPI_MERGE && tok < p.S) ? p.pre_lse[((size_t)b * p.Hq + h) * p.S + tok]
                                                          : -CUDART_INF_F;
    float m_run = -CUDART_INF_F;
    float l_run = 0.f;
    bool ok = wait_bar_warp(sh.q_full, 0, sh, status);
    if (ok) {
      // this thread's Q row (128 bf16, 128-byte swizzled in two 64-dim halves)
      // into TMEM columns [TMEM_Q, TMEM_Q + 64): the A operand of QK^T
      const uint32_t qrow = smem_u32(sQ) + r * 128;
#pragma unroll
      for (int hf = 0; hf < 2; ++hf) {
        uint32_t qv[32];
#pragma unroll
        for (int ch = 0; ch < 8; ++ch) {
          const uint32_t addr = qrow + hf * (BM * 128) + ((ch ^ (r & 7)) << 4);
          asm volatile("ld.shared.v4.b32 {%0, %1, %2, %3}, [%4];"
                       : "=r"(qv[ch * 4]), "=r"(qv[ch * 4 + 1]), "=r"(qv[ch * 4 + 2]), "=r"(qv[ch * 4 + 3])
                       : "r"(addr));
        }
        tmem_st_32x32(tmem + TMEM_Q + lane_off + hf * 32, qv);
      }
      tmem_st_wait();
      tc_fence_before_sync();
      __syncwarp();
      if (lane == 0) mbar_arrive(sh.q_tmem);
    }
    for (int jj = 0; ok && jj < nt; ++jj) {
      const uint32_t tS = tmem + TMEM_S0 + (uint32_t)(jj & 1) * BN + lane_off;
      const Tile t = tile_at(p, u, clist, j0 + jj);
      if (!(ok = wait_bar_warp(&sh.s_full[jj & 1], (jj >> 1) & 1, sh, status))) break;
      tc_fence_after_sync();
      // S row of this thread.  A tail tile (fewer than BN valid keys) sets
      // the columns past its keys to -inf first; full tiles skip that block.
      uint32_t sv[NC];
#pragma unroll
      for (int c = 0; c < NC / 32; ++c)
        tmem_ld_32x32(tS + c * 32, *reinterpret_cast<uint32_t(*)[32]>(&sv[c * 32]));
      tmem_ld_wait();
      if (t.nvalid < NC) {
#pragma unroll
        for (int c = 0; c < NC; ++c)
          if (c >= t.nvalid) sv[c] = 0xff800000u;  // -inf
      }
      float* s = reinterpret_cast<float*>(sv);  // S, then p in place
      float mx0 = fmax3(s[0], s[1], s[2]), mx1 = fmax3(s[3], s[4], s[5]);
#pragma unroll
      for (int c = 6; c + 4 <= NC; c += 4) {
        mx0 = fmax3(mx0, s[c], s[c + 1]);
        mx1 = fmax3(mx1, s[c + 2], s[c + 3]);
      }
      // NC - 6 is a multiple of 4 plus 2: the last two columns
      mx0 = fmax3(mx0, mx1, fmaxf(s[NC - 2], s[NC - 1]));
      const float mt = mx0 * c2;
      const bool need = mt > m_run + RESCALE_LOG2;
      const float m_new = need ? mt : m_run;
      const float alpha = ex2_approx(m_run - m_new);  // 0 when m_run = -inf
      const float m_use = (m_new == -CUDART_INF_F) ? 0.f : m_new;
      // p = 2^(s * c2 - m): packed FMA for the argument; three of every four
      // pairs through MUFU.EX2, one through the FMA-pipe polynomial
      const float2 c2v = make_float2(c2, c2), mv = make_float2(-m_use, -m_use);
      float2 la = make_float2(0.f, 0.f), lb = make_float2(0.f, 0.f);
#pragma unroll
      for (int c = 0; c < NC; c += 8) {
        float2 x0 = ffma2(make_float2(s[c], s[c + 1]), c2v, mv);
        float2 x1 = ffma2(make_float2(s[c + 2], s[c + 3]), c2v, mv);
        float2 x2 = ffma2(make_float2(s[c + 4], s[c + 5]), c2v, mv);
        float2 x3 = ffma2(make_float2(s[c + 6], s[c + 7]), c2v, mv);
        x0 = make_float2(ex2_approx(x0.x), ex2_approx(x0.y));
        x1 = make_float2(ex2_approx(x1.x), ex2_approx(x1.y));
        x2 = make_float2(ex2_approx(x2.x), ex2_approx(x2.y));
        x3 = exp2_poly2(x3);
        s[c] = x0.x; s[c + 1] = x0.y; s[c + 2] = x1.x; s[c + 3] = x1.y;
        s[c + 4] = x2.x; s[c + 5] = x2.y; s[c + 6] = x3.x; s[c + 7] = x3.y;
        la = fadd2(la, fadd2(x0, x1));
        lb = fadd2(lb, fadd2(x2, x3));
      }
      const float l0 = la.x, l1 = la.y, l2 = lb.x, l3 = lb.y;
      l_run = l_run * alpha + ((l0 + l1) + (l2 + l3));
      m_run = m_new;

      if (jj > 0 && __any_sync(0xffffffffu, need)) {
        // Rows whose max moved rescale the accumulator once PV(j - 1) is
        // done.  PV(j - 1) commits to o_done[(j - 1) % 2], whose next phase
        // is PV(j + 1), behind this tile's P: the barrier is never two phases
        // ahead of this wait even though tiles without a rescale skip it.
        if (!(ok = wait_bar_warp(&sh.o_done[(jj - 1) & 1], ((jj - 1) >> 1) & 1, sh, status))) break;
        tc_fence_after_sync();
#pragma unroll
        for (int c = 0; c < HD / 32; ++c) {
          uint32_t ov[32];
          tmem_ld_32x32(tO + c * 32, ov);
          tmem_ld_wait();
#pragma unroll
          for (int i = 0; i < 32; ++i) ov[i] = __float_as_uint(__uint_as_float(ov[i]) * alpha);
          tmem_st_32x32(tO + c * 32, ov);
        }
      }
      // P as bf16 pairs over the first 64 columns of this S buffer: the
      // A operand of PV, read from tensor memory.
#pragma unroll
      for (int c = 0; c < NC / 64; ++c) {
        uint32_t pk[32];
#pragma unroll
        for (int i = 0; i < 32; ++i) pk[i] = pack_bf16x2(s[c * 64 + 2 * i], s[c * 64 + 2 * i + 1]);
        tmem_st_32x32(tS + c * 32, pk);
      }
      tmem_st_wait();
      tc_fence_before_sync();
      __syncwarp();
      if (lane == 0) mbar_arrive(&sh.p_full[jj & 1]);
    }
    if (ok && nt > 0) {
      ok = wait_bar_warp(&sh.o_done[(nt - 1) & 1], ((nt - 1) >> 1) & 1, sh, status);
      tc_fence_after_sync();
    }
    if (ok && pre_smem) ok = wait_bar_warp(sh.pre_full, 0, sh, status);
    // ---------------------------------------------------------------- epilogue
    const bool row_ok = ok && tok < p.S;
    const bool empty = (nt == 0) || !(l_run > 0.f);
    const float inv_l = empty ? 0.f : 1.f / l_run;
    const float lse2 = empty ? -CUDART_INF_F : m_run + log2f(l_run);  // log2 of Z
    // the whole accumulator row in one batch of TMEM loads
    uint32_t ov[HD];
    if (nt > 0) {
#pragma unroll
      for (int c = 0; c < HD / 32; ++c)
        tmem_ld_32x32(tO + c * 32, *reinterpret_cast<uint32_t(*)[32]>(&ov[c * 32]));
      tmem_ld_wait();
    } else {
#pragma unroll
      for (int i = 0; i < HD; ++i) ov[i] = 0u;
    }
    // The output tile is staged in ring slots 0-1 (every K/V tile has been
    // consumed once the last PV is done; slots 4-5 may hold O_pre) in the
    // 128-byte-swizzled packed-row layout of its tensor map, then written by
    // one TMA store per 128-byte column block: coalesced, and rows past the
    // block's last token are dropped by the copy.
    uint8_t* stage = sRing;
    const uint32_t st_row = smem_u32(stage) + r * 128;
    if (EPI == EPI_PARTIAL) {
      if (ok) {
#pragma unroll
        for (int c = 0; c < HD / 32; ++c)
#pragma unroll
          for (int ch = 0; ch < 8; ++ch) {
            const int i = c * 32 + ch * 4;
            st_shared_v4(st_row + c * (BM * 128) + ((ch ^ (r & 7)) << 4),
                         __float_as_uint(__uint_as_float(ov[i]) * inv_l),
                         __float_as_uint(__uint_as_float(ov[i + 1]) * inv_l),
                         __float_as_uint(__uint_as_float(ov[i + 2]) * inv_l),
                         __float_as_uint(__uint_as_float(ov[i + 3]) * inv_l));
          }
      }
      if (p.dyn) {
        if (ok) p.out_lse[(size_t)blockIdx.x * BM + r] = lse2 * LN2;  // slot layout: every row
      } else if (row_ok) {
        p.out_lse[(((size_t)split * p.B + b) * p.Hq + h) * p.S + tok] = lse2 * LN2;
      }
    } else {
      const size_t orow = ((size_t)b * p.S + tok) * p.Hq + h;
      float wp = 0.f, wo = inv_l, inv_den = 1.f, lse_out2 = lse2;
      if (EPI == EPI_MERGE) {
        // merge equation in base 2: weights e^{L - m} become 2^{L2 - M}
        const float lp2 = row_ok ? lp_nat * 1.4426950408889634f : -CUDART_INF_F;
        const float M = fmaxf(lp2, lse2);
        const float Ms = (M == -CUDART_INF_F) ? 0.f : M;
        wp = ex2_approx(lp2 - Ms);
        const float wi = ex2_approx(lse2 - Ms);
        const float den = wp + wi;
        inv_den = den > 0.f ? 1.f / den : 0.f;
        wo = empty ? 0.f : ex2_approx(m_run - Ms);  // = wi / l_run
        lse_out2 = den > 0.f ? Ms + log2f(den) : -CUDART_INF_F;
      }
      const float* pre = (EPI == EPI_MERGE) ? p.pre_o + orow * HD : nullptr;
      if (row_ok) {
#pragma unroll
        for (int c = 0; c < HD / 32; ++c) {
          float o[32];
#pragma unroll
          for (int i = 0; i < 32; ++i) o[i] = __uint_as_float(ov[c * 32 + i]) * wo;
          if (EPI == EPI_MERGE) {
            const uint8_t* prow = sRing + PRE_SLOT * SLOT_BYTES + c * (BM * 128) + r * 128;
#pragma unroll
            for (int i = 0; i < 32; i += 4) {
              const float4 q = pre_smem ? *reinterpret_cast<const float4*>(prow + (((i >> 2) ^ (r & 7)) << 4))
                                        : *reinterpret_cast<const float4*>(pre + c * 32 + i);
              o[i] = (o[i] + wp * q.x) * inv_den;
              o[i + 1] = (o[i + 1] + wp * q.y) * inv_den;
              o[i + 2] = (o[i + 2] + wp * q.z) * inv_den;
              o[i + 3] = (o[i + 3] + wp * q.w) * inv_den;
            }
          }
          // 32 columns = chunks (c & 1) * 4 .. + 3 of the 64-dim half c >> 1
#pragma unroll
          for (int i = 0; i < 32; i += 8) {
            const int ch = (c & 1) * 4 + (i >> 3);
            st_shared_v4(st_row + (c >> 1) * (BM * 128) + ((ch ^ (r & 7)) << 4), pack_bf16x2(o[i], o[i + 1]),
                         pack_bf16x2(o[i + 2], o[i + 3]), pack_bf16x2(o[i + 4], o[i + 5]),
                         pack_bf16x2(o[i + 6], o[i + 7]));
          }
        }
        if (p.out_lse) p.out_lse[((size_t)b * p.Hq + h) * p.S + tok] = lse_out2 * LN2;
      }
    }
    fence_proxy_async_smem();
    named_bar_sync(1, 4 * 32);
    if (r == 0 && !*sh.abort_flag) {
      const int t0 = rt * (BM / p.G);
      if (EPI == EPI_PARTIAL) {
#pragma unroll
        for (int c = 0; c < HD / 32; ++c)
          tma_store_4d(&tmO, stage + c * (BM * 128), c * 32, p.dyn ? 0 : kvh * p.G, p.dyn ? 0 : t0,
                       p.dyn ? (int)blockIdx.x : split * p.B + b);
      } else {
#pragma unroll
        for (int hf = 0; hf < 2; ++hf) tma_store_4d(&tmO, stage + hf * (BM * 128), hf * 64, kvh * p.G, t0, b);
      }
      tma_store_commit();
      tma_store_wait_read();
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
// equation applied across splits, in a fixed order).  One warp per row: lanes
// read the splits' LSEs in parallel, then each lane accumulates four output
// columns over the splits.  The partials come in one of three layouts: one
// [B][S][Hq] set per split, the active-unit slots (CombineParams::dyn), or
// the tail slots of the two-tile kernel (CombineParams::tail_k, only the
// tail units' rows).
constexpr int CMB_WARPS = 4;
constexpr int CMB_INFLIGHT = 16;  // split loads in flight per lane (divides 32)
static_assert(TC_MAX_SPLITS == 128, "combine holds four split weights per lane");

__device__ __forceinline__ float warp_max_f(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}
__device__ __forceinline__ float warp_sum_f(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

__global__ void __launch_bounds__(CMB_WARPS * 32) combine_kernel(const CombineParams c) {
  pdl_wait();
  pdl_launch_dependents();
  const int wi = threadIdx.x >> 5;
  long long row = (long long)blockIdx.x * CMB_WARPS + wi;
  const int lane = threadIdx.x & 31;
  const long long nrows = (long long)c.B * c.S * c.Hq;
  int h, t, b;
  const float* base;
  const float* lbase;
  size_t so, sl;  // split strides of the partial O and LSE
  int nsplit;
  if (c.tail_k > 0) {
    // the tail units' rows (two tiles of 128 packed rows per unit) from the
    // slots (tail unit, split, tile) of the two-tile kernel's tail splits
    if (row >= (long long)c.tail_units * 2 * TC_BM) return;
    const int ti = (int)(row / (2 * TC_BM));
    const int rr = (int)(row % (2 * TC_BM));
    long long u = (long long)c.tail_u0 + ti;
    const int pair = (int)(u % c.npair);
    u /= c.npair;
    const int kvh = (int)(u % c.Hkv);
    b = (int)(u / c.Hkv);
    const int pr = pair * 2 * TC_BM + rr;  // packed query row of the unit
    if (pr >= c.S * c.G) return;
    t = pr / c.G;
    h = kvh * c.G + pr % c.G;
    row = ((long long)b * c.S + t) * c.Hq + h;
    const size_t slot0 = (size_t)ti * c.tail_k * 2 + rr / TC_BM;
    base = c.part_o + (slot0 * TC_BM + rr % TC_BM) * c.D;
    lbase = c.part_lse + slot0 * TC_BM + rr % TC_BM;
    so = (size_t)2 * TC_BM * c.D;
    sl = 2 * TC_BM;
    nsplit = c.tail_k;
  } else {
    if (row >= nrows) return;
    h = (int)(row % c.Hq);
    const long long bt = row / c.Hq;
    t = (int)(bt % c.S);
    b = (int)(bt / c.S);
    base = c.part_o + row * c.D;
    lbase = c.part_lse + ((size_t)b * c.Hq + h) * c.S + t;
    so = (size_t)nrows * c.D;
    sl = (size_t)c.B * c.Hq * c.S;
    nsplit = c.nsplit;
  }
  const size_t lrow = ((size_t)b * c.Hq + h) * c.S + t;
  const int unit = b * (c.Hq / c.G) + h / c.G;
  if (c.unit_mask && c.unit_mask[unit] == 0) return;  // unit not refreshed
  if (c.dyn) {
    // active-unit slots: (rank of the unit, query tile, split) -> [128][D] rows
    const int na = active_count(c.unit_mask, c.B * (c.Hq / c.G));
    const int a = active_rank(c.unit_mask, unit);
    nsplit = active_splits(c.grid, na, c.n_rt);
    const int pr = t * c.G + h % c.G;  // packed query row of the unit
    const size_t slot0 = ((size_t)a * c.n_rt + pr / TC_BM) * nsplit;
    base = c.part_o + (slot0 * TC_BM + pr % TC_BM) * c.D;
    lbase = c.part_lse + slot0 * TC_BM + pr % TC_BM;
    so = (size_t)TC_BM * c.D;
    sl = TC_BM;
  }
  // the cached pair as one more partial (a tail split of the step: the
  // merge equation over the splits and the pair at once)
  const bool pre = c.tail_k > 0 && c.pre_o != nullptr;
  if (pre || (nsplit <= 32 && c.D == 4 * 32)) {
    // up to 32 partials: every load in flight at once -- lane l reads
    // partial l's LSE and the four output columns 4l..4l+3 of every partial
    const int nterm = nsplit + (pre ? 1 : 0);
    float lse_l = lane < nsplit ? lbase[lane * sl] : -CUDART_INF_F;
    if (pre && lane == nsplit) lse_l = c.pre_lse[lrow];
    float4 v[32];
#pragma unroll
    for (int i = 0; i < 32; ++i) {
      if (i < nsplit)
        v[i] = __ldg(reinterpret_cast<const float4*>(base + i * so + lane * 4));
      else if (pre && i == nsplit)
        v[i] = __ldg(reinterpret_cast<const float4*>(c.pre_o + row * c.D + lane * 4));
    }
    const float M = warp_max_f(lse_l);
    const bool empty = (M == -CUDART_INF_F);
    const float w_l = (empty || lse_l == -CUDART_INF_F) ? 0.f : expf(lse_l - M);
    const float den = warp_sum_f(w_l);
    const float inv = den > 0.f ? 1.f / den : 0.f;
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
    for (int i = 0; i < 32; ++i) {
      const float w = __shfl_sync(0xffffffffu, w_l, i);  // partial order, as below
      if (i < nterm) {
        acc.x = fmaf(w, v[i].x, acc.x);
        acc.y = fmaf(w, v[i].y, acc.y);
        acc.z = fmaf(w, v[i].z, acc.z);
        acc.w = fmaf(w, v[i].w, acc.w);
      }
    }
    acc = make_float4(acc.x * inv, acc.y * inv, acc.z * inv, acc.w * inv);
    const int d0 = lane * 4;
    if (c.out_o32) {
      *reinterpret_cast<float4*>(c.out_o32 + row * c.D + d0) = acc;
    } else if (c.out_bf16) {
      uint2 u = make_uint2(pack_bf16x2(acc.x, acc.y), pack_bf16x2(acc.z, acc.w));
      *reinterpret_cast<uint2*>(reinterpret_cast<__nv_bfloat16*>(c.out_o) + row * c.D + d0) = u;
    } else {
      *reinterpret_cast<float4*>(reinterpret_cast<float*>(c.out_o) + row * c.D + d0) = acc;
    }
    if (lane == 0 && c.out_lse) c.out_lse[lrow] = empty ? -CUDART_INF_F : M + logf(den);
    return;
  }
  // lane l holds the LSE (then the weight) of splits l, l + 32, l + 64, l + 96
  constexpr int PER_LANE = TC_MAX_SPLITS / 32;
  float wreg[PER_LANE];
  float M = -CUDART_INF_F;
#pragma unroll
  for (int k = 0; k < PER_LANE; ++k) {
    const int s = lane + 32 * k;
    wreg[k] = s < nsplit ? lbase[s * sl] : -CUDART_INF_F;
    M = fmaxf(M, wreg[k]);
  }
  M = warp_max_f(M);
  const bool empty = (M == -CUDART_INF_F);
  float den = 0.f;
#pragma unroll
  for (int k = 0; k < PER_LANE; ++k) {
    wreg[k] = (empty || wreg[k] == -CUDART_INF_F) ? 0.f : expf(wreg[k] - M);
    den += wreg[k];
  }
  den = warp_sum_f(den);
  const float inv = den > 0.f ? 1.f / den : 0.f;
  for (int d0 = lane * 4; d0 < c.D; d0 += 128) {
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    // CMB_INFLIGHT splits' loads in flight at once, then the weighted sum in
    // split order
    for (int s0 = 0; s0 < nsplit; s0 += CMB_INFLIGHT) {
      float4 v[CMB_INFLIGHT];
#pragma unroll
      for (int i = 0; i < CMB_INFLIGHT; ++i)
        if (s0 + i < nsplit) v[i] = __ldg(reinterpret_cast<const float4*>(base + (s0 + i) * so + d0));
      const int k = s0 >> 5;  // the same for the whole batch (CMB_INFLIGHT divides 32)
      const float wk = k == 0 ? wreg[0] : k == 1 ? wreg[1] : k == 2 ? wreg[2] : wreg[3];
#pragma unroll
      for (int i = 0; i < CMB_INFLIGHT; ++i) {
        const float w = __shfl_sync(0xffffffffu, wk, (s0 + i) & 31);
        if (s0 + i < nsplit) {
          acc.x = fmaf(w, v[i].x, acc.x);
          acc.y = fmaf(w, v[i].y, acc.y);
          acc.z = fmaf(w, v[i].z, acc.z);
          acc.w = fmaf(w, v[i].w, acc.w);
        }
      }
    }
    acc.x *= inv;
    acc.y *= inv;
    acc.z *= inv;
    acc.w *= inv;
    if (c.out_o32) {
      *reinterpret_cast<float4*>(c.out_o32 + row * c.D + d0) = acc;
    } else if (c.out_bf16) {
      uint2 v = make_uint2(pack_bf16x2(acc.x, acc.y), pack_bf16x2(acc.z, acc.w));
      *reinterpret_cast<uint2*>(reinterpret_cast<__nv_bfloat16*>(c.out_o) + row * c.D + d0) = v;
    } else {
      *reinterpret_cast<float4*>(reinterpret_cast<float*>(c.out_o) + row * c.D + d0) = acc;
    }
  }
  if (lane == 0 && c.out_lse) c.out_lse[lrow] = empty ? -CUDART_INF_F : M + logf(den);
}

}  // namespace

size_t tc_smem_bytes() { return SMEM_BYTES; }

cudaError_t launch_attn_tc(const AttnParams& p, const CUtensorMap& tmQ, const CUtensorMap& tmKp,
                           const CUtensorMap& tmVp, const CUtensorMap& tmKb, const CUtensorMap& tmVb,
                           const CUtensorMap& tmPre, const CUtensorMap& tmO, int grid, cudaStream_t stream) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  int which;
  void (*kern)(CUtensorMap, CUtensorMap, CUtensorMap, CUtensorMap, CUtensorMap, CUtensorMap, CUtensorMap,
               AttnParams);
  if (p.epi == EPI_PARTIAL) {
    kern = attn_tc_kernel<EPI_PARTIAL>;
    which = 0;
  } else if (p.epi == EPI_MERGE) {
    kern = attn_tc_kernel<EPI_MERGE>;
    which = 1;
  } else {
    kern = attn_tc_kernel<EPI_NORM>;
    which = 2;
  }
  // (set once per device and kernel; concurrent first calls both set it)
  static std::atomic<bool> configured[64][3];
  if (dev >= 64 || !configured[dev][which].load(std::memory_order_acquire)) {
    e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)SMEM_BYTES);
    if (e != cudaSuccess) return e;
    if (dev < 64) configured[dev][which].store(true, std::memory_order_release);
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)grid);
  cfg.blockDim = dim3(TC_THREADS);
  cfg.dynamicSmemBytes = SMEM_BYTES;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  e = cudaLaunchKernelEx(&cfg, kern, tmQ, tmKp, tmVp, tmKb, tmVb, tmPre, tmO, p);
  note_launch();
  return e != cudaSuccess ? e : cudaGetLastError();
}

cudaError_t launch_combine(const CombineParams& c, cudaStream_t stream) {
  const long long rows = c.tail_k > 0 ? (long long)c.tail_units * 2 * TC_BM : (long long)c.B * c.S * c.Hq;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)((rows + CMB_WARPS - 1) / CMB_WARPS));
  cfg.blockDim = dim3(CMB_WARPS * 32);
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  cudaError_t e = cudaLaunchKernelEx(&cfg, combine_kernel, c);
  note_launch();
  return e != cudaSuccess ? e : cudaGetLastError();
}

}  // namespace fb
