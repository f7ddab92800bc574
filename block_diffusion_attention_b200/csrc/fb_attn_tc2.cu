// fb_attn_tc2.cu -- bf16 attention partials on the sm_100a tensor cores, two
// 128-row query tiles per CTA.
//
// The same computation as attn_tc_kernel (fb_attn_tc.cu): one (batch b, kv
// head, query rows, key-range split) work item of softmax attention, the
// partial (A, L = log Z) of the Core Mechanism of "FlashBlock: Attention
// Caching for Efficient Long-Context Block Diffusion" (Technical Summary §2),
// with the same three epilogues (EPI_PARTIAL, EPI_MERGE, EPI_NORM).  Here a
// CTA owns two query tiles A and B of the same unit, so
//   * every K/V tile is brought into shared memory once for 256 query rows
//     (a unit of two tiles -- the batched sparse workload -- streams its keys
//     once instead of twice), and
//   * the tensor pipe always has the other tile's work queued while one
//     tile's softmax runs: per key tile j the MMA warp issues
//         PV_A(j), QK_A(j+1), PV_B(j), QK_B(j+1)
//     so the softmax of A(j+1) overlaps PV_B(j) and QK_B(j+1), and the
//     softmax of B(j+1) overlaps PV_A(j+1) and QK_A(j+2).
//
// Warp roles (384 threads, three warpgroups):
//   warpgroup 0  softmax + epilogue of tile A: thread r owns query row r (TMEM
//                lane r); online softmax in fp32 with base-2 exponentials (a
//                quarter of them on the FMA pipe), P written back over S in
//                tensor memory as bf16 pairs, lazy rescaling of O;
//   warpgroup 1  the same for tile B;
//   warpgroup 2  warp 8: TMA producer of Q (both tiles, once) and the K
//                tiles; warp 9: TMEM owner and MMA issuer (the whole warp runs
//                the issue loop, one elected lane issues); warp 10: TMA
//                producer of the V tiles; warp 11: idle.
// Registers: launched at 168 per thread; warpgroup 2 gives its registers
// back (setmaxnreg.dec to 72) and the two softmax warpgroups take them
// (setmaxnreg.inc to 216): 2 x 128 x 216 + 128 x 72 = 168 x 384.
//
// Tensor memory (512 columns): S_A [0, 128), S_B [128, 256) -- tile X's P
// overwrites the first 64 columns of S_X -- O_A [256, 384), O_B [384, 512).
// QK^T reads Q from shared memory (both operands K-major, 128-byte swizzle),
// PV reads P from tensor memory and V (MN-major) from shared memory.
// The tensor pipe runs tcgen05.mma in issue order, and every barrier signal
// is a tcgen05.commit that completes after all earlier MMAs, so:
//   * QK_X(j+1), issued after PV_X(j), overwrites S_X only after PV_X(j) has
//     read P_X(j);
//   * once S_X(j+1) is signalled, PV_X(j) is done: the softmax may rescale
//     O_X without waiting for it separately.
// Shared memory (1024-byte aligned, 128-byte swizzle everywhere):
//   Q_A, Q_B  2 x [2 halves of 64 dims][128 rows][128 B]    64 KB
//   ring      5 x 32 KB slots: K(j) is item 2j, V(j) item 2j + 1, slot =
//             item mod 5; each producer waits for its item's slot to be
//             released (K(j) after QK_B(j), V(j) after PV_B(j))        160 KB
//   chunk list of the unit (sparse prefix, up to 256 entries)          1 KB
// The epilogue of tile X stages its output in Q_X's region (every QK^T is
// done once the last PV_X is).
//
// A pass whose last wave of CTAs is only partly full may split the keys of
// those last units (AttnParams::tail_k): such a CTA writes f32 partial rows
// to its tiles' slots through the second output map, and the combine merges
// them (for the step, together with the cached pair).
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

constexpr int NSLOT2 = 5;
constexpr int THREADS2 = 384;
constexpr uint32_t OFF_Q2 = 0;                                // Q_A, then Q_B
constexpr uint32_t OFF_RING2 = OFF_Q2 + 2 * Q_BYTES;
constexpr uint32_t OFF_BAR2 = OFF_RING2 + NSLOT2 * SLOT_BYTES;
constexpr int NUM_BARS2 = 1 + 2 * NSLOT2 + 2 + 2 + 2 + 1;
constexpr uint32_t OFF_CL2 = OFF_BAR2 + 256;                  // chunk-list copy
constexpr int CL_MAX = 256;
constexpr uint32_t SMEM2_BYTES = OFF_CL2 + CL_MAX * 4 + 1024;  // + alignment slack
constexpr uint32_t TMEM2_COLS = 512;
constexpr uint32_t TMEM2_O = 256;  // O_A at 256, O_B at 384; S_A at 0, S_B at 128
constexpr uint32_t REG_LAUNCH = 168, REG_SOFTMAX = 216, REG_OTHER = 72;

static_assert(NUM_BARS2 * 8 + 8 <= 256, "barrier area");
static_assert(SMEM2_BYTES <= 232448, "shared memory");
static_assert(2 * 128 * REG_SOFTMAX + 128 * REG_OTHER <= REG_LAUNCH * THREADS2, "register split");

struct Shared2 {
  uint64_t* q_full;
  uint64_t* full;     // [NSLOT2] ring slot loaded
  uint64_t* empty;    // [NSLOT2] ring slot consumed
  uint64_t* s_full;   // [2] S_X written by QK_X(j)
  uint64_t* p_full;   // [2] P_X(j) written by softmax X (4 warps)
  uint64_t* o_final;  // [2] the last PV_X done
  uint64_t* drain;
  uint32_t* tmem_slot;
  volatile int* abort_flag;
  int32_t* clist;     // [CL_MAX]
};

// The CTA's work, decoded once by every thread before the register split and
// kept in shared memory: the roles read it back after the split, so no value
// computed before it has to live across it.
struct Work2 {
  int b, kvh, rtA, hasB, split, skip, j0, nt;
  int n0, n1, L;        // UnitTiles of the unit
  int list_in_smem;     // sparse chunk list copied to Shared2::clist
  int tail;             // index of a tail split CTA (AttnParams::tail_k), else -1
  uint32_t tmem;        // tensor-memory base
};
constexpr uint32_t OFF_WORK2 = 160;  // inside the barrier area, after the barriers
static_assert(NUM_BARS2 * 8 + 8 <= (int)OFF_WORK2 && OFF_WORK2 + sizeof(Work2) <= 256, "barrier area");

__device__ __forceinline__ uint8_t* smem_base2() {
  extern __shared__ uint8_t smem_raw[];
  return reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
}

__device__ __forceinline__ Shared2 shared2(uint8_t* smem) {
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + OFF_BAR2);
  Shared2 sh;
  sh.q_full = bars;
  sh.full = bars + 1;
  sh.empty = sh.full + NSLOT2;
  sh.s_full = sh.empty + NSLOT2;
  sh.p_full = sh.s_full + 2;
  sh.o_final = sh.p_full + 2;
  sh.drain = sh.o_final + 2;
  sh.tmem_slot = reinterpret_cast<uint32_t*>(sh.drain + 1);
  sh.abort_flag = reinterpret_cast<volatile int*>(sh.tmem_slot + 1);
  sh.clist = reinterpret_cast<int32_t*>(smem + OFF_CL2);
  return sh;
}

// Reads the work record (after the register split: the asm barrier orders
// the loads after it).
__device__ __forceinline__ Work2 load_work2(uint8_t* smem) {
  asm volatile("" ::: "memory");
  const volatile Work2* w = reinterpret_cast<const volatile Work2*>(smem + OFF_BAR2 + OFF_WORK2);
  Work2 r;
  r.b = w->b; r.kvh = w->kvh; r.rtA = w->rtA; r.hasB = w->hasB; r.split = w->split; r.skip = w->skip;
  r.j0 = w->j0; r.nt = w->nt; r.n0 = w->n0; r.n1 = w->n1; r.L = w->L; r.list_in_smem = w->list_in_smem;
  r.tail = w->tail;
  r.tmem = w->tmem;
  return r;
}

__device__ __forceinline__ const int32_t* unit_list(const AttnParams& p, const Work2& w, const Shared2& sh) {
  if (!p.src.chunk_idx) return nullptr;
  return w.list_in_smem ? sh.clist : p.src.chunk_idx + ((size_t)w.b * p.Hkv + w.kvh) * p.src.topk;
}

__device__ __forceinline__ bool wait2(uint64_t* bar, uint32_t parity, const Shared2& sh, int32_t* status,
                                      bool honour_abort = true) {
  return bounded_wait(bar, parity, sh.abort_flag, status, honour_abort);
}
// Whole-warp wait: the warp agrees on the outcome before any collective.
__device__ __forceinline__ bool wait2_warp(uint64_t* bar, uint32_t parity, const Shared2& sh, int32_t* status) {
  return __all_sync(0xffffffffu, wait2(bar, parity, sh, status));
}

__device__ __forceinline__ int slot2(int item) { return item % NSLOT2; }
__device__ __forceinline__ uint32_t use2(int item) { return (uint32_t)(item / NSLOT2); }

__device__ __forceinline__ void setmaxnreg_inc_softmax() {
  asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(REG_SOFTMAX) : "memory");
}
__device__ __forceinline__ void setmaxnreg_dec_other() {
  asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(REG_OTHER) : "memory");
}

// ------------------------------------------------------------- TMA producers
// kv = 0: Q of both tiles (once) and the K tiles; kv = 1: the V tiles.
__device__ __forceinline__ void producer_role(const CUtensorMap* tmQ, const CUtensorMap* tmKp,
                                              const CUtensorMap* tmVp, const CUtensorMap* tmKb,
                                              const CUtensorMap* tmVb, const AttnParams& p, int kv) {
  uint8_t* smem = smem_base2();
  const Shared2 sh = shared2(smem);
  const Work2 w = load_work2(smem);
  uint8_t* sQ = smem + OFF_Q2;
  uint8_t* sRing = smem + OFF_RING2;
  int32_t* status = p.dev_status;
  const UnitTiles u{w.n0, w.n1, w.L};
  const int32_t* clist = unit_list(p, w, sh);
  const uint64_t policy = p.kv_stream_once ? l2_policy_evict_first() : l2_policy_evict_normal();
  if (kv == 0) {
    mbar_arrive_expect_tx(sh.q_full, (w.hasB ? 2u : 1u) * Q_BYTES);
    for (int x = 0; x < (w.hasB ? 2 : 1); ++x) {
      const int t0 = (w.rtA + x) * (BM / p.G);
      tma_load_4d(sQ + x * Q_BYTES, tmQ, sh.q_full, 0, w.kvh * p.G, t0, w.b);
      tma_load_4d(sQ + x * Q_BYTES + BM * 128, tmQ, sh.q_full, 64, w.kvh * p.G, t0, w.b);
    }
  }
  int issued = 0;  // tiles whose item this producer has issued
  for (int jj = 0; jj < w.nt; ++jj) {
    const Tile t = tile_at(p, u, clist, w.j0 + jj);
    const int item = 2 * jj + kv;
    const int sl = slot2(item);
    if (!wait2(&sh.empty[sl], (use2(item) & 1) ^ 1, sh, status)) break;
    issued = jj + 1;
#ifdef FB_TEST_HOOKS
    if (p.test_skip_k1 && kv == 0 && jj == 1) continue;  // never loaded: its wait runs out
#endif
    mbar_arrive_expect_tx(&sh.full[sl], SLOT_BYTES);
    load_kv_tile(sRing + sl * SLOT_BYTES, kv ? tmVp : tmKp, kv ? tmVb : tmKb, &sh.full[sl], p, u, t, w.b, w.kvh,
                 policy);
  }
  // After an abort, let the copies in flight land before the CTA exits (this
  // producer's own: its last three items at most).
  if (*sh.abort_flag) {
    if (kv == 0) wait2(sh.q_full, 0, sh, nullptr, false);
    for (int jj = max(0, issued - (NSLOT2 + 1) / 2); jj < issued; ++jj) {
#ifdef FB_TEST_HOOKS
      if (p.test_skip_k1 && kv == 0 && jj == 1) continue;
#endif
      const int item = 2 * jj + kv;
      wait2(&sh.full[slot2(item)], use2(item) & 1, sh, nullptr, false);
    }
  }
}

// ---------------------------------------------------------------- MMA issuer
// The whole warp runs the issue loop (warp-uniform indices and descriptors);
// one elected lane issues each group of tcgen05.mma and its commits.
__device__ __forceinline__ void mma_role(const AttnParams& p) {
  constexpr int NC = BN;
  constexpr uint32_t IDESC_PV = idesc_bf16_f32(BM, HD, false, true);
  constexpr uint32_t IDESC_QK_FULL = idesc_bf16_f32(BM, NC, false, false);
  uint8_t* smem = smem_base2();
  const Shared2 sh = shared2(smem);
  const Work2 w = load_work2(smem);
  uint8_t* sRing = smem + OFF_RING2;
  int32_t* status = p.dev_status;
  const int lane = threadIdx.x & 31;
  const UnitTiles u{w.n0, w.n1, w.L};
  const int32_t* clist = unit_list(p, w, sh);
  const bool hasB = w.hasB != 0;
  const int nt = w.nt;
  // Shared-memory descriptors: an operand at byte offset `off` from its base
  // is the base descriptor plus off >> 4.
  const uint64_t dQ = sw128_desc(smem_u32(smem + OFF_Q2), 16, 1024);
  const uint64_t dK = sw128_desc(smem_u32(sRing), 16, 1024);
  const uint64_t dV = sw128_desc(smem_u32(sRing), HALF_BYTES, 1024);
  const bool leader = elect_one_sync();
  // QK^T of tile x: N = (valid keys rounded up to 16) on a tail tile
  auto issue_qk = [&](int x, int jj, int nvalid) {
    const uint32_t idesc =
        nvalid >= NC ? IDESC_QK_FULL : idesc_bf16_f32(BM, min(NC, (nvalid + 15) & ~15), false, false);
    const uint64_t dq = dQ + ((x * Q_BYTES) >> 4);
    const uint64_t dk = dK + ((slot2(2 * jj) * SLOT_BYTES) >> 4);
    const uint32_t tS = w.tmem + (uint32_t)x * BN;
    if (leader) {
#pragma unroll
      for (int kk = 0; kk < HD / 16; ++kk) {
        const uint32_t off = ((kk >> 2) * HALF_BYTES + (kk & 3) * 32) >> 4;
        umma_bf16_ss(tS, dq + off, dk + off, idesc, kk > 0);
      }
    }
  };
  // O_x += P_x V: as many 16-key steps as the tile has valid keys
  auto issue_pv = [&](int x, int jj, int nvalid) {
    const uint64_t dv = dV + ((slot2(2 * jj + 1) * SLOT_BYTES) >> 4);
    const uint32_t tP = w.tmem + (uint32_t)x * BN;
    const uint32_t tO = w.tmem + TMEM2_O + (uint32_t)x * BN;
    const int ksteps = (nvalid + 15) >> 4;
    if (leader) {
#pragma unroll
      for (int kk = 0; kk < NC / 16; ++kk)
        if (kk < ksteps)
          umma_bf16_ts(tO, tP + kk * 8, dv + ((kk * 16 * 128) >> 4), IDESC_PV, (jj > 0 || kk > 0) ? 1u : 0u);
    }
  };
  bool ok = wait2_warp(sh.q_full, 0, sh, status);
  if (ok && nt > 0) {
    Tile tc = tile_at(p, u, clist, w.j0);
    ok = wait2_warp(&sh.full[slot2(0)], 0, sh, status);
    if (ok) {
      tc_fence_after_sync();
      issue_qk(0, 0, tc.nvalid);
      if (leader) tc_commit(&sh.s_full[0]);
      if (hasB) {
        issue_qk(1, 0, tc.nvalid);
        if (leader) tc_commit(&sh.s_full[1]);
      }
      if (leader) tc_commit(&sh.empty[slot2(0)]);  // K(0) read by both QK^T
    }
    for (int jj = 0; ok && jj < nt; ++jj) {
      const bool last = jj + 1 == nt;
      const int iv = 2 * jj + 1;
      if (!(ok = wait2_warp(&sh.full[slot2(iv)], use2(iv) & 1, sh, status))) break;
      if (tc.seg == 0 && (tc.nvalid & 15)) {
        // Cache rows past the prefix may hold anything (even NaN); P is 0
        // there but 0 * NaN is not, so clear the V rows up to the next 16-key
        // step that PV reads (at most 15 rows, once per unit).
        uint8_t* dVs = sRing + slot2(iv) * SLOT_BYTES;
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
      // PV_A(j), then QK_A(j + 1): the softmax of A(j + 1) starts while the
      // pipe runs PV_B(j) and QK_B(j + 1)
      if (!(ok = wait2_warp(&sh.p_full[0], jj & 1, sh, status))) break;
      tc_fence_after_sync();
      issue_pv(0, jj, tc.nvalid);
      if (last && leader) tc_commit(&sh.o_final[0]);
      Tile tn = tc;
      const int ik = 2 * (jj + 1);
      if (!last) {
        tn = tile_at(p, u, clist, w.j0 + jj + 1);
        if (!(ok = wait2_warp(&sh.full[slot2(ik)], use2(ik) & 1, sh, status))) break;
        tc_fence_after_sync();
        issue_qk(0, jj + 1, tn.nvalid);
        if (leader) tc_commit(&sh.s_full[0]);
      }
      if (hasB) {
        if (!(ok = wait2_warp(&sh.p_full[1], jj & 1, sh, status))) break;
        tc_fence_after_sync();
        issue_pv(1, jj, tc.nvalid);
        if (last && leader) tc_commit(&sh.o_final[1]);
      }
      if (leader) tc_commit(&sh.empty[slot2(iv)]);  // V(j) read by both PV
      if (!last) {
        if (hasB) {
          issue_qk(1, jj + 1, tn.nvalid);
          if (leader) tc_commit(&sh.s_full[1]);
        }
        if (leader) tc_commit(&sh.empty[slot2(ik)]);  // K(j + 1) read by both QK^T
      }
      tc = tn;
    }
  }
  // Drain every MMA this warp issued before TMEM can be released.
  if (leader) tc_commit(sh.drain);
  __syncwarp();
  wait2(sh.drain, 0, sh, status, false);
}

// ------------------------------------------------------ softmax + epilogue
// Warpgroup x (0: tile A, 1: tile B); thread r owns query row r (TMEM lane r).
template <int EPI>
__device__ __forceinline__ void softmax_role(const CUtensorMap* tmO, const CUtensorMap* tmT, const AttnParams& p,
                                             int x) {
  constexpr int NC = BN;
  uint8_t* smem = smem_base2();
  const Shared2 sh = shared2(smem);
  const Work2 w = load_work2(smem);
  int32_t* status = p.dev_status;
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const UnitTiles u{w.n0, w.n1, w.L};
  const int32_t* clist = unit_list(p, w, sh);
  const int nt = w.nt;
  const int r = (warp & 3) * 32 + lane;
  const uint32_t lane_off = (uint32_t)((warp & 3) * 32) << 16;
  const uint32_t tS = w.tmem + (uint32_t)x * BN + lane_off;
  const uint32_t tO = w.tmem + TMEM2_O + (uint32_t)x * BN + lane_off;
  const float c2 = p.scale_log2;
  const int rt = w.rtA + x;
  const int pr = rt * BM + r;
  const int tok = pr / p.G;
  const int h = w.kvh * p.G + (pr - tok * p.G);
  // cached LSE of this row, read before the key loop so its latency hides
  const float lp_nat = (EPI == EPI_MERGE && tok < p.S) ? p.pre_lse[((size_t)w.b * p.Hq + h) * p.S + tok]
                                                        : -CUDART_INF_F;
  float m_run = -CUDART_INF_F;
  float l_run = 0.f;
  bool ok = true;
  for (int jj = 0; ok && jj < nt; ++jj) {
    const Tile t = tile_at(p, u, clist, w.j0 + jj);
    if (!(ok = wait2_warp(&sh.s_full[x], jj & 1, sh, status))) break;
    tc_fence_after_sync();
    // S row of this thread; columns past a tail tile's keys are -inf
    uint32_t sv[NC];
#pragma unroll
    for (int c = 0; c < NC / 32; ++c) tmem_ld_32x32(tS + c * 32, *reinterpret_cast<uint32_t(*)[32]>(&sv[c * 32]));
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
    mx0 = fmax3(mx0, mx1, fmaxf(s[NC - 2], s[NC - 1]));
    const float mt = mx0 * c2;
    const bool need = mt > m_run + RESCALE_LOG2;
    const float m_new = need ? mt : m_run;
    const float alpha = ex2_approx(m_run - m_new);  // 0 when m_run = -inf
    const float m_use = (m_new == -CUDART_INF_F) ? 0.f : m_new;
    // p = 2^(s * c2 - m): three of every four pairs through MUFU.EX2, one
    // through the FMA-pipe polynomial
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
      if (c == NC / 2 - 8) {
        // P of the first 64 keys (bf16 pairs over the first 32 columns of
        // S_X) stored while the second half's exponentials run
        uint32_t pk[32];
#pragma unroll
        for (int i = 0; i < 32; ++i) pk[i] = pack_bf16x2(s[2 * i], s[2 * i + 1]);
        tmem_st_32x32(tS, pk);
      }
    }
    l_run = l_run * alpha + ((la.x + la.y) + (lb.x + lb.y));
    m_run = m_new;
    if (jj > 0 && __any_sync(0xffffffffu, need)) {
      // Rows whose max moved rescale O_X: PV_X(j - 1) is done, because S_X(j)
      // was signalled after it.
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
    // P as bf16 pairs over the first 64 columns of S_X: the A operand of PV
    {
      // P of the last 64 keys: the A operand of PV is the first 64 columns of S_X
      uint32_t pk[32];
#pragma unroll
      for (int i = 0; i < 32; ++i) pk[i] = pack_bf16x2(s[NC / 2 + 2 * i], s[NC / 2 + 2 * i + 1]);
      tmem_st_32x32(tS + 32, pk);
    }
    tmem_st_wait();
    tc_fence_before_sync();
    __syncwarp();
    if (lane == 0) mbar_arrive(&sh.p_full[x]);
  }
  if (ok && nt > 0) {
    ok = wait2_warp(&sh.o_final[x], 0, sh, status);
    tc_fence_after_sync();
  }
  // The output is staged in Q_X's region: its last reader, QK^T of the last
  // key tile, is done once the last PV_X is (and with no key tile, once Q
  // has landed).
  if (ok) ok = wait2_warp(sh.q_full, 0, sh, status);
  // -------------------------------------------------------------- epilogue
  const bool row_ok = ok && tok < p.S;
  const bool empty = (nt == 0) || !(l_run > 0.f);
  const float inv_l = empty ? 0.f : 1.f / l_run;
  const float lse2 = empty ? -CUDART_INF_F : m_run + log2f(l_run);  // log2 of Z
  uint32_t ov[HD];
  if (nt > 0 && ok) {
#pragma unroll
    for (int c = 0; c < HD / 32; ++c) tmem_ld_32x32(tO + c * 32, *reinterpret_cast<uint32_t(*)[32]>(&ov[c * 32]));
    tmem_ld_wait();
  } else {
#pragma unroll
    for (int i = 0; i < HD; ++i) ov[i] = 0u;
  }
  uint8_t* stage = smem + OFF_Q2 + x * Q_BYTES;
  const uint32_t st_row = smem_u32(stage) + r * 128;
  const int t0 = rt * (BM / p.G);
  const bool store = ok && t0 < p.S;  // rows of this tile exist
  if (EPI == EPI_PARTIAL || w.tail >= 0) {
    // the f32 tile (64 KB) in two rounds of 64 columns through the 32 KB stage
    // (a tail split of the uncached pass or of the step writes its partial
    // rows the same way; the combine does the rest)
#pragma unroll
    for (int hf = 0; hf < 2; ++hf) {
      if (ok) {
#pragma unroll
        for (int cc = 0; cc < 2; ++cc)
#pragma unroll
          for (int ch = 0; ch < 8; ++ch) {
            const int i = (2 * hf + cc) * 32 + ch * 4;
            st_shared_v4(st_row + cc * (BM * 128) + ((ch ^ (r & 7)) << 4),
                         __float_as_uint(__uint_as_float(ov[i]) * inv_l),
                         __float_as_uint(__uint_as_float(ov[i + 1]) * inv_l),
                         __float_as_uint(__uint_as_float(ov[i + 2]) * inv_l),
                         __float_as_uint(__uint_as_float(ov[i + 3]) * inv_l));
          }
      }
      fence_proxy_async_smem();
      named_bar_sync(1 + x, 4 * 32);
      if (r == 0 && store && !*sh.abort_flag) {
#pragma unroll
        for (int cc = 0; cc < 2; ++cc) {
          if (w.tail >= 0)  // a tail split: the tile's slot of tail_o
            tma_store_4d(tmT, stage + cc * (BM * 128), (2 * hf + cc) * 32, 0, 0, 2 * w.tail + x);
          else
            tma_store_4d(tmO, stage + cc * (BM * 128), (2 * hf + cc) * 32, w.kvh * p.G, t0, w.split * p.B + w.b);
        }
        tma_store_commit();
        tma_store_wait_read();
      }
      named_bar_sync(1 + x, 4 * 32);  // the stage may be written again
    }
    if (w.tail >= 0) {
      if (ok) p.tail_lse[(size_t)(2 * w.tail + x) * BM + r] = lse2 * LN2;  // slot layout: every row
    } else if (row_ok) {
      p.out_lse[(((size_t)w.split * p.B + w.b) * p.Hq + h) * p.S + tok] = lse2 * LN2;
    }
  } else {
    const size_t orow = ((size_t)w.b * p.S + tok) * p.Hq + h;
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
#pragma unroll
          for (int i = 0; i < 32; i += 4) {
            const float4 q = *reinterpret_cast<const float4*>(pre + c * 32 + i);
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
      if (p.out_lse) p.out_lse[((size_t)w.b * p.Hq + h) * p.S + tok] = lse_out2 * LN2;
    }
    fence_proxy_async_smem();
    named_bar_sync(1 + x, 4 * 32);
    if (r == 0 && store && !*sh.abort_flag) {
#pragma unroll
      for (int hf = 0; hf < 2; ++hf) tma_store_4d(tmO, stage + hf * (BM * 128), hf * 64, w.kvh * p.G, t0, w.b);
      tma_store_commit();
      tma_store_wait_read();
    }
  }
}

template <int EPI>
__global__ void __launch_bounds__(THREADS2, 1)
    attn_tc2_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmKp,
                    const __grid_constant__ CUtensorMap tmVp, const __grid_constant__ CUtensorMap tmKb,
                    const __grid_constant__ CUtensorMap tmVb, const __grid_constant__ CUtensorMap tmO,
                    const __grid_constant__ CUtensorMap tmT, const AttnParams p) {
  uint8_t* smem = smem_base2();
  const Shared2 sh = shared2(smem);
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    mbar_init(sh.q_full, 1);
    for (int i = 0; i < NSLOT2; ++i) {
      mbar_init(&sh.full[i], 1);
      mbar_init(&sh.empty[i], 1);
    }
    for (int x = 0; x < 2; ++x) {
      mbar_init(&sh.s_full[x], 1);
      mbar_init(&sh.p_full[x], 4);
      mbar_init(&sh.o_final[x], 1);
    }
    mbar_init(sh.drain, 1);
    *sh.abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 9) {
    tmem_alloc(sh.tmem_slot, TMEM2_COLS);
    tmem_relinquish();
  }
  if (warp == 8 && lane == 0) {
    // tensor maps are kernel parameters: fetch them while the previous kernel finishes
    tma_prefetch_map(&tmQ);
    tma_prefetch_map(&tmKp);
    tma_prefetch_map(&tmVp);
    tma_prefetch_map(&tmKb);
    tma_prefetch_map(&tmVb);
    tma_prefetch_map(&tmO);
    if (p.tail_k > 0) tma_prefetch_map(&tmT);
  }
  {
    // This CTA's (b, kv head, query-tile pair, key split) from its grid index.
    const int npair = (p.n_rt + 1) >> 1;
    unsigned bid = blockIdx.x;
    int split, nsplit = p.nsplit, tail = -1;
    if (p.tail_k > 0 && bid >= (unsigned)p.tail_u0) {
      // a key split of one of the last units (the tail wave)
      tail = (int)(bid - (unsigned)p.tail_u0);
      split = tail % p.tail_k;
      nsplit = p.tail_k;
      bid = (unsigned)p.tail_u0 + (unsigned)(tail / p.tail_k);
    } else {
      split = (int)(bid % (unsigned)p.nsplit);
      bid /= (unsigned)p.nsplit;
    }
    const int pair = (int)(bid % (unsigned)npair);
    bid /= (unsigned)npair;
    const int kvh = (int)(bid % (unsigned)p.Hkv);
    const int b = (int)(bid / (unsigned)p.Hkv);

    // Everything above touches no global memory; from here on inputs may
    // come from the previous kernel in the stream.
    pdl_wait();
    pdl_launch_dependents();

    const bool skip = p.unit_mask != nullptr && p.unit_mask[b * p.Hkv + kvh] == 0;
    UnitTiles u{0, 0, 0};
    if (!skip) u = unit_tiles(p, b, kvh, threadIdx.x == 0);
    // the unit's sparse chunk list, copied to shared memory when it fits
    const bool list_in_smem = p.src.chunk_idx != nullptr && p.src.topk <= CL_MAX;
    if (list_in_smem && !skip) {
      const int32_t* g = p.src.chunk_idx + ((size_t)b * p.Hkv + kvh) * p.src.topk;
      for (int i = threadIdx.x; i < p.src.topk; i += THREADS2) sh.clist[i] = g[i];
    }
    if (threadIdx.x == 0) {
      const int ntot = u.n0 + u.n1;
      Work2* wk = reinterpret_cast<Work2*>(smem + OFF_BAR2 + OFF_WORK2);
      wk->b = b;
      wk->kvh = kvh;
      wk->rtA = 2 * pair;
      wk->hasB = 2 * pair + 1 < p.n_rt;  // the last pair of an odd tile count has one tile
      wk->split = split;
      wk->skip = skip;
      // split * ntot < 2^7 * 2^23: 32-bit arithmetic is exact
      const int j0 = (int)(((unsigned)split * (unsigned)ntot) / (unsigned)nsplit);
      const int j1 = (int)(((unsigned)(split + 1) * (unsigned)ntot) / (unsigned)nsplit);
      wk->j0 = j0;
      wk->nt = j1 - j0;
      wk->n0 = u.n0;
      wk->n1 = u.n1;
      wk->L = u.L;
      wk->list_in_smem = list_in_smem;
      wk->tail = tail;
      wk->tmem = *sh.tmem_slot;
    }
  }
  tc_fence_before_sync();
  __syncthreads();
  tc_fence_after_sync();

  if (warp >= 8) {
    setmaxnreg_dec_other();
    const bool skip = load_work2(smem).skip != 0;
    if (!skip && (warp == 8 || warp == 10) && lane == 0)
      producer_role(&tmQ, &tmKp, &tmVp, &tmKb, &tmVb, p, warp == 10 ? 1 : 0);
    else if (!skip && warp == 9)
      mma_role(p);
  } else {
    setmaxnreg_inc_softmax();
    const Work2 w = load_work2(smem);
    const int x = warp >> 2;  // 0: tile A, 1: tile B
    if (!w.skip && (x == 0 || w.hasB)) softmax_role<EPI>(&tmO, &tmT, p, x);
  }

  tc_fence_before_sync();
  __syncthreads();
  if (warp == 9) {
    tc_fence_after_sync();
    tmem_dealloc(load_work2(smem).tmem, TMEM2_COLS);
  }
}

}  // namespace

size_t tc2_smem_bytes() { return SMEM2_BYTES; }

cudaError_t launch_attn_tc2(const AttnParams& p, const CUtensorMap& tmQ, const CUtensorMap& tmKp,
                            const CUtensorMap& tmVp, const CUtensorMap& tmKb, const CUtensorMap& tmVb,
                            const CUtensorMap& tmO, const CUtensorMap& tmT, int grid, cudaStream_t stream) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  int which;
  void (*kern)(CUtensorMap, CUtensorMap, CUtensorMap, CUtensorMap, CUtensorMap, CUtensorMap, CUtensorMap,
               AttnParams);
  if (p.epi == EPI_PARTIAL) {
    kern = attn_tc2_kernel<EPI_PARTIAL>;
    which = 0;
  } else if (p.epi == EPI_MERGE) {
    kern = attn_tc2_kernel<EPI_MERGE>;
    which = 1;
  } else {
    kern = attn_tc2_kernel<EPI_NORM>;
    which = 2;
  }
  // Set once per device and kernel.  The register split needs the kernel to
  // be launched with exactly REG_LAUNCH registers per thread (setmaxnreg.inc
  // draws on the registers the CTA was launched with): checked here before
  // the first launch.
  static std::atomic<bool> configured[64][3];
  if (dev >= 64 || !configured[dev][which].load(std::memory_order_acquire)) {
    cudaFuncAttributes fa;
    e = cudaFuncGetAttributes(&fa, kern);
    if (e != cudaSuccess) return e;
    if (fa.numRegs != (int)REG_LAUNCH) return cudaErrorInvalidConfiguration;
    e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)SMEM2_BYTES);
    if (e != cudaSuccess) return e;
    if (dev < 64) configured[dev][which].store(true, std::memory_order_release);
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)grid);
  cfg.blockDim = dim3(THREADS2);
  cfg.dynamicSmemBytes = SMEM2_BYTES;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  e = cudaLaunchKernelEx(&cfg, kern, tmQ, tmKp, tmVp, tmKb, tmVb, tmO, tmT, p);
  note_launch();
  return e != cudaSuccess ? e : cudaGetLastError();
}

}  // namespace fb
