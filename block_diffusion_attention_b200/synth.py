"""Seeded synthetic inputs for the five attention workloads.

This module draws random numbers and lays them out; it holds none of the
attention arithmetic.  Both the CUDA tests/benchmark and the float64 oracle
read their inputs from here, so the two sides see the same values.

Workloads (one attention layer each):

* ``tiny_fp32``      B1, 1 head, D64, prefix 256, block 16, 4 steps, fp32.
* ``lm_gqa``         B1, 32 q / 8 kv heads, D128, block 32, prefix 8192,
                     8 steps per block, 4 consecutive blocks appended.
* ``long_ctx``       as ``lm_gqa`` with a 131072-token prefix, 1 block.
* ``video``          B1, 40 heads (MHA), D128, block 4680, prefix 32760,
                     4 steps, drift 0.1.
* ``batched_sparse`` B16, 32/8 heads, D128, block 64, varlen prefix uniform in
                     [16384, 32768], top-16 of 256-token chunks, refresh at
                     steps 0 and 4.

Value recipe: prefix K, V ~ N(0, 1); the block's base Q, K, V ~ N(0, 1) with Q
multiplied by ``q_std``; step s of a block uses base + N(0, drift^2) drawn
independently per step (not a random walk).  Every draw comes from
``numpy.random.default_rng([workload_id, block, step, tensor_id])``.
bf16 workloads round the float32 draws once to bf16 (round-to-nearest-even);
the oracle then reads exactly those rounded values, upcast to float64.
"""
from __future__ import annotations

import dataclasses
import math
from typing import Optional, Tuple

import numpy as np

# tensor ids of the seed tuple
T_Q, T_K, T_V, T_PREFIX_K, T_LENS, T_PREFIX_V, T_PAGES = 0, 1, 2, 3, 4, 5, 6
T_JUMP, T_UPDATE = 7, 8
BASE_STEP = 0xBA5E  # "step" slot of the seed tuple used for a block's base draw


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    wid: int                 # workload id, first element of every seed tuple
    batch: int
    num_q_heads: int
    num_kv_heads: int
    head_dim: int
    block_len: int           # S: tokens in the active block
    prefix_len: int          # L: prefix length (max of the varlen range)
    steps: int               # denoising steps per block
    blocks: int = 1          # consecutive blocks (each appended to the cache)
    dtype: str = "bf16"      # "bf16" or "fp32"
    q_std: float = 1.0
    drift: float = 0.05
    softmax_scale: float = 1.0
    refresh: Tuple[int, ...] = (0,)
    prefix_min: Optional[int] = None   # varlen: lengths ~ U[prefix_min, prefix_len]
    chunk_size: int = 256
    topk: int = 0            # 0 = dense prefix
    page_size: int = 0       # 0 = contiguous cache

    @property
    def group(self) -> int:
        return self.num_q_heads // self.num_kv_heads

    @property
    def capacity(self) -> int:
        """Cache rows per sequence: the longest prefix plus every appended block."""
        return self.prefix_len + self.blocks * self.block_len

    def scaled(self, **kw) -> "Workload":
        return dataclasses.replace(self, **kw)


WORKLOADS = {
    "tiny_fp32": Workload("tiny_fp32", 1, 1, 1, 1, 64, 16, 256, 4, dtype="fp32",
                          q_std=1.0, drift=0.05, softmax_scale=1.0 / 8.0, refresh=(0,)),
    "lm_gqa": Workload("lm_gqa", 2, 1, 32, 8, 128, 32, 8192, 8, blocks=4,
                       q_std=1.0 / math.sqrt(128), drift=0.05, softmax_scale=1.0),
    "long_ctx": Workload("long_ctx", 3, 1, 32, 8, 128, 32, 131072, 8,
                         q_std=1.0 / math.sqrt(128), drift=0.05, softmax_scale=1.0),
    "video": Workload("video", 4, 1, 40, 40, 128, 4680, 32760, 4,
                      q_std=1.0, drift=0.1, softmax_scale=1.0 / math.sqrt(128)),
    "batched_sparse": Workload("batched_sparse", 5, 16, 32, 8, 128, 64, 32768, 8,
                               q_std=1.0 / math.sqrt(128), drift=0.05, softmax_scale=1.0,
                               refresh=(0, 4), prefix_min=16384, chunk_size=256, topk=16),
}


def rng(w: Workload, block: int, step: int, tid: int) -> np.random.Generator:
    return np.random.default_rng([w.wid, block, step, tid])


def prefix_lens(w: Workload) -> np.ndarray:
    """Per-sequence prefix lengths [B] int32 (fixed, or uniform integers)."""
    if w.prefix_min is None:
        return np.full(w.batch, w.prefix_len, dtype=np.int32)
    r = rng(w, 0, 0, T_LENS)
    return r.integers(w.prefix_min, w.prefix_len, size=w.batch, endpoint=True).astype(np.int32)


def prefix_kv(w: Workload) -> Tuple[np.ndarray, np.ndarray, np.ndarray]:
    """Contiguous prefix cache K, V [B, capacity, Hkv, D] float32 plus lengths.

    Rows at and beyond a sequence's length are zero (room for appended blocks).
    """
    lens = prefix_lens(w)
    shape = (w.batch, w.capacity, w.num_kv_heads, w.head_dim)
    K = np.zeros(shape, dtype=np.float32)
    V = np.zeros(shape, dtype=np.float32)
    rk = rng(w, 0, 0, T_PREFIX_K)
    rv = rng(w, 0, 0, T_PREFIX_V)
    for b in range(w.batch):
        n = int(lens[b])
        K[b, :n] = rk.standard_normal((n, w.num_kv_heads, w.head_dim), dtype=np.float32)
        V[b, :n] = rv.standard_normal((n, w.num_kv_heads, w.head_dim), dtype=np.float32)
    return K, V, lens


def _block_shapes(w: Workload):
    q = (w.batch, w.block_len, w.num_q_heads, w.head_dim)
    kv = (w.batch, w.block_len, w.num_kv_heads, w.head_dim)
    return q, kv


def block_base(w: Workload, block: int):
    """Base Q, K, V of one block (float32)."""
    qs, kvs = _block_shapes(w)
    Q = rng(w, block, BASE_STEP, T_Q).standard_normal(qs, dtype=np.float32) * np.float32(w.q_std)
    K = rng(w, block, BASE_STEP, T_K).standard_normal(kvs, dtype=np.float32)
    V = rng(w, block, BASE_STEP, T_V).standard_normal(kvs, dtype=np.float32)
    return Q, K, V


def step_inputs(w: Workload, block: int, step: int, base=None, drift: Optional[float] = None,
                q_drift: bool = True):
    """Q_s, K_s, V_s of denoising step ``step``: base + independent N(0, drift^2).

    ``q_drift=False`` keeps the queries at their base values (the
    unchanged-query case); K and V still drift.
    """
    if base is None:
        base = block_base(w, block)
    sig = np.float32(w.drift if drift is None else drift)
    Q0, K0, V0 = base
    Q = Q0 + sig * rng(w, block, step, T_Q).standard_normal(Q0.shape, dtype=np.float32) if q_drift else Q0.copy()
    K = K0 + sig * rng(w, block, step, T_K).standard_normal(K0.shape, dtype=np.float32)
    V = V0 + sig * rng(w, block, step, T_V).standard_normal(V0.shape, dtype=np.float32)
    return Q, K, V


def headwise_steps(w: Workload, block: int, steps: int, p_jump: float = 0.35, rel_drift: float = 0.05,
                   base=None):
    """Steps for the head-wise reuse policy: per (b, kv head) unit, the
    queries either stay near their current values (independent
    N(0, (rel_drift * q_std)^2) noise per step) or, with probability p_jump at
    each step after the first, are redrawn as a whole (N(0, q_std^2)).  K and
    V drift as in ``step_inputs``.  Returns lists of float32 (Q, K, V)."""
    if base is None:
        base = block_base(w, block)
    Q0 = base[0]
    B, S, Hq, D = Q0.shape
    G = w.group
    cur = Q0.copy()
    out = []
    for s in range(steps):
        if s > 0:
            r = rng(w, block, s, T_JUMP)
            jump = r.random((B, w.num_kv_heads)) < p_jump
            fresh = r.standard_normal(Q0.shape, dtype=np.float32) * np.float32(w.q_std)
            for b in range(B):
                for kvh in range(w.num_kv_heads):
                    if jump[b, kvh]:
                        cur[b, :, kvh * G:(kvh + 1) * G] = fresh[b, :, kvh * G:(kvh + 1) * G]
        noise = rng(w, block, s, T_Q).standard_normal(Q0.shape, dtype=np.float32)
        Q = cur + np.float32(rel_drift * w.q_std) * noise
        _, K, V = step_inputs(w, block, s, base, q_drift=False)
        out.append((Q, K, V))
    return out


def threshold_steps(w: Workload, block: int, steps: int, max_updates: Optional[int] = None,
                    noise: float = 0.01, base=None):
    """Steps for the threshold reuse policy: at each step after the first,
    every sequence redraws the K and V (N(0, 1)) of a seeded number of its
    block tokens, uniform in [0, max_updates] (default S/2), chosen at
    random; all tokens also carry independent N(0, noise^2) noise per step.
    Queries drift as in ``step_inputs``.  Returns lists of float32 (Q, K, V)."""
    if base is None:
        base = block_base(w, block)
    Q0, K0, V0 = base
    B, S = K0.shape[0], K0.shape[1]
    top = S // 2 if max_updates is None else max_updates
    K, V = K0.copy(), V0.copy()
    out = []
    for s in range(steps):
        if s > 0:
            r = rng(w, block, s, T_UPDATE)
            n = r.integers(0, top, size=B, endpoint=True)
            for b in range(B):
                toks = r.choice(S, size=int(n[b]), replace=False)
                K[b, toks] = r.standard_normal((len(toks),) + K0.shape[2:], dtype=np.float32)
                V[b, toks] = r.standard_normal((len(toks),) + V0.shape[2:], dtype=np.float32)
        Q, _, _ = step_inputs(w, block, s, base)
        nk = rng(w, block, s, T_K).standard_normal(K0.shape, dtype=np.float32)
        nv = rng(w, block, s, T_V).standard_normal(V0.shape, dtype=np.float32)
        out.append((Q, K + np.float32(noise) * nk, V + np.float32(noise) * nv))
    return out


def page_table(w: Workload, page_size: int, lens_cap: Optional[int] = None):
    """A seeded page table for a paged copy of the cache.

    Returns (block_table [B, max_pages] int32, num_pages): sequence b's page p
    lives at pool page block_table[b, p]; pool pages are a random permutation
    so that neighbouring logical pages are not neighbours in memory.
    """
    cap = w.capacity if lens_cap is None else lens_cap
    max_pages = -(-cap // page_size)
    num_pages = w.batch * max_pages
    perm = rng(w, 0, 0, T_PAGES).permutation(num_pages).astype(np.int32)
    return perm.reshape(w.batch, max_pages), num_pages


def to_paged(cache: np.ndarray, table: np.ndarray, page_size: int) -> np.ndarray:
    """Scatter a contiguous cache [B, cap, H, D] into a page pool [P, page, H, D]."""
    B, cap, H, D = cache.shape
    max_pages = table.shape[1]
    pool = np.zeros((B * max_pages, page_size, H, D), dtype=cache.dtype)
    padded = np.zeros((B, max_pages * page_size, H, D), dtype=cache.dtype)
    padded[:, :cap] = cache
    for b in range(B):
        for p in range(max_pages):
            pool[table[b, p]] = padded[b, p * page_size:(p + 1) * page_size]
    return pool


def round_bf16(x: np.ndarray):
    """Round float32 values to bf16 once (RNE, via torch).

    Returns (torch bf16 CPU tensor, float64 numpy copy of the rounded values).
    """
    import torch
    t = torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32)).to(torch.bfloat16)
    return t, t.to(torch.float64).numpy()


def as_dtype(w: Workload, x: np.ndarray):
    """The workload's input dtype: (torch CPU tensor, float64 numpy of its values)."""
    import torch
    if w.dtype == "bf16":
        return round_bf16(x)
    t = torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32))
    return t, t.to(torch.float64).numpy()
