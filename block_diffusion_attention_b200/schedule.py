"""One attention layer's FlashBlock state on one GPU, driven through the C ABI.

``CachedBlockAttention`` owns the device buffers of a layer -- the KV cache
(contiguous or paged), the prefix lengths, the cached block-external pair
(O_pre, LSE_pre), the split workspace, the sparse-prefix chunk means and
chunk list -- and exposes the calls of one block of denoising steps:

    refresh(Q)            prefix partial with this step's queries (refresh step)
    adapt(Q, Kblk, Vblk)  policy mode: refresh mask, then the masked prefix partial
    step(Q, Kblk, Vblk)   in-block partial merged with the cached pair -> O
    step_append(...)      the block's last step and its append in one call
    full(Q, Kblk, Vblk)   uncached attention over [prefix ; block] -> O
    append(Kblk, Vblk)    finalized block joins the cache

Each call is one or two C-ABI calls on the current CUDA stream; PyTorch only
allocates the buffers.
"""
from __future__ import annotations

from typing import Optional

import torch

from . import flashblock as fbl


class CachedBlockAttention:
    def __init__(self, batch: int, num_q_heads: int, num_kv_heads: int, head_dim: int, block_len: int,
                 capacity: int, dtype: str = "bf16", softmax_scale: float = 1.0, page_size: int = 0,
                 block_table: Optional[torch.Tensor] = None, num_pages: int = 0,
                 chunk_size: int = 0, topk: int = 0, num_splits: int = 0, residual: bool = False,
                 policy: Optional[str] = None, gamma: float = 0.9, tau: int = 1, eps: float = 0.25,
                 device="cuda"):
        self.device = torch.device(device)
        self.tdtype = torch.bfloat16 if dtype == "bf16" else torch.float32
        self.B, self.Hq, self.Hkv, self.D, self.S = batch, num_q_heads, num_kv_heads, head_dim, block_len
        self.page_size = page_size
        self.chunk_size, self.topk = chunk_size, topk
        dev = self.device
        if page_size > 0:
            assert block_table is not None and num_pages > 0
            self.block_table = block_table.to(dev, torch.int32).contiguous()
            self.max_pages = self.block_table.shape[1]
            self.num_pages = num_pages
            cache_shape = (num_pages, page_size, num_kv_heads, head_dim)
            self.capacity = self.max_pages * page_size
        else:
            self.block_table = None
            self.max_pages = self.num_pages = 0
            cache_shape = (batch, capacity, num_kv_heads, head_dim)
            self.capacity = capacity
        self.K = torch.zeros(cache_shape, dtype=self.tdtype, device=dev)
        self.V = torch.zeros(cache_shape, dtype=self.tdtype, device=dev)
        self.lens = torch.zeros(batch, dtype=torch.int32, device=dev)
        self.desc = fbl.make_desc(
            batch, num_q_heads, num_kv_heads, head_dim, block_len,
            dtype=fbl.FB_BF16 if dtype == "bf16" else fbl.FB_FP32, softmax_scale=softmax_scale,
            kv_capacity=self.capacity if page_size == 0 else 0, page_size=page_size,
            max_pages=self.max_pages, num_pages=self.num_pages, block_table=self.block_table,
            prefix_lens=self.lens, chunk_size=chunk_size, topk=topk, num_splits=num_splits)
        self.residual = residual and topk > 0
        self.O_pre = torch.empty((batch, block_len, num_q_heads, head_dim), dtype=torch.float32, device=dev)
        self.LSE_pre = torch.empty((batch, num_q_heads, block_len), dtype=torch.float32, device=dev)
        self.LSE = torch.empty((batch, num_q_heads, block_len), dtype=torch.float32, device=dev)
        ws = fbl.fb_workspace_bytes(self.desc)
        if self.residual:
            # residual mode: the complement list is a chunk list of up to every chunk
            nch = -(-self.capacity // chunk_size)
            self.desc_res = fbl.make_desc(
                batch, num_q_heads, num_kv_heads, head_dim, block_len,
                dtype=self.desc.dtype, softmax_scale=softmax_scale,
                kv_capacity=self.desc.kv_capacity, page_size=page_size, max_pages=self.max_pages,
                num_pages=self.num_pages, block_table=self.block_table, prefix_lens=self.lens,
                chunk_size=chunk_size, topk=nch, num_splits=num_splits)
            ws = max(ws, fbl.fb_workspace_bytes(self.desc_res))
            self.comp_idx = torch.full((batch, num_kv_heads, nch), -1, dtype=torch.int32, device=dev)
            shape_o = (batch, block_len, num_q_heads, head_dim)
            shape_l = (batch, num_q_heads, block_len)
            self.O_res = torch.empty(shape_o, dtype=torch.float32, device=dev)
            self.LSE_res = torch.empty(shape_l, dtype=torch.float32, device=dev)
            self.O_sel = torch.empty(shape_o, dtype=torch.float32, device=dev)
            self.LSE_sel = torch.empty(shape_l, dtype=torch.float32, device=dev)
        # adaptive reuse: a policy decides at every step which units refresh
        assert policy in (None, "headwise", "threshold")
        assert policy is None or (topk == 0 and not residual), "refresh policies use the dense prefix"
        self.policy, self.gamma, self.tau, self.eps = policy, gamma, tau, eps
        if policy is not None:
            self.unit_mask = torch.ones((batch, num_kv_heads), dtype=torch.int32, device=dev)
        if policy == "headwise":
            self.Q_ref = torch.zeros((batch, block_len, num_q_heads, head_dim), dtype=self.tdtype, device=dev)
            self.sim = torch.zeros((batch, num_kv_heads), dtype=torch.float32, device=dev)
        elif policy == "threshold":
            self.K_prev = torch.zeros((batch, block_len, num_kv_heads, head_dim), dtype=self.tdtype, device=dev)
            self.V_prev = torch.zeros_like(self.K_prev)
            self.updated = torch.zeros(batch, dtype=torch.int32, device=dev)
        self.workspace = torch.empty(max(ws, 16) // 4 + 4, dtype=torch.float32, device=dev) if ws else None
        self.status = torch.zeros(1, dtype=torch.int32, device=dev)
        if topk > 0:
            nch = -(-self.capacity // chunk_size)
            self.Kmean = torch.zeros((batch, num_kv_heads, nch, head_dim), dtype=torch.float32, device=dev)
            self.chunk_idx = torch.full((batch, num_kv_heads, topk), -1, dtype=torch.int32, device=dev)
        else:
            self.Kmean = self.chunk_idx = None

    # ------------------------------------------------------------------ state
    def load_prefix(self, K: torch.Tensor, V: torch.Tensor, lens) -> None:
        """Place a contiguous prefix [B, rows, Hkv, D] into the cache (rows >= lens are ignored)."""
        lens = [int(x) for x in lens]
        if self.page_size == 0:
            n = min(K.shape[1], self.capacity)
            self.K[:, :n].copy_(K[:, :n])
            self.V[:, :n].copy_(V[:, :n])
        else:
            ps = self.page_size
            bt = self.block_table.cpu()
            for b in range(self.B):
                for p in range(-(-lens[b] // ps)):
                    lo, hi = p * ps, min((p + 1) * ps, K.shape[1])
                    pg = int(bt[b, p])
                    self.K[pg, :hi - lo].copy_(K[b, lo:hi])
                    self.V[pg, :hi - lo].copy_(V[b, lo:hi])
        self.lens.copy_(torch.tensor(lens, dtype=torch.int32))
        if self.topk > 0:
            self.update_chunk_means(0, -(-self.capacity // self.chunk_size))

    def update_chunk_means(self, c0: int, c1: int) -> None:
        fbl.fb_chunk_means(self.desc, self.K, c0, c1, self.Kmean, self.status)

    # ------------------------------------------------------------------ steps
    def refresh(self, Q: torch.Tensor) -> None:
        """Refresh step: recompute the cached block-external pair with Q
        (``select`` then ``prefix``)."""
        self.select(Q)
        self.prefix(Q)

    def select(self, Q: torch.Tensor) -> None:
        """Sparse prefix: pick this refresh's chunks (and, in residual mode,
        their complement).  Nothing to do for a dense prefix."""
        if self.topk > 0:
            fbl.fb_select_chunks(self.desc, Q, self.Kmean, self.chunk_idx, self.status)
        if self.residual:
            cap = self.comp_idx.shape[2]
            fbl.fb_complement_chunks(self.desc, self.chunk_idx, self.comp_idx, cap, self.status)

    def prefix(self, Q: torch.Tensor) -> None:
        """The prefix partial of a refresh (after ``select``): over the whole
        prefix or the selected chunks into (O_pre, LSE_pre); in residual mode
        over the chunks left out, into the cached residual (the selected
        chunks are recomputed at every step)."""
        if self.residual:
            fbl.fb_prefix_partial(self.desc_res, Q, self.K, self.V, self.comp_idx, self.O_res, self.LSE_res,
                                  self.workspace, self.status)
            return
        fbl.fb_prefix_partial(self.desc, Q, self.K, self.V, self.chunk_idx if self.topk > 0 else None,
                              self.O_pre, self.LSE_pre, self.workspace, self.status)

    def adapt(self, Q, Kblk, Vblk, first: bool) -> None:
        """Adaptive refresh (policy mode): decide per unit whether the cached
        pair is recomputed at this step, then recompute the chosen units.  The
        first step of a block refreshes every unit."""
        if self.policy == "headwise":
            fbl.fb_headwise_refresh_mask(self.desc, Q, self.Q_ref, float("inf") if first else self.gamma,
                                         self.unit_mask, self.sim)
        else:
            fbl.fb_threshold_refresh_mask(self.desc, self.K_prev, self.V_prev, Kblk, Vblk, self.eps,
                                          0 if first else self.tau, self.unit_mask, self.updated,
                                          self.workspace)
        fbl.fb_prefix_partial_masked(self.desc, Q, self.K, self.V, None, self.unit_mask, self.O_pre,
                                     self.LSE_pre, self.workspace, self.status)

    def cached_step(self, s: int, Q, Kblk, Vblk, refresh_steps=(0,), out: Optional[torch.Tensor] = None,
                    lse: bool = False, append: bool = False, advance: bool = True):
        """Step s of a block: the refresh its schedule (or policy) asks for,
        then the fused step (with ``append``: the block's last step, which
        also appends this step's K/V -- see ``step_append``)."""
        if self.policy is not None:
            self.adapt(Q, Kblk, Vblk, first=(s == 0))
        elif s in refresh_steps:
            self.refresh(Q)
        if append:
            return self.step_append(Q, Kblk, Vblk, out=out, lse=lse, advance=advance)
        return self.step(Q, Kblk, Vblk, out=out, lse=lse)

    def _residual_merge(self, Q) -> None:
        # residual mode: the cached residual merged with a fresh partial over
        # the selected chunks (three partials in all, with the step's own)
        fbl.fb_prefix_partial(self.desc, Q, self.K, self.V, self.chunk_idx, self.O_sel, self.LSE_sel,
                              self.workspace, self.status)
        fbl.fb_merge_partials(self.desc, self.O_res, self.LSE_res, self.O_sel, self.LSE_sel,
                              self.O_pre, self.LSE_pre)

    def step(self, Q, Kblk, Vblk, out: Optional[torch.Tensor] = None, lse: bool = False):
        """Cached denoising step: O = merge(cached pair, in-block partial).

        Residual mode: the cached residual is first merged with a fresh
        partial over the selected chunks (three partials in all)."""
        if out is None:
            out = torch.empty_like(Q)
        if self.residual:
            self._residual_merge(Q)
        fbl.fb_block_step(self.desc, Q, Kblk, Vblk, self.O_pre, self.LSE_pre, out,
                          self.LSE if lse else None, self.status, workspace=self.workspace)
        return out

    def step_append(self, Q, Kblk, Vblk, out: Optional[torch.Tensor] = None, lse: bool = False,
                    advance: bool = True):
        """The last denoising step of a block together with the block's
        append (one kernel for short blocks): the same as ``step`` then
        ``append(Kblk, Vblk, advance)``."""
        if out is None:
            out = torch.empty_like(Q)
        if self.residual:
            self._residual_merge(Q)
        fbl.fb_block_step_append(self.desc, Q, Kblk, Vblk, self.O_pre, self.LSE_pre, out,
                                 self.LSE if lse else None, self.K, self.V, self.lens if advance else None,
                                 self.status, workspace=self.workspace)
        if advance and self.topk > 0:
            fbl.fb_chunk_means_tail(self.desc, self.K, self.S, self.Kmean, self.status)
        return out

    def full(self, Q, Kblk, Vblk, out: Optional[torch.Tensor] = None, lse: bool = False):
        """Uncached step: attention over [prefix ; block] in one pass."""
        if out is None:
            out = torch.empty_like(Q)
        fbl.fb_full_reference_gpu(self.desc, Q, self.K, self.V, Kblk, Vblk, out,
                                  self.LSE if lse else None, self.workspace, self.status)
        return out

    def append(self, Kblk, Vblk, advance: bool = True) -> None:
        """Block end: write the finalized block's K/V after the prefix and grow it.

        The prefix lengths live on the device: the append reads them, writes
        the rows and advances them, and (sparse prefix) the means of the
        chunks it touched are recomputed from the advanced device lengths, so
        no host round trip is needed and a recorded block replays correctly
        block after block.  ``advance=False`` writes the rows but keeps the
        prefix length (a benchmark holds its workload fixed this way)."""
        fbl.fb_kv_append(self.desc, Kblk, Vblk, self.K, self.V, self.lens if advance else None, self.status)
        if advance and self.topk > 0:
            fbl.fb_chunk_means_tail(self.desc, self.K, self.S, self.Kmean, self.status)

    # ------------------------------------------------------------ graphs
    def _issue_block(self, steps, outs, refresh_steps, append_kv, advance, cached, prologue=None, epilogue=None):
        # the block's append rides on its last cached step when it appends
        # that step's own K/V
        last = len(steps) - 1
        fuse = (cached and append_kv is not None and last >= 0 and append_kv[0] is steps[last][1]
                and append_kv[1] is steps[last][2])
        for s, (Q, Kb, Vb) in enumerate(steps):
            if prologue is not None:
                prologue(s)
            if cached:
                self.cached_step(s, Q, Kb, Vb, refresh_steps, out=outs[s], append=fuse and s == last,
                                 advance=advance)
            else:
                self.full(Q, Kb, Vb, out=outs[s])
            if epilogue is not None:
                epilogue(s)
        if append_kv is not None and not fuse:
            self.append(append_kv[0], append_kv[1], advance=advance)

    def run_block(self, steps, outs, refresh_steps, append_kv=None, advance=True, cached=True):
        """Issue one block of denoising steps: ``steps`` is a list of (Q, Kblk,
        Vblk) device tensors, ``outs`` the per-step outputs.  Cached: refresh at
        ``refresh_steps``, fused step everywhere; uncached: full attention at
        every step.  Ends with the append of ``append_kv`` when given (fused
        into the last cached step when it is that step's K/V)."""
        self._issue_block(steps, outs, refresh_steps, append_kv, advance, cached)

    def capture_block(self, steps, outs, refresh_steps, append_kv=None, cached=True, prologue=None,
                      epilogue=None, advance=True):
        """Record one block of calls (see ``run_block``) into a CUDA graph.

        The library's calls are capturable: they allocate nothing, never
        synchronise, and pass their TMA descriptors by value.  The block runs
        once eagerly first, so one-time kernel attribute settings happen
        outside the capture (that run is a real block: with ``advance`` it
        appends, and the prefix grows by one block).  The append is recorded
        with the device-side length update (``advance=True``): each replay
        appends after the current prefix and grows it, and the graph can be
        replayed for consecutive blocks once the next block's inputs are
        copied into the tensors it was recorded with.  ``prologue``/
        ``epilogue`` (callables) are recorded before/after each step, e.g.
        host<->device copies.  Returns the ``torch.cuda.CUDAGraph``.
        """
        def body():
            self._issue_block(steps, outs, refresh_steps, append_kv, advance, cached, prologue, epilogue)

        body()
        torch.cuda.synchronize()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            body()
        torch.cuda.synchronize()
        return g

    def check(self) -> None:
        """Synchronise and raise if a kernel recorded a device-side error."""
        torch.cuda.current_stream().synchronize()
        st = int(self.status.item())
        if st != 0:
            self.status.zero_()
            raise fbl.FlashBlockError("device", st)
