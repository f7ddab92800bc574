"""Shared driver of the GPU parity tests: runs one workload's cached and
uncached schedules through the C ABI and the float64 oracle on the same
seeded inputs, and compares them with the tolerances of the method's
precision (bf16 inputs with fp32 accumulation: max |diff| <= 2e-2 and
relative Frobenius error <= 1e-2; fp32 inputs: both <= 1e-5)."""
from __future__ import annotations

import numpy as np
import torch

from block_diffusion_attention_b200 import synth
from block_diffusion_attention_b200.schedule import CachedBlockAttention
from oracle import flashblock_oracle as ora

TOL = {"bf16": (2e-2, 1e-2), "fp32": (1e-5, 1e-5)}


def compare(name, got, ref, dtype):
    """max-abs and relative-Frobenius check; -inf entries must agree exactly."""
    atol, rtol = TOL[dtype]
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    assert got.shape == ref.shape, f"{name}: shape {got.shape} vs {ref.shape}"
    ninf_g, ninf_r = np.isneginf(got), np.isneginf(ref)
    assert np.array_equal(ninf_g, ninf_r), f"{name}: -inf pattern differs"
    g = np.where(ninf_r, 0.0, got)
    r = np.where(ninf_r, 0.0, ref)
    assert np.all(np.isfinite(g)), f"{name}: non-finite values"
    diff = np.abs(g - r)
    mx = float(diff.max()) if diff.size else 0.0
    den = float(np.linalg.norm(r))
    rel = float(np.linalg.norm(g - r)) / den if den > 0 else mx
    assert mx <= atol and rel <= rtol, f"{name}: max|diff|={mx:.3e} rel={rel:.3e} (tol {atol}, {rtol})"
    return mx, rel


def tensors(w, x):
    t, x64 = synth.as_dtype(w, x)
    return t.cuda(), x64


def make_layer(w, page_size=0, num_splits=0, topk=None, residual=False):
    topk = w.topk if topk is None else topk
    bt, npages = (None, 0)
    if page_size:
        table, npages = synth.page_table(w, page_size)
        bt = torch.from_numpy(table)
    return CachedBlockAttention(
        w.batch, w.num_q_heads, w.num_kv_heads, w.head_dim, w.block_len, w.capacity, dtype=w.dtype,
        softmax_scale=w.softmax_scale, page_size=page_size, block_table=bt, num_pages=npages,
        chunk_size=w.chunk_size if topk else 0, topk=topk, num_splits=num_splits, residual=residual)


def run_workload(w, page_size=0, num_splits=0, check_full=True, steps=None, blocks=None, v_scale=1.0):
    """Runs the workload on GPU and oracle; returns per-step error records.

    v_scale (a power of two, so the scaled values round to bf16 exactly as
    the unscaled ones do) multiplies every value row, prefix and block."""
    K, V, lens = synth.prefix_kv(w)
    V = V * np.float32(v_scale)
    Kt, K64 = tensors(w, K)
    Vt, V64 = tensors(w, V)
    layer = make_layer(w, page_size, num_splits)
    layer.load_prefix(Kt, Vt, lens)
    lens_o = lens.astype(np.int64).copy()
    Kc, Vc = K64.copy(), V64.copy()
    records = []
    nsteps = w.steps if steps is None else steps
    nblocks = w.blocks if blocks is None else blocks
    for blk in range(nblocks):
        base = synth.block_base(w, blk)
        pre = None
        for s in range(nsteps):
            Q, Kb, Vb = synth.step_inputs(w, blk, s, base)
            Vb = Vb * np.float32(v_scale)
            Qt, Q64 = tensors(w, Q)
            Kbt, Kb64 = tensors(w, Kb)
            Vbt, Vb64 = tensors(w, Vb)
            if s in w.refresh or pre is None:
                layer.refresh(Qt)
                idx = None
                if w.topk:
                    Km, valid = ora.chunk_means(Kc, lens_o, w.chunk_size)
                    idx = ora.select_chunks(Q64, Km, valid, w.topk)
                    gidx = layer.chunk_idx.cpu().numpy()
                    assert np.array_equal(gidx, idx), f"block {blk} step {s}: chunk selection differs"
                pre = ora.prefix_partial(Q64, Kc, Vc, lens_o, w.softmax_scale, idx, w.chunk_size)
                torch.cuda.synchronize()
                records.append(("O_pre", blk, s) + compare(f"O_pre b{blk} s{s}", layer.O_pre.cpu().numpy(), pre[0], w.dtype))
                records.append(("LSE_pre", blk, s) + compare(f"LSE_pre b{blk} s{s}", layer.LSE_pre.cpu().numpy(), pre[1], w.dtype))
            O = layer.step(Qt, Kbt, Vbt, lse=True)
            o_ref, l_ref = ora.block_step(Q64, Kb64, Vb64, pre[0], pre[1], w.softmax_scale)
            torch.cuda.synchronize()
            records.append(("O", blk, s) + compare(f"O b{blk} s{s}", O.float().cpu().numpy(), o_ref, w.dtype))
            records.append(("LSE", blk, s) + compare(f"LSE b{blk} s{s}", layer.LSE.cpu().numpy(), l_ref, w.dtype))
            if check_full:
                Of = layer.full(Qt, Kbt, Vbt, lse=True)
                of_ref, lf_ref = ora.full_attention(Q64, Kc, Vc, lens_o, Kb64, Vb64, w.softmax_scale)
                torch.cuda.synchronize()
                records.append(("O_full", blk, s) + compare(f"O_full b{blk} s{s}", Of.float().cpu().numpy(), of_ref, w.dtype))
                records.append(("LSE_full", blk, s) + compare(f"LSE_full b{blk} s{s}", layer.LSE.cpu().numpy(), lf_ref, w.dtype))
        # block end: the last step's K/V joins the prefix
        layer.append(Kbt, Vbt)
        for b in range(w.batch):
            L = int(lens_o[b])
            if L + w.block_len <= Kc.shape[1]:
                Kc[b, L:L + w.block_len] = Kb64[b]
                Vc[b, L:L + w.block_len] = Vb64[b]
                lens_o[b] = L + w.block_len
    layer.check()
    assert np.array_equal(layer.lens.cpu().numpy(), lens_o), "prefix lengths after append"
    return records


def run_residual(w, steps=None):
    """Residual reuse with sparse attention: GPU block vs the oracle's."""
    K, V, lens = synth.prefix_kv(w)
    Kt, K64 = tensors(w, K)
    Vt, V64 = tensors(w, V)
    layer = make_layer(w, residual=True)
    layer.load_prefix(Kt, Vt, lens)
    base = synth.block_base(w, 0)
    nsteps = w.steps if steps is None else steps
    Qs, Kbs, Vbs, outs = [], [], [], []
    for s in range(nsteps):
        Q, Kb, Vb = synth.step_inputs(w, 0, s, base)
        Qt, Q64 = tensors(w, Q)
        Kbt, Kb64 = tensors(w, Kb)
        Vbt, Vb64 = tensors(w, Vb)
        if s in w.refresh:
            layer.refresh(Qt)
        outs.append(layer.step(Qt, Kbt, Vbt).float().cpu().numpy())
        Qs.append(Q64)
        Kbs.append(Kb64)
        Vbs.append(Vb64)
    layer.check()
    ref = ora.residual_block(Qs, Kbs, Vbs, K64, V64, lens.astype(np.int64), w.softmax_scale, w.refresh, w.topk,
                             w.chunk_size)
    return [compare(f"residual O s{s}", outs[s], ref[s], w.dtype) for s in range(nsteps)]


def run_policy(w, policy, steps, gamma=0.9, tau=None, eps=0.25, margin=1e-3):
    """Adaptive reuse on the GPU vs the oracle's ``headwise_block`` /
    ``threshold_block`` on the policy input generators.

    The decisions are compared exactly; the inputs are first checked to keep
    every decision at least ``margin`` away from its threshold (computed from
    the oracle's own decisions), so that rounding cannot flip one."""
    K, V, lens = synth.prefix_kv(w)
    Kt, K64 = tensors(w, K)
    Vt, V64 = tensors(w, V)
    gen = synth.headwise_steps if policy == "headwise" else synth.threshold_steps
    raw = gen(w, 0, steps)
    if tau is None:
        tau = max(1, w.block_len // 4)
    layer = CachedBlockAttention(
        w.batch, w.num_q_heads, w.num_kv_heads, w.head_dim, w.block_len, w.capacity, dtype=w.dtype,
        softmax_scale=w.softmax_scale, policy=policy, gamma=gamma, tau=tau, eps=eps)
    layer.load_prefix(Kt, Vt, lens)
    Qs, Kbs, Vbs, outs, masks, stats = [], [], [], [], [], []
    for s, (Q, Kb, Vb) in enumerate(raw):
        Qt, Q64 = tensors(w, Q)
        Kbt, Kb64 = tensors(w, Kb)
        Vbt, Vb64 = tensors(w, Vb)
        outs.append(layer.cached_step(s, Qt, Kbt, Vbt).float().cpu().numpy())
        masks.append(layer.unit_mask.cpu().numpy().astype(bool))
        stats.append((layer.sim if policy == "headwise" else layer.updated).cpu().numpy())
        Qs.append(Q64)
        Kbs.append(Kb64)
        Vbs.append(Vb64)
    layer.check()
    L64 = lens.astype(np.int64)
    if policy == "headwise":
        ref, ref_masks = ora.headwise_block(Qs, Kbs, Vbs, K64, V64, L64, w.softmax_scale, gamma)
        # the similarity each decision was taken on, with the oracle's reference queries
        Qref = Qs[0].copy()
        G = w.group
        for s in range(1, steps):
            sim = ora.unit_query_similarity(Qs[s], Qref, w.num_kv_heads)
            assert np.abs(sim - gamma).min() > margin, f"step {s}: a similarity is within {margin} of gamma"
            np.testing.assert_allclose(stats[s], sim, atol=1e-4, err_msg=f"similarity at step {s}")
            for b in range(w.batch):
                for kvh in range(w.num_kv_heads):
                    if ref_masks[s][b, kvh]:
                        Qref[b, :, kvh * G:(kvh + 1) * G] = Qs[s][b, :, kvh * G:(kvh + 1) * G]
        for s in range(steps):
            assert np.array_equal(masks[s], ref_masks[s]), f"step {s}: refresh mask differs"
    else:
        ref, ref_flags = ora.threshold_block(Qs, Kbs, Vbs, K64, V64, L64, w.softmax_scale, tau, eps)
        for s in range(1, steps):
            dk = np.abs(Kbs[s] - Kbs[s - 1]).max(axis=(2, 3))
            dv = np.abs(Vbs[s] - Vbs[s - 1]).max(axis=(2, 3))
            assert np.abs(np.maximum(dk, dv) - eps).min() > margin, f"step {s}: a token change is near eps"
            count = ora.updated_tokens(Kbs[s - 1], Vbs[s - 1], Kbs[s], Vbs[s], eps)
            assert np.array_equal(stats[s], count), f"step {s}: updated-token counts differ"
        for s in range(steps):
            want = np.repeat(ref_flags[s][:, None], w.num_kv_heads, axis=1)
            assert np.array_equal(masks[s], want), f"step {s}: refresh flags differ"
    errs = [compare(f"{policy} O s{s}", outs[s], ref[s], w.dtype) for s in range(steps)]
    return errs, masks
