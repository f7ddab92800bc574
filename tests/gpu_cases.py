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


def run_workload(w, page_size=0, num_splits=0, check_full=True, steps=None, blocks=None):
    """Runs the workload on GPU and oracle; returns per-step error records."""
    K, V, lens = synth.prefix_kv(w)
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
