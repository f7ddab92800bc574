"""Adaptive reuse on the GPU ("Adaptive Reuse Strategies": Head-wise
Selection and Threshold-based Reuse) against the float64 oracle: refresh
masks, the similarity / updated-token statistics they are taken on, and the
step outputs."""
import numpy as np
import pytest

from block_diffusion_attention_b200 import synth
from gpu_cases import run_policy

pytestmark = pytest.mark.gpu

W_BF16 = synth.WORKLOADS["lm_gqa"].scaled(batch=3, prefix_len=1500, blocks=1)
W_FP32 = synth.WORKLOADS["tiny_fp32"].scaled(batch=2, num_q_heads=4, num_kv_heads=2, prefix_len=300)


def _mixed(masks):
    later = np.stack(masks[1:])
    return later.any() and not later.all()


@pytest.mark.parametrize("w", [W_BF16, W_FP32], ids=["bf16", "fp32"])
def test_headwise_policy_matches_oracle(w):
    errs, masks = run_policy(w, "headwise", steps=6, gamma=0.9)
    assert masks[0].all()
    assert _mixed(masks), "the inputs should make some units refresh and others reuse"


@pytest.mark.parametrize("w", [W_BF16, W_FP32], ids=["bf16", "fp32"])
def test_threshold_policy_matches_oracle(w):
    errs, masks = run_policy(w, "threshold", steps=6, tau=max(1, w.block_len // 4), eps=0.25)
    assert masks[0].all()
    assert _mixed(masks), "the inputs should make some sequences refresh and others reuse"


def test_headwise_extremes_bf16():
    # gamma above any similarity: every unit refreshes at every step (the
    # uncached result); gamma below any: nothing refreshes after step 0
    _, masks = run_policy(W_BF16, "headwise", steps=3, gamma=1.5)
    assert all(m.all() for m in masks)
    _, masks = run_policy(W_BF16, "headwise", steps=3, gamma=-1.5)
    assert not any(m.any() for m in masks[1:])


def test_threshold_extremes_bf16():
    _, masks = run_policy(W_BF16, "threshold", steps=3, tau=0)
    assert all(m.all() for m in masks)
    _, masks = run_policy(W_BF16, "threshold", steps=3, tau=W_BF16.block_len + 1)
    assert not any(m.any() for m in masks[1:])


MASKED_SHAPES = {
    # one query tile per unit (the grid may be shared out among the selected units)
    "lm": dict(batch=2, prefix_len=5000, blocks=1),
    # two and three query tiles per unit: the two-tile kernel, masked units skipped
    "pair": dict(batch=2, block_len=64, prefix_len=3000, blocks=1),
    "mha": dict(batch=1, num_q_heads=4, num_kv_heads=4, block_len=300, prefix_len=2000, blocks=1),
}


@pytest.mark.parametrize("shape,num_splits,page_size", [("lm", 0, 0), ("lm", 5, 0), ("lm", 0, 128), ("lm", 3, 64),
                                                        ("pair", 0, 0), ("pair", 3, 128), ("mha", 0, 0),
                                                        ("mha", 2, 0)])
def test_masked_prefix_pass_random_masks(shape, num_splits, page_size):
    """fb_prefix_partial_masked against the oracle's prefix partial: the rows
    of selected units are recomputed, the others are left untouched (also
    when the grid is shared out among the selected units only)."""
    import torch
    from block_diffusion_attention_b200 import flashblock as fbl
    from gpu_cases import compare, make_layer, tensors
    from oracle import flashblock_oracle as ora

    w = synth.WORKLOADS["lm_gqa"].scaled(**MASKED_SHAPES[shape])
    K, V, lens = synth.prefix_kv(w)
    Kt, K64 = tensors(w, K)
    Vt, V64 = tensors(w, V)
    layer = make_layer(w, page_size=page_size, num_splits=num_splits)
    layer.load_prefix(Kt, Vt, lens)
    Q, _, _ = synth.step_inputs(w, 0, 0)
    Qt, Q64 = tensors(w, Q)
    ref_o, ref_l = ora.prefix_partial(Q64, K64, V64, lens.astype(np.int64), w.softmax_scale)
    rng = np.random.default_rng(7)
    masks = [np.ones((w.batch, w.num_kv_heads), np.int32), np.zeros((w.batch, w.num_kv_heads), np.int32),
             (rng.random((w.batch, w.num_kv_heads)) < 0.3).astype(np.int32)]
    one = np.zeros((w.batch, w.num_kv_heads), np.int32)
    one[w.batch - 1, w.num_kv_heads - 1] = 1
    masks.append(one)
    G = w.group
    for mk in masks:
        mask = torch.from_numpy(mk).cuda()
        layer.O_pre.fill_(7.0)
        layer.LSE_pre.fill_(3.0)
        fbl.fb_prefix_partial_masked(layer.desc, Qt, layer.K, layer.V, None, mask, layer.O_pre, layer.LSE_pre,
                                     layer.workspace, layer.status)
        layer.check()
        O = layer.O_pre.cpu().numpy()
        L = layer.LSE_pre.cpu().numpy()
        for b in range(w.batch):
            for kvh in range(w.num_kv_heads):
                hs = slice(kvh * G, (kvh + 1) * G)
                if mk[b, kvh]:
                    compare(f"O_pre b{b} kvh{kvh}", O[b, :, hs], ref_o[b, :, hs], w.dtype)
                    compare(f"LSE_pre b{b} kvh{kvh}", L[b, hs], ref_l[b, hs], w.dtype)
                else:
                    assert np.all(O[b, :, hs] == 7.0) and np.all(L[b, hs] == 3.0), f"unit {b},{kvh} was written"
