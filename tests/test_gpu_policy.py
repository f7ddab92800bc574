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
