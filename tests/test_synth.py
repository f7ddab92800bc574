"""The seeded input generators (CPU): the recipe the workloads, the parity
tests and the benchmark rely on -- deterministic seeds, independent per-step
drift, zero rows past each prefix, one bf16 rounding, and the clear margins
the adaptive-reuse generators are built to have."""
import os
import sys

import numpy as np
import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

from block_diffusion_attention_b200 import synth  # noqa: E402

W = synth.WORKLOADS


def small(name="lm_gqa", **kw):
    base = dict(prefix_len=300, blocks=2, steps=4)
    base.update(kw)
    return W[name].scaled(**base)


def test_seeds_are_deterministic_and_streams_independent():
    w = small()
    K1, V1, l1 = synth.prefix_kv(w)
    K2, V2, l2 = synth.prefix_kv(w)
    assert np.array_equal(K1, K2) and np.array_equal(V1, V2) and np.array_equal(l1, l2)
    a = synth.step_inputs(w, 0, 1)
    b = synth.step_inputs(w, 0, 1)
    for x, y in zip(a, b):
        assert np.array_equal(x, y)
    # other step, other block, other tensor: different draws
    c = synth.step_inputs(w, 0, 2)
    d = synth.step_inputs(w, 1, 1)
    assert not np.array_equal(a[0], c[0]) and not np.array_equal(a[0], d[0])
    assert not np.array_equal(K1, V1)


def test_drift_is_independent_per_step_not_a_walk():
    w = small(batch=2, block_len=64)
    base = synth.block_base(w, 0)
    d1 = synth.step_inputs(w, 0, 1, base)[1] - base[1]
    d3 = synth.step_inputs(w, 0, 3, base)[1] - base[1]
    # each step: base + N(0, drift^2); a random walk would grow with the step
    assert np.std(d1) == pytest.approx(w.drift, rel=0.05)
    assert np.std(d3) == pytest.approx(w.drift, rel=0.05)
    assert abs(np.corrcoef(d1.ravel(), d3.ravel())[0, 1]) < 0.05
    # queries keep their base with q_drift=False; keys still drift
    q, k, _ = synth.step_inputs(w, 0, 1, base, q_drift=False)
    assert np.array_equal(q, base[0]) and not np.array_equal(k, base[1])


def test_query_scale_and_prefix_values():
    w = small(prefix_len=2000)
    Q0 = synth.block_base(w, 0)[0]
    assert np.std(Q0) == pytest.approx(w.q_std, rel=0.05)
    K, V, lens = synth.prefix_kv(w)
    n = int(lens[0])
    assert np.std(K[0, :n]) == pytest.approx(1.0, rel=0.02) and abs(np.mean(V[0, :n])) < 0.02
    # room for the appended blocks is zero
    assert K.shape[1] == w.capacity and not K[0, n:].any() and not V[0, n:].any()


def test_varlen_lengths_in_range():
    w = W["batched_sparse"].scaled(prefix_len=1000, prefix_min=400, batch=64)
    lens = synth.prefix_lens(w)
    assert lens.dtype == np.int32 and lens.shape == (64,)
    assert lens.min() >= 400 and lens.max() <= 1000 and len(set(lens.tolist())) > 20
    K, _, _ = synth.prefix_kv(w.scaled(batch=4))
    l4 = synth.prefix_lens(w.scaled(batch=4))
    for b in range(4):
        n = int(l4[b])
        assert K[b, n - 1].any() and not K[b, n:].any()


def test_bf16_inputs_are_one_rne_rounding():
    import torch
    x = np.random.default_rng(7).standard_normal(4096).astype(np.float32)
    t, x64 = synth.round_bf16(x)
    assert t.dtype == torch.bfloat16 and x64.dtype == np.float64
    # every value is a bf16 value (rounding it again changes nothing) ...
    again = torch.from_numpy(x64.astype(np.float32)).to(torch.bfloat16).to(torch.float64).numpy()
    assert np.array_equal(again, x64)
    # ... within half a bf16 ulp of the float32 draw (8 significant bits)
    ulp = np.exp2(np.floor(np.log2(np.abs(x.astype(np.float64)))) - 7)
    assert np.all(np.abs(x64 - x) <= ulp / 2 + 1e-300)
    # fp32 workloads keep their values as drawn
    t32, v32 = synth.as_dtype(W["tiny_fp32"], x)
    assert np.array_equal(v32, x.astype(np.float64))


def test_headwise_generator_units_stay_or_jump_clearly():
    w = small(batch=2)
    steps = synth.headwise_steps(w, 0, 6)
    G = w.group
    stay = jump = 0
    for s in range(1, 6):
        prev, cur = steps[s - 1][0], steps[s][0]
        for b in range(w.batch):
            for kvh in range(w.num_kv_heads):
                a = prev[b, :, kvh * G:(kvh + 1) * G].ravel().astype(np.float64)
                c = cur[b, :, kvh * G:(kvh + 1) * G].ravel().astype(np.float64)
                cos = a @ c / np.sqrt((a @ a) * (c @ c))
                assert cos > 0.99 or cos < 0.2, cos  # never near a threshold in between
                stay += cos > 0.99
                jump += cos < 0.2
    assert stay > 0 and jump > 0


def test_threshold_generator_tokens_move_clearly_or_not():
    w = small(batch=3, block_len=32)
    steps = synth.threshold_steps(w, 0, 5)
    moved_counts = []
    for s in range(1, 5):
        dk = np.abs(steps[s][1] - steps[s - 1][1]).max(axis=(2, 3))
        dv = np.abs(steps[s][2] - steps[s - 1][2]).max(axis=(2, 3))
        d = np.maximum(dk, dv)                      # [B, S]: each token's largest change
        moved = d > 0.25
        assert np.all(d[moved] > 0.5) and np.all(d[~moved] < 0.1)
        counts = moved.sum(axis=1)
        assert np.all(counts <= w.block_len // 2)
        moved_counts.extend(counts.tolist())
    assert len(set(moved_counts)) > 1


def test_page_table_is_a_permutation_and_paging_round_trips():
    w = small(batch=3, prefix_len=500)
    table, num_pages = synth.page_table(w, 64)
    assert sorted(table.ravel().tolist()) == list(range(num_pages))
    K, _, _ = synth.prefix_kv(w)
    pool = synth.to_paged(K, table, 64)
    back = np.concatenate([pool[table[b]].reshape(-1, *K.shape[2:])[None, :K.shape[1]]
                           for b in range(w.batch)])
    assert np.array_equal(back, K)
