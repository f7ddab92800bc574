"""The launch plans the library picks for the five workloads on a 148-SM B200,
read through fb_workspace_bytes (host logic only: no kernel is launched, and
without a GPU the library plans for 148 SMs).

The split workspace holds one f32 partial (D + 1 floats: O and LSE) per query
row and key split, or, for a tail split, one per (tail unit, split, query
tile) and 128 rows; so its size names the plan:

* long_ctx, 128K: 17 key splits x 8 one-tile units = 136 CTAs for the prefix
  pass and for the uncached pass (the cost model's best alone is 18; for
  one-tile units the fewest splits within 7 % of it are taken);
* lm_gqa, 8K (65 key tiles in the 8320-row cache): 17 splits x 8 units;
* video: 760 two-tile units are five full waves of 148 and a sixth of 20, so
  the prefix pass, the uncached pass and the block step run those 20 units
  split 7 ways over their keys (148 / 20 = 7);
* batched_sparse: the top-16 prefix pass is one wave of 128 unsplit two-tile
  units (no workspace); the uncached pass over the dense 32K prefix (258 key
  tiles) takes 8 splits, 1024 CTAs in 7 waves (two-tile units keep the
  model's best: one unsplit wave measured 504 us against 457-487 us);
* tiny_fp32: the fp32 kernel never splits.
"""
import pytest
import torch

from block_diffusion_attention_b200 import flashblock as fbl, synth

F32 = 4
SLOT = 128 * (128 + 1) * F32  # one 128-row tile's partial


def _desc(w):
    lens = torch.zeros(w.batch, dtype=torch.int32)
    d = fbl.make_desc(w.batch, w.num_q_heads, w.num_kv_heads, w.head_dim, w.block_len,
                      dtype=fbl.FB_BF16 if w.dtype == "bf16" else fbl.FB_FP32, kv_capacity=w.capacity,
                      prefix_lens=lens, chunk_size=w.chunk_size if w.topk else 0, topk=w.topk)
    return d, lens


def _split_bytes(w, splits):
    rows = w.batch * w.block_len * w.num_q_heads
    return splits * rows * (w.head_dim + 1) * F32


@pytest.fixture(autouse=True)
def _b200_sm_count():
    if torch.cuda.is_available() and torch.cuda.get_device_properties(0).multi_processor_count != 148:
        pytest.skip("the plans below are those of a 148-SM B200")


@pytest.mark.parametrize("name,expected", [
    ("long_ctx", lambda w: _split_bytes(w, 17)),
    ("lm_gqa", lambda w: _split_bytes(w, 17)),
    ("video", lambda w: 20 * 7 * 2 * SLOT),
    ("batched_sparse", lambda w: _split_bytes(w, 8)),
])
def test_split_workspace_names_the_plan(name, expected):
    w = synth.WORKLOADS[name]
    d, _ = _desc(w)
    assert fbl.fb_workspace_bytes(d) == expected(w)


def test_fp32_path_needs_no_split_workspace():
    w = synth.WORKLOADS["tiny_fp32"]
    d, _ = _desc(w)
    assert fbl.fb_workspace_bytes(d) < SLOT


def test_explicit_split_count_is_taken_as_given():
    # num_splits > 0 overrides the cost model (capped at the key tiles)
    w = synth.WORKLOADS["long_ctx"]
    d, _ = _desc(w)
    for ns in (1, 5, 18, 64):
        d.num_splits = ns
        assert fbl.fb_workspace_bytes(d) == (_split_bytes(w, ns) if ns > 1 else
                                             # the masked pass's active-unit slots (8 units, one split)
                                             8 * SLOT)
