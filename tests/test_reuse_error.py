"""The reuse error of the method: the oracle's cached schedule (Core Mechanism
of "FlashBlock: Attention Caching for Efficient Long-Context Block
Diffusion", Technical Summary §2: the block-external pair of the last refresh
reused on later steps) against its uncached full attention on the same
synthetic inputs.  It is a property of the method, not a tolerance: zero at
refresh steps and without drift, and about proportional to the per-step drift
of the block's queries for small drift."""
import numpy as np

from block_diffusion_attention_b200 import synth
from oracle import flashblock_oracle as ora


def _reuse_errors(drift):
    w = synth.WORKLOADS["lm_gqa"].scaled(prefix_len=300, blocks=1, steps=4, block_len=8, num_q_heads=8,
                                         num_kv_heads=2)
    K, V, lens = synth.prefix_kv(w)
    base = synth.block_base(w, 0)
    steps = [synth.step_inputs(w, 0, s, base, drift=drift) for s in range(w.steps)]
    f64 = lambda x: x.astype(np.float64)  # noqa: E731
    Qs = [f64(q) for q, _, _ in steps]
    Kbs = [f64(k) for _, k, _ in steps]
    Vbs = [f64(v) for _, _, v in steps]
    outs, _ = ora.cached_block(Qs, Kbs, Vbs, f64(K), f64(V), lens, w.softmax_scale, (0,))
    errs = []
    for s in range(w.steps):
        Of, _ = ora.full_attention(Qs[s], f64(K), f64(V), lens, Kbs[s], Vbs[s], w.softmax_scale)
        errs.append(float(np.linalg.norm(outs[s] - Of) / np.linalg.norm(Of)))
    return errs


def test_reuse_error_grows_with_drift():
    # the workloads' drifts (0.05, 0.1) are large beside the queries' own
    # scale here (1 / sqrt(128)), so the errors are of order one
    e0, e1, e2 = _reuse_errors(0.0), _reuse_errors(0.05), _reuse_errors(0.1)
    for e in (e0, e1, e2):
        assert e[0] < 1e-12, "the refresh step recomputes the pair: no reuse error"
    assert max(e0[1:]) < 1e-12, "without drift, reuse equals recomputation"
    for s in range(1, 4):
        assert 0 < e1[s] < e2[s], f"step {s}: the error grows with the drift"


def test_reuse_error_is_first_order_in_small_drift():
    e1, e2 = _reuse_errors(0.002), _reuse_errors(0.004)
    ratio = sum(e2[1:]) / sum(e1[1:])
    assert 1.8 < ratio < 2.2, f"doubling a small drift about doubles the error ({ratio:.2f})"
