"""The FMA-pipe 2^x used for part of the softmax exponentials, checked on the
CPU: the coefficients are read from the CUDA header and the float32 steps
(rounding-constant split, cubic in f, exponent-field add) are replayed bit for
bit with numpy, then compared with 2^x in float64."""
import os
import re

import numpy as np

HDR = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))),
                   "block_diffusion_attention_b200", "csrc", "fb_ptx.cuh")


def _coefs():
    src = open(HDR).read()
    vals = {}
    for name in ("EXP2_C1", "EXP2_C2", "EXP2_C3"):
        m = re.search(name + r"\s*=\s*([0-9.eE+-]+)f", src)
        assert m, name
        vals[name] = np.float32(float(m.group(1)))
    return vals["EXP2_C1"], vals["EXP2_C2"], vals["EXP2_C3"]


def _emulate(x):
    c1, c2, c3 = _coefs()
    one = np.float32(1.0)
    k = np.float32(12582912.0)
    x = np.maximum(x.astype(np.float32), np.float32(-126.0))
    t = (x + k).astype(np.float32)
    r = (t + (-k)).astype(np.float32)
    f = (r * np.float32(-1.0) + x).astype(np.float32)
    p = (c3 * f + c2).astype(np.float32)
    p = (p * f + c1).astype(np.float32)
    p = (p * f + one).astype(np.float32)
    bits = (p.view(np.int32).astype(np.int64) + (t.view(np.int32).astype(np.int64) << 23)) & 0xFFFFFFFF
    return bits.astype(np.uint32).view(np.float32)


def test_relative_error_bound():
    rng = np.random.default_rng(0)
    x = np.concatenate([rng.uniform(-125.0, 8.0, 2_000_000), np.arange(-125, 9, dtype=np.float64),
                        np.arange(-125, 8, dtype=np.float64) + 0.5]).astype(np.float32)
    got = _emulate(x).astype(np.float64)
    ref = np.exp2(x.astype(np.float64))
    rel = np.abs(got / ref - 1.0)
    # the fit's own error is 1.0e-4; float32 evaluation adds a few ulp
    assert rel.max() < 1.2e-4, rel.max()


def test_special_values():
    x = np.array([0.0, 1.0, -1.0, 8.0, -np.inf, -1000.0], dtype=np.float32)
    got = _emulate(x)
    assert abs(got[0] - 1.0) < 1e-4 and abs(got[1] - 2.0) < 2e-4 and abs(got[2] - 0.5) < 1e-4
    assert abs(got[3] - 256.0) < 256 * 1.2e-4
    # far-negative inputs are clamped to 2^-126 (negligible beside the row max)
    assert got[4] == got[5] and 0 < got[4] < 1.5 * 2.0 ** -126


def test_monotone_on_a_fine_grid():
    x = np.linspace(-20, 8, 200001).astype(np.float32)
    got = _emulate(x).astype(np.float64)
    assert np.all(np.diff(got) >= 0)
