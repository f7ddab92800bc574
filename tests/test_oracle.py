"""The float64 oracle against its pins, and planted mistakes against the pins.

CPU only.  The second half plants one plausible mistake at a time in a copy of
the oracle's source (a dropped term, a wrong sign, index or base, a transposed
operand) and checks that at least one pin catches it.
"""
import importlib.util
import os

import numpy as np
import pytest

import oracle_pins
from oracle import flashblock_oracle as ora

ORACLE_SRC = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))),
                          "oracle", "flashblock_oracle.py")


@pytest.mark.parametrize("pin", oracle_pins.ALL_PINS, ids=lambda p: p.__name__)
def test_oracle_pin(pin):
    pin(ora)


MUTANTS = {
    "lse_log2": ("lse = m[:, 0] + np.log(zsum)", "lse = m[:, 0] + np.log2(zsum)"),
    "scale_dropped": ("z = scale * (q @ k.T)", "z = (q @ k.T)"),
    "no_normalise": ("o = (e @ v) / zsum[:, None]", "o = (e @ v)"),
    "merge_sign": ("np.exp(lse_b - m_safe))", "np.exp(m_safe - lse_b))"),
    "merge_drop_m": ("m_safe + np.log(den_safe)", "np.log(den_safe)"),
    "merge_swap_weights": ("(w_a[..., None] * o_a + w_b[..., None] * o_b)",
                           "(w_b[..., None] * o_a + w_a[..., None] * o_b)"),
    "gqa_index": ("h = kvh * G + g", "h = g * Hkv + kvh"),
    "tie_break": ("key=lambda c: (-sc[b, kvh, c], c)", "key=lambda c: (-sc[b, kvh, c], -c)"),
    "chunk_mean_div": ("Km[b, :, c, :] = Kc[b, lo:hi, :, :].mean(axis=0)",
                       "Km[b, :, c, :] = Kc[b, lo:hi, :, :].sum(axis=0) / chunk_size"),
    "block_keys_reversed": ("Kb[b, :, kvh, :]], axis=0)", "Kb[b, ::-1, kvh, :]], axis=0)"),
    "chunk_clip": ("hi = min((c + 1) * chunk_size, int(prefix_len))", "hi = (c + 1) * chunk_size"),
    "inblock_gqa": ("Vb[b, :, h // G, :], scale)", "Vb[b, :, h % Vb.shape[2], :], scale)"),
    "prefix_len_off_by_one": ("pos = np.arange(L)", "pos = np.arange(max(L - 1, 0))"),
    "reuse_never_refresh": ("if s in refresh_steps or pre is None:", "if pre is None:"),
    "residual_stale_selected": ("sel = prefix_partial(Q, Kc, Vc, prefix_lens, scale, idx, chunk_size)",
                                "sel = prefix_partial(Qs[0], Kc, Vc, prefix_lens, scale, idx, chunk_size)"),
    "headwise_keeps_stale_ref": ("                            Qref[b, :, hs] = Q[b, :, hs]\n", ""),
    "similarity_unnormalised": ("sim[b, kvh] = (a @ r) / den if den > 0 else 1.0", "sim[b, kvh] = (a @ r) if den > 0 else 1.0"),
    "threshold_inverted": ("updated_tokens(Kbs[s - 1], Vbs[s - 1], Kbs[s], Vbs[s], eps) >= tau",
                           "updated_tokens(Kbs[s - 1], Vbs[s - 1], Kbs[s], Vbs[s], eps) < tau"),
    "updated_ignores_v": ("return ((dk > eps) | (dv > eps)).sum(axis=1)", "return (dk > eps).sum(axis=1)"),
    "complement_drops_last": ("comp[b, kvh, :len(rest)] = rest", "comp[b, kvh, :len(rest) - 1] = rest[:-1]"),
}


def _mutant(name, old, new):
    src = open(ORACLE_SRC).read()
    assert old in src, f"mutation {name}: pattern not found in the oracle"
    src = src.replace(old, new, 1)
    spec = importlib.util.spec_from_loader(f"oracle_mutant_{name}", loader=None)
    mod = importlib.util.module_from_spec(spec)
    exec(compile(src, f"<mutant {name}>", "exec"), mod.__dict__)
    return mod


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_planted_mistake_is_caught(name):
    old, new = MUTANTS[name]
    mod = _mutant(name, old, new)
    with np.errstate(all="ignore"):
        bad = oracle_pins.failing_pins(mod)
    assert bad, f"planted mistake {name} passed every pin"
