"""Pins of the float64 oracle against facts the method and the mathematics fix.

Each ``pin_*`` takes the oracle module (or a planted-mistake copy of it) and
raises AssertionError when the oracle disagrees with the fact.  The facts:

* brute force: pure-Python term-by-term softmax on tiny inputs (no max trick);
* worked examples derived by hand (tests/golden/*.txt);
* closed forms: one key, identical keys, constant values, logit shift,
  key/value permutation;
* merge of exact partials == attention over the union of keys (the merge
  equation of the Core Mechanism is exact), merge algebra (commutative,
  associative, (0, -inf) is the identity);
* reuse with unchanged queries == full recompute;
* rows of the weight matrix sum to 1;
* sparse prefix: chunk selection by brute force, topk >= #chunks == dense,
  selected chunks merged with their complement == dense.
"""
from __future__ import annotations

import math
import os

import numpy as np

import brute

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def _rand(rng, *shape):
    return rng.standard_normal(shape)


def _close(a, b, tol, what):
    a = np.asarray(a, dtype=np.float64)
    b = np.asarray(b, dtype=np.float64)
    assert a.shape == b.shape, f"{what}: shape {a.shape} vs {b.shape}"
    both_inf = np.isneginf(a) & np.isneginf(b)
    diff = np.where(both_inf, 0.0, np.abs(np.where(both_inf, 0.0, a) - np.where(both_inf, 0.0, b)))
    err = float(np.nanmax(diff)) if diff.size else 0.0
    assert np.all(np.isfinite(diff)) and err <= tol, f"{what}: max |diff| = {err} > {tol}"


def load_golden(name):
    vals = {}
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            key, rest = line.split(":", 1)
            vals[key.strip()] = np.array([float(x) for x in rest.split()])
    return vals


# ---------------------------------------------------------------------------

def pin_brute_partial(ora):
    rng = np.random.default_rng(11)
    for (R, N, D, scale) in [(1, 1, 1, 1.0), (3, 5, 4, 0.5), (4, 8, 3, 1.3), (2, 7, 4, 1.0 / 2)]:
        q, k, v = _rand(rng, R, D), _rand(rng, N, D), _rand(rng, N, D)
        o, l = ora.attention_partial(q, k, v, scale)
        bo, bl = brute.partial(brute.tolist(q), brute.tolist(k), brute.tolist(v), scale)
        _close(o, bo, 1e-12, "brute O")
        _close(l, bl, 1e-12, "brute LSE")


def pin_brute_layer(ora):
    """Whole-layer wrappers (GQA mapping, varlen prefix, block concat) vs brute force."""
    rng = np.random.default_rng(12)
    B, S, Hq, Hkv, D, Lcap = 2, 3, 4, 2, 4, 6
    Q = _rand(rng, B, S, Hq, D)
    Kc, Vc = _rand(rng, B, Lcap, Hkv, D), _rand(rng, B, Lcap, Hkv, D)
    Kb, Vb = _rand(rng, B, S, Hkv, D), _rand(rng, B, S, Hkv, D)
    lens = np.array([5, 2], dtype=np.int32)
    scale = 0.7
    O, L = ora.full_attention(Q, Kc, Vc, lens, Kb, Vb, scale)
    bO, bL = brute.layer_full(Q, Kc, Vc, lens, Kb, Vb, scale)
    for (b, t, h), o in bO.items():
        _close(O[b, t, h], o, 1e-12, f"full O[{b},{t},{h}]")
    for (b, h, t), l in bL.items():
        _close(L[b, h, t], l, 1e-12, f"full LSE[{b},{h},{t}]")
    # prefix-only and block-only partials through the same brute force
    zero_blk = np.zeros((B, 0, Hkv, D))
    Op, Lp = ora.prefix_partial(Q, Kc, Vc, lens, scale)
    bO, bL = brute.layer_full(Q, Kc, Vc, lens, zero_blk, zero_blk, scale)
    for (b, t, h), o in bO.items():
        _close(Op[b, t, h], o, 1e-12, "prefix O")
    for (b, h, t), l in bL.items():
        _close(Lp[b, h, t], l, 1e-12, "prefix LSE")
    Oi, Li = ora.inblock_partial(Q, Kb, Vb, scale)
    bO, bL = brute.layer_full(Q, Kc, Vc, np.zeros(B, dtype=np.int32), Kb, Vb, scale)
    for (b, t, h), o in bO.items():
        _close(Oi[b, t, h], o, 1e-12, "in-block O")
    for (b, h, t), l in bL.items():
        _close(Li[b, h, t], l, 1e-12, "in-block LSE")


def pin_golden(ora):
    g = load_golden("attention_worked_example.txt")
    k = np.stack([g["k0"], g["k1"], g["k2"]])
    v = np.stack([g["v0"], g["v1"], g["v2"]])
    o, l = ora.attention_partial(g["q"][None, :], k, v, 1.0)
    _close(o[0], g["a"], 1e-14, "worked attention A")
    _close(l[0], g["l"][0], 1e-14, "worked attention L")
    m = load_golden("merge_worked_example.txt")
    o, l = ora.merge_partials(m["a_out"][None], m["l_out"], m["a_in"][None], m["l_in"])
    _close(o[0], m["a_full"], 1e-14, "worked merge A")
    _close(l[0], m["l_full"][0], 1e-14, "worked merge L")


def pin_closed_forms(ora):
    rng = np.random.default_rng(13)
    D = 5
    q = _rand(rng, 3, D)
    # one key: O = v, LSE = z
    k, v = _rand(rng, 1, D), _rand(rng, 1, D)
    o, l = ora.attention_partial(q, k, v, 0.9)
    _close(o, np.repeat(v, 3, axis=0), 1e-13, "one key O")
    _close(l, 0.9 * (q @ k[0]), 1e-13, "one key LSE")
    # N identical keys: O = mean(V), LSE = z + log N
    N = 7
    k = np.repeat(_rand(rng, 1, D), N, axis=0)
    v = _rand(rng, N, D)
    o, l = ora.attention_partial(q, k, v, 1.1)
    _close(o, np.repeat(v.mean(axis=0, keepdims=True), 3, axis=0), 1e-13, "identical keys O")
    _close(l, 1.1 * (q @ k[0]) + math.log(N), 1e-13, "identical keys LSE")
    # constant value rows: O = c
    k = _rand(rng, 9, D)
    c = _rand(rng, 1, D)
    o, _ = ora.attention_partial(q, k, np.repeat(c, 9, axis=0), 1.0)
    _close(o, np.repeat(c, 3, axis=0), 1e-13, "constant V")
    # a logit shift (add a multiple of q to every key) shifts LSE and leaves O
    v = _rand(rng, 9, D)
    o1, l1 = ora.attention_partial(q[:1], k, v, 1.0)
    o2, l2 = ora.attention_partial(q[:1], k + 0.5 * q[:1], v, 1.0)
    _close(o1, o2, 1e-12, "shift O")
    _close(l2 - l1, 0.5 * (q[0] @ q[0]) * np.ones(1), 1e-12, "shift LSE")
    # permuting keys together with values changes nothing
    perm = rng.permutation(9)
    o3, l3 = ora.attention_partial(q, k[perm], v[perm], 1.0)
    o4, l4 = ora.attention_partial(q, k, v, 1.0)
    _close(o3, o4, 1e-13, "perm O")
    _close(l3, l4, 1e-13, "perm LSE")
    # empty key set
    o, l = ora.attention_partial(q, np.zeros((0, D)), np.zeros((0, D)), 1.0)
    assert np.all(o == 0) and np.all(np.isneginf(l)), "empty key set"


def pin_merge_is_concat(ora):
    rng = np.random.default_rng(14)
    for (na, nb) in [(1, 1), (5, 3), (12, 1), (0, 4), (4, 0)]:
        q = _rand(rng, 4, 6)
        ka, va = _rand(rng, na, 6) * 2, _rand(rng, na, 6)
        kb, vb = _rand(rng, nb, 6) * 2, _rand(rng, nb, 6)
        oa, la = ora.attention_partial(q, ka, va, 0.8)
        ob, lb = ora.attention_partial(q, kb, vb, 0.8)
        om, lm = ora.merge_partials(oa, la, ob, lb)
        of, lf = ora.attention_partial(q, np.concatenate([ka, kb]), np.concatenate([va, vb]), 0.8)
        _close(om, of, 1e-12, f"merge==concat O ({na},{nb})")
        _close(lm, lf, 1e-12, f"merge==concat LSE ({na},{nb})")


def pin_merge_algebra(ora):
    rng = np.random.default_rng(15)
    o = [_rand(rng, 3, 4) for _ in range(3)]
    l = [_rand(rng, 3) * 3 for _ in range(3)]
    ab = ora.merge_partials(o[0], l[0], o[1], l[1])
    ba = ora.merge_partials(o[1], l[1], o[0], l[0])
    _close(ab[0], ba[0], 1e-13, "commutative O")
    _close(ab[1], ba[1], 1e-13, "commutative LSE")
    left = ora.merge_partials(ab[0], ab[1], o[2], l[2])
    bc = ora.merge_partials(o[1], l[1], o[2], l[2])
    right = ora.merge_partials(o[0], l[0], bc[0], bc[1])
    _close(left[0], right[0], 1e-13, "associative O")
    _close(left[1], right[1], 1e-13, "associative LSE")
    ident = ora.merge_partials(o[0], l[0], np.zeros((3, 4)), np.full(3, -np.inf))
    _close(ident[0], o[0], 0.0, "identity O")
    _close(ident[1], l[0], 0.0, "identity LSE")
    both = ora.merge_partials(np.zeros((3, 4)), np.full(3, -np.inf), np.zeros((3, 4)), np.full(3, -np.inf))
    assert np.all(both[0] == 0) and np.all(np.isneginf(both[1])), "empty + empty"


def pin_refresh_step_exact(ora):
    """At a refresh step, merging the prefix and in-block partials equals full attention."""
    rng = np.random.default_rng(16)
    B, S, Hq, Hkv, D, Lcap = 2, 5, 6, 3, 8, 40
    Q = _rand(rng, B, S, Hq, D)
    Kc, Vc = _rand(rng, B, Lcap, Hkv, D), _rand(rng, B, Lcap, Hkv, D)
    Kb, Vb = _rand(rng, B, S, Hkv, D), _rand(rng, B, S, Hkv, D)
    lens = np.array([37, 0], dtype=np.int32)
    Op, Lp = ora.prefix_partial(Q, Kc, Vc, lens, 0.4)
    O, L = ora.block_step(Q, Kb, Vb, Op, Lp, 0.4)
    Of, Lf = ora.full_attention(Q, Kc, Vc, lens, Kb, Vb, 0.4)
    _close(O, Of, 1e-12, "refresh step O")
    _close(L, Lf, 1e-12, "refresh step LSE")


def pin_reuse_unchanged_queries(ora):
    """With the queries held fixed across steps (K/V of the block still drift),
    reusing the refresh-step prefix partial equals recomputing it."""
    rng = np.random.default_rng(17)
    B, S, Hq, Hkv, D, Lcap = 1, 4, 2, 1, 6, 30
    Q = _rand(rng, B, S, Hq, D)
    Kc, Vc = _rand(rng, B, Lcap, Hkv, D), _rand(rng, B, Lcap, Hkv, D)
    lens = np.array([30], dtype=np.int32)
    Kbase, Vbase = _rand(rng, B, S, Hkv, D), _rand(rng, B, S, Hkv, D)
    Ks = [Kbase + 0.05 * _rand(rng, B, S, Hkv, D) for _ in range(4)]
    Vs = [Vbase + 0.05 * _rand(rng, B, S, Hkv, D) for _ in range(4)]
    outs, _ = ora.cached_block([Q] * 4, Ks, Vs, Kc, Vc, lens, 0.5, refresh_steps=(0,))
    for s in range(4):
        Of, _ = ora.full_attention(Q, Kc, Vc, lens, Ks[s], Vs[s], 0.5)
        _close(outs[s], Of, 1e-12, f"reuse with fixed Q, step {s}")


def pin_refresh_recomputes(ora):
    """Every refresh step recomputes the prefix partial with that step's queries,
    so the output at any refresh step equals full attention even when the
    queries drift between steps."""
    rng = np.random.default_rng(20)
    B, S, Hq, Hkv, D, Lcap = 1, 2, 2, 1, 3, 5
    Qs = [_rand(rng, B, S, Hq, D) for _ in range(3)]
    Ks = [_rand(rng, B, S, Hkv, D) for _ in range(3)]
    Kc = _rand(rng, B, Lcap, Hkv, D)
    lens = np.array([5], dtype=np.int32)
    outs, _ = ora.cached_block(Qs, Ks, Ks, Kc, Kc, lens, 1.0, refresh_steps=(0, 2))
    for s in (0, 2):
        Of, _ = ora.full_attention(Qs[s], Kc, Kc, lens, Ks[s], Ks[s], 1.0)
        _close(outs[s], Of, 1e-12, f"refresh step {s}")
    Of, _ = ora.full_attention(Qs[1], Kc, Kc, lens, Ks[1], Ks[1], 1.0)
    assert np.max(np.abs(outs[1] - Of)) > 1e-6, "a reuse step must use the stale prefix partial"


def pin_rows_sum_to_one(ora):
    rng = np.random.default_rng(18)
    q, k = _rand(rng, 5, 7), _rand(rng, 33, 7) * 3
    W = ora.attention_weights(q, k, 0.9)
    _close(W.sum(axis=1), np.ones(5), 1e-12, "rows sum to 1")
    assert np.all(W >= 0)


def pin_sparse(ora):
    rng = np.random.default_rng(19)
    B, S, Hq, Hkv, D, Lcap, chunk = 2, 3, 4, 2, 4, 37, 8
    Q = _rand(rng, B, S, Hq, D)
    Kc, Vc = _rand(rng, B, Lcap, Hkv, D), _rand(rng, B, Lcap, Hkv, D)
    lens = np.array([37, 19], dtype=np.int32)
    Km, valid = ora.chunk_means(Kc, lens, chunk)
    # chunk means against a direct average of the valid rows
    for b in range(B):
        for c in range(Km.shape[2]):
            lo, hi = c * chunk, min((c + 1) * chunk, int(lens[b]))
            assert valid[b, c] == (hi > lo), "chunk validity"
            if hi > lo:
                _close(Km[b, :, c], Kc[b, lo:hi].sum(axis=0) / (hi - lo), 1e-13, "chunk mean")
    for topk in (1, 2, 3):
        idx = ora.select_chunks(Q, Km, valid, topk)
        bsel = brute.chunk_select(Q, Kc, lens, chunk, topk)
        for (b, kv), chosen in bsel.items():
            got = [int(c) for c in idx[b, kv] if c >= 0]
            assert got == chosen, f"selection b={b} kv={kv} topk={topk}: {got} vs {chosen}"
            assert list(idx[b, kv, len(chosen):]) == [-1] * (topk - len(chosen)), "padding"
    # every chunk selected -> the dense prefix partial
    idx = ora.select_chunks(Q, Km, valid, 64)
    Os, Ls = ora.prefix_partial(Q, Kc, Vc, lens, 0.6, idx, chunk)
    Od, Ld = ora.prefix_partial(Q, Kc, Vc, lens, 0.6)
    _close(Os, Od, 1e-12, "all chunks == dense O")
    _close(Ls, Ld, 1e-12, "all chunks == dense LSE")
    # a selection merged with its complement == dense
    idx = ora.select_chunks(Q, Km, valid, 2)
    nch = Km.shape[2]
    comp = np.full((B, Hkv, nch), -1, dtype=np.int32)
    for b in range(B):
        for kv in range(Hkv):
            rest = [c for c in range(nch) if valid[b, c] and c not in set(idx[b, kv].tolist())]
            comp[b, kv, :len(rest)] = rest
    Oa, La = ora.prefix_partial(Q, Kc, Vc, lens, 0.6, idx, chunk)
    Ob, Lb = ora.prefix_partial(Q, Kc, Vc, lens, 0.6, comp, chunk)
    Om, Lm = ora.merge_partials(Oa, La.transpose(0, 2, 1), Ob, Lb.transpose(0, 2, 1))
    _close(Om, Od, 1e-12, "selection + complement == dense O")
    _close(Lm.transpose(0, 2, 1), Ld, 1e-12, "selection + complement == dense LSE")


def pin_residual_reuse(ora):
    """Residual reuse with sparse attention: at a refresh step the residual +
    selected + in-block merge equals full attention; with queries held fixed
    every step does; with drifting queries the reuse steps differ."""
    rng = np.random.default_rng(21)
    B, S, Hq, Hkv, D, Lcap, chunk = 2, 3, 4, 2, 4, 45, 8
    Kc, Vc = _rand(rng, B, Lcap, Hkv, D), _rand(rng, B, Lcap, Hkv, D)
    lens = np.array([45, 30], dtype=np.int32)
    Kbs = [_rand(rng, B, S, Hkv, D) for _ in range(3)]
    Vbs = [_rand(rng, B, S, Hkv, D) for _ in range(3)]
    Qfix = _rand(rng, B, S, Hq, D)
    outs = ora.residual_block([Qfix] * 3, Kbs, Vbs, Kc, Vc, lens, 0.7, (0,), 2, chunk)
    for s in range(3):
        Of, _ = ora.full_attention(Qfix, Kc, Vc, lens, Kbs[s], Vbs[s], 0.7)
        _close(outs[s], Of, 1e-12, f"residual reuse, fixed Q, step {s}")
    Qs = [Qfix + 0.3 * _rand(rng, B, S, Hq, D) for _ in range(3)]
    outs = ora.residual_block(Qs, Kbs, Vbs, Kc, Vc, lens, 0.7, (0,), 2, chunk)
    Of, _ = ora.full_attention(Qs[0], Kc, Vc, lens, Kbs[0], Vbs[0], 0.7)
    _close(outs[0], Of, 1e-12, "residual reuse, refresh step")
    Of, _ = ora.full_attention(Qs[2], Kc, Vc, lens, Kbs[2], Vbs[2], 0.7)
    assert np.max(np.abs(outs[2] - Of)) > 1e-6, "reuse steps use the stale residual"
    # every chunk selected: no residual, so each step is exact even with drift
    outs = ora.residual_block(Qs, Kbs, Vbs, Kc, Vc, lens, 0.7, (0,), 64, chunk)
    for s in range(3):
        Of, _ = ora.full_attention(Qs[s], Kc, Vc, lens, Kbs[s], Vbs[s], 0.7)
        _close(outs[s], Of, 1e-12, f"residual reuse, all chunks selected, step {s}")
    # nothing selected: everything is residual, i.e. the plain cached schedule
    outs = ora.residual_block(Qs, Kbs, Vbs, Kc, Vc, lens, 0.7, (0,), 0, chunk)
    cached, _ = ora.cached_block(Qs, Kbs, Vbs, Kc, Vc, lens, 0.7, (0,))
    for s in range(3):
        _close(outs[s], cached[s], 1e-12, f"residual reuse, no chunk selected, step {s}")
    # the complement of a selection covers every other valid chunk exactly once
    Km, valid = ora.chunk_means(Kc, lens, chunk)
    idx = ora.select_chunks(Qfix, Km, valid, 2)
    comp = ora.complement_chunks(idx, valid)
    for b in range(B):
        for kv in range(Hkv):
            a = sorted([int(c) for c in idx[b, kv] if c >= 0] + [int(c) for c in comp[b, kv] if c >= 0])
            assert a == [c for c in range(valid.shape[1]) if valid[b, c]], "selection + complement"


def _drift_block(rng, B=2, S=3, Hq=4, Hkv=2, D=4, Lcap=20, steps=4, sig=0.3):
    Kc, Vc = _rand(rng, B, Lcap, Hkv, D), _rand(rng, B, Lcap, Hkv, D)
    lens = np.array([Lcap, Lcap - 7], dtype=np.int32)[:B]
    Q0, K0, V0 = _rand(rng, B, S, Hq, D), _rand(rng, B, S, Hkv, D), _rand(rng, B, S, Hkv, D)
    Qs = [Q0 + sig * _rand(rng, B, S, Hq, D) for _ in range(steps)]
    Ks = [K0 + sig * _rand(rng, B, S, Hkv, D) for _ in range(steps)]
    Vs = [V0 + sig * _rand(rng, B, S, Hkv, D) for _ in range(steps)]
    return Kc, Vc, lens, Qs, Ks, Vs


def pin_headwise_refresh(ora):
    """gamma above 1 refreshes every unit every step (= full attention);
    gamma at -1 never refreshes after step 0 (= the cached schedule); the
    similarity is 1 for identical queries and symmetric."""
    rng = np.random.default_rng(22)
    Kc, Vc, lens, Qs, Ks, Vs = _drift_block(rng)
    outs, masks = ora.headwise_block(Qs, Ks, Vs, Kc, Vc, lens, 0.6, 1.5)
    for s in range(len(Qs)):
        Of, _ = ora.full_attention(Qs[s], Kc, Vc, lens, Ks[s], Vs[s], 0.6)
        _close(outs[s], Of, 1e-12, f"head-wise, gamma 1.5, step {s}")
        assert masks[s].all()
    outs, masks = ora.headwise_block(Qs, Ks, Vs, Kc, Vc, lens, 0.6, -1.0)
    cached, _ = ora.cached_block(Qs, Ks, Vs, Kc, Vc, lens, 0.6, (0,))
    for s in range(len(Qs)):
        _close(outs[s], cached[s], 1e-12, f"head-wise, gamma -1, step {s}")
        assert masks[s].all() if s == 0 else not masks[s].any()
    # refresh decisions: a big query jump refreshes, a repeat of the new
    # queries then reuses (the reference moved with the refresh)
    Qj = [Qs[0], Qs[0] + 5.0 * _rand(rng, *Qs[0].shape)]
    Qj.append(Qj[1].copy())
    outs, masks = ora.headwise_block(Qj, Ks[:3], Vs[:3], Kc, Vc, lens, 0.6, 0.999)
    assert masks[1].all() and not masks[2].any(), [m.tolist() for m in masks]
    sim = ora.unit_query_similarity(Qs[1], Qs[2], 2)
    _close(sim, ora.unit_query_similarity(Qs[2], Qs[1], 2), 1e-14, "similarity symmetric")
    _close(ora.unit_query_similarity(Qs[1], Qs[1], 2), np.ones((2, 2)), 1e-14, "self-similarity")
    # a unit whose queries are a positive multiple of the reference: similarity 1
    _close(ora.unit_query_similarity(3.0 * Qs[1], Qs[1], 2), np.ones((2, 2)), 1e-14, "scale invariance")


def pin_threshold_refresh(ora):
    """tau = 0 refreshes every step (= full attention); tau above S never
    refreshes (= the cached schedule); the updated-token count by hand."""
    rng = np.random.default_rng(23)
    Kc, Vc, lens, Qs, Ks, Vs = _drift_block(rng)
    outs, flags = ora.threshold_block(Qs, Ks, Vs, Kc, Vc, lens, 0.6, 0, 1e-3)
    for s in range(len(Qs)):
        Of, _ = ora.full_attention(Qs[s], Kc, Vc, lens, Ks[s], Vs[s], 0.6)
        _close(outs[s], Of, 1e-12, f"threshold, tau 0, step {s}")
    outs, flags = ora.threshold_block(Qs, Ks, Vs, Kc, Vc, lens, 0.6, 99, 1e-3)
    cached, _ = ora.cached_block(Qs, Ks, Vs, Kc, Vc, lens, 0.6, (0,))
    for s in range(len(Qs)):
        _close(outs[s], cached[s], 1e-12, f"threshold, tau 99, step {s}")
    K1, V1 = Ks[0].copy(), Vs[0].copy()
    K1[0, 1, 1, 2] += 0.5      # token 1 of sequence 0 moves in K
    V1[1, 0, 0, 0] -= 0.01     # token 0 of sequence 1 moves a little in V
    V1[1, 2, 1, 3] += 0.2      # token 2 of sequence 1 moves in V
    m = ora.updated_tokens(Ks[0], Vs[0], K1, V1, 0.05)
    assert m.tolist() == [1, 1], m


def pin_selection_ties(ora):
    """Equal scores: the lower chunk index wins."""
    D = 2
    Q = np.ones((1, 1, 1, D))
    # chunks 0..3 with means giving scores 1, 2, 2, 1 -> top-2 = {1, 2}; top-1 = {1}
    Km = np.array([[[[0.5, 0.5], [1.0, 1.0], [1.0, 1.0], [0.5, 0.5]]]])
    valid = np.ones((1, 4), dtype=bool)
    assert ora.select_chunks(Q, Km, valid, 1)[0, 0].tolist() == [1]
    assert ora.select_chunks(Q, Km, valid, 2)[0, 0].tolist() == [1, 2]
    assert ora.select_chunks(Q, Km, valid, 3)[0, 0].tolist() == [0, 1, 2]
    valid[0, 0] = False
    assert ora.select_chunks(Q, Km, valid, 4)[0, 0].tolist() == [1, 2, 3, -1]


ALL_PINS = [pin_brute_partial, pin_brute_layer, pin_golden, pin_closed_forms,
            pin_merge_is_concat, pin_merge_algebra, pin_refresh_step_exact,
            pin_reuse_unchanged_queries, pin_refresh_recomputes, pin_rows_sum_to_one, pin_sparse,
            pin_residual_reuse, pin_headwise_refresh, pin_threshold_refresh, pin_selection_ties]


def failing_pins(ora):
    """Names of the pins that the given oracle namespace fails."""
    bad = []
    for pin in ALL_PINS:
        try:
            pin(ora)
        except (AssertionError, ValueError, IndexError, FloatingPointError) as e:  # noqa: PERF203
            bad.append((pin.__name__, str(e)[:120]))
    return bad
