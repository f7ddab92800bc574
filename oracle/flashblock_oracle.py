"""Float64 CPU oracle for FlashBlock cached block-diffusion attention.

TEST INFRASTRUCTURE ONLY.  Nothing on the product path may import, call or run
this module: only the tests, ``__graft_entry__.smoke()`` and the ``cpu_baseline``
/ ``--impl reference`` legs of ``bench.py`` use it.  It shares no code with the
CUDA library (no kernels, headers, helpers, tables or pre/post-processing) and
imports nothing from the package.

Source of every definition: the page "FlashBlock: Attention Caching for
Efficient Long-Context Block Diffusion" (gist.science explainer of arXiv
2602.05305), Technical Summary:

* §1 Problem Statement -- standard block diffusion recomputes attention over
  the whole growing KV cache at every denoising step (the uncached baseline,
  :func:`full_attention`).
* §2 Methodology, Core Mechanism -- attention is split into a block-internal
  partial over the current block's tokens J_in and a block-external partial
  over the tokens outside it, J_out (:func:`attention_partial`); the external
  pair (A_out, L_out = log Z_out) is cached and reused on later steps; the two
  are recombined with the log-space merge equation (:func:`merge_partials`).
* §2 Methodology, Adaptive Reuse Strategies, "Compatibility with Sparse
  Attention" -- unselected sparse keys play the role of J_out
  (:func:`select_chunks`, :func:`chunk_token_positions`); their cached
  residual is merged with the freshly computed selected keys
  (:func:`complement_chunks`, :func:`residual_block`).
* §2 Methodology, Adaptive Reuse Strategies, "Threshold-based Reuse" and
  "Head-wise Selection" -- refresh decisions by updated-token count tau and by
  per-head similarity gamma (:func:`threshold_block`, :func:`headwise_block`).

Readings where the page is silent:
  L is the natural log of the unnormalised sum Z; J_out is the finalized
  prefix; the block is attended bidirectionally with no mask; query head h
  reads KV head h // G; an empty key set gives (O = 0, L = -inf); the sparse
  chunk score is mean(block Q over tokens and group heads) . mean(chunk keys),
  top-k by descending score with ties broken towards the lower chunk index,
  returned in ascending chunk order and padded with -1; head-wise
  similarity is the cosine of a (b, kv head) unit's block queries against
  the queries its cached pair was computed with; an updated token is a block
  token whose K or V moved by more than eps since the previous step.

Arrays are float64 numpy.  Layouts follow the C library's:
  Q, O           [B, S, Hq, D]
  K/V cache      [B, Lcap, Hkv, D]   (valid rows j < prefix_lens[b])
  K/V block      [B, S, Hkv, D]
  LSE            [B, Hq, S]          natural log
"""
from __future__ import annotations

import numpy as np

NEG_INF = -np.inf


# ---------------------------------------------------------------------------
# Core mechanism: one attention partial and the log-space merge
# ---------------------------------------------------------------------------

def attention_partial(q, k, v, scale):
    """Softmax attention of query rows over one key set.

    Core Mechanism (Technical Summary §2): a partial over a token set J is the
    pair (A_J, L_J) with z_j = scale * q . k_j, Z_J = sum_j exp(z_j),
    L_J = log Z_J and A_J = sum_j exp(z_j) v_j / Z_J.

    q: [R, D], k: [N, D], v: [N, Dv]  ->  (o [R, Dv], lse [R]).
    N == 0 gives o = 0 and lse = -inf (an empty sum).
    """
    q = np.asarray(q, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)
    v = np.asarray(v, dtype=np.float64)
    rows = q.shape[0]
    if k.shape[0] == 0:
        return np.zeros((rows, v.shape[1])), np.full(rows, NEG_INF)
    z = scale * (q @ k.T)                       # [R, N] logits
    m = z.max(axis=1, keepdims=True)            # subtract the row max before exp
    e = np.exp(z - m)
    zsum = e.sum(axis=1)
    lse = m[:, 0] + np.log(zsum)
    o = (e @ v) / zsum[:, None]
    return o, lse


def merge_partials(o_a, lse_a, o_b, lse_b):
    """Log-space composition of two partials (Core Mechanism, merge equation).

    With m = max(L_a, L_b):
        A = (e^{L_a - m} A_a + e^{L_b - m} A_b) / (e^{L_a - m} + e^{L_b - m})
    and the merged normaliser is L = m + log(e^{L_a - m} + e^{L_b - m}).
    Rows where both sides are empty (L = -inf) stay empty: A = 0, L = -inf.

    o_*: [..., Dv], lse_*: [...]  ->  (o, lse) of the same shapes.
    """
    o_a = np.asarray(o_a, dtype=np.float64)
    o_b = np.asarray(o_b, dtype=np.float64)
    lse_a = np.asarray(lse_a, dtype=np.float64)
    lse_b = np.asarray(lse_b, dtype=np.float64)
    m = np.maximum(lse_a, lse_b)
    empty = np.isneginf(m)
    m_safe = np.where(empty, 0.0, m)
    w_a = np.where(np.isneginf(lse_a), 0.0, np.exp(lse_a - m_safe))
    w_b = np.where(np.isneginf(lse_b), 0.0, np.exp(lse_b - m_safe))
    den = w_a + w_b
    den_safe = np.where(empty, 1.0, den)
    o = (w_a[..., None] * o_a + w_b[..., None] * o_b) / den_safe[..., None]
    o = np.where(empty[..., None], 0.0, o)
    lse = np.where(empty, NEG_INF, m_safe + np.log(den_safe))
    return o, lse


# ---------------------------------------------------------------------------
# Key sets of one attention layer
# ---------------------------------------------------------------------------

def _group(hq, hkv):
    if hq % hkv:
        raise ValueError("num_q_heads must be a multiple of num_kv_heads")
    return hq // hkv


def chunk_token_positions(chunk_idx_row, chunk_size, prefix_len):
    """Cache positions covered by a list of selected chunks (ascending, -1 = unused).

    Each chunk c covers [c*chunk_size, (c+1)*chunk_size) clipped to prefix_len.
    """
    pos = []
    for c in chunk_idx_row:
        c = int(c)
        if c < 0:
            continue
        lo = c * chunk_size
        hi = min((c + 1) * chunk_size, int(prefix_len))
        pos.extend(range(lo, hi))
    return np.asarray(pos, dtype=np.int64)


def prefix_partial(Q, Kc, Vc, prefix_lens, scale, chunk_idx=None, chunk_size=256):
    """Block-external partial (A_out, L_out) over the finalized prefix.

    Core Mechanism: J_out is every token outside the current block; with
    block-causal generation these are the finalized prefix tokens
    j < prefix_lens[b].  With ``chunk_idx`` [B, Hkv, topk] (sparse prefix), the
    key set of KV head (b, kvh) is the union of the listed chunks' valid tokens.

    Returns O_pre [B, S, Hq, D] and LSE_pre [B, Hq, S].
    """
    B, S, Hq, D = Q.shape
    Hkv = Kc.shape[2]
    Dv = Vc.shape[3]
    G = _group(Hq, Hkv)
    O = np.zeros((B, S, Hq, Dv))
    LSE = np.full((B, Hq, S), NEG_INF)
    for b in range(B):
        L = int(prefix_lens[b])
        for kvh in range(Hkv):
            if chunk_idx is None:
                pos = np.arange(L)
            else:
                pos = chunk_token_positions(chunk_idx[b, kvh], chunk_size, L)
            k = Kc[b, pos, kvh, :]
            v = Vc[b, pos, kvh, :]
            for g in range(G):
                h = kvh * G + g
                o, lse = attention_partial(Q[b, :, h, :], k, v, scale)
                O[b, :, h, :] = o
                LSE[b, h, :] = lse
    return O, LSE


def inblock_partial(Q, Kb, Vb, scale):
    """Block-internal partial (A_in, L_in): bidirectional attention of the block's
    queries over the block's own keys, no mask (Core Mechanism, J_in)."""
    B, S, Hq, D = Q.shape
    Hkv = Kb.shape[2]
    G = _group(Hq, Hkv)
    O = np.zeros((B, S, Hq, Vb.shape[3]))
    LSE = np.zeros((B, Hq, S))
    for b in range(B):
        for h in range(Hq):
            o, lse = attention_partial(Q[b, :, h, :], Kb[b, :, h // G, :], Vb[b, :, h // G, :], scale)
            O[b, :, h, :] = o
            LSE[b, h, :] = lse
    return O, LSE


def block_step(Q, Kb, Vb, O_pre, LSE_pre, scale):
    """One cached denoising step: fresh in-block partial merged with the cached
    block-external pair (Core Mechanism, merge equation).

    Returns O [B, S, Hq, D] and the merged LSE [B, Hq, S].
    """
    O_in, LSE_in = inblock_partial(Q, Kb, Vb, scale)
    # LSE is [B, Hq, S]; move it to [B, S, Hq] to sit beside O's row layout.
    lp = np.transpose(LSE_pre, (0, 2, 1))
    li = np.transpose(LSE_in, (0, 2, 1))
    o, lse = merge_partials(O_pre, lp, O_in, li)
    return o, np.transpose(lse, (0, 2, 1))


def full_attention(Q, Kc, Vc, prefix_lens, Kb, Vb, scale):
    """Uncached block diffusion (Problem Statement): attention of the block's
    queries over the concatenation [prefix tokens ; block tokens], computed in
    one softmax from the definition -- no partials, no merge."""
    B, S, Hq, D = Q.shape
    Hkv = Kc.shape[2]
    G = _group(Hq, Hkv)
    O = np.zeros((B, S, Hq, Vc.shape[3]))
    LSE = np.zeros((B, Hq, S))
    for b in range(B):
        L = int(prefix_lens[b])
        for kvh in range(Hkv):
            k = np.concatenate([Kc[b, :L, kvh, :], Kb[b, :, kvh, :]], axis=0)
            v = np.concatenate([Vc[b, :L, kvh, :], Vb[b, :, kvh, :]], axis=0)
            for g in range(G):
                h = kvh * G + g
                o, lse = attention_partial(Q[b, :, h, :], k, v, scale)
                O[b, :, h, :] = o
                LSE[b, h, :] = lse
    return O, LSE


# ---------------------------------------------------------------------------
# Sparse prefix: chunk means and top-k chunk selection
# ---------------------------------------------------------------------------

def chunk_means(Kc, prefix_lens, chunk_size):
    """Mean key of every chunk over its valid tokens.

    Returns Kmean [B, Hkv, nchunks, D] (nchunks = ceil(Lcap / chunk_size)) and
    a mask valid [B, nchunks]: a chunk is valid iff it holds at least one
    token j < prefix_lens[b].  Invalid chunks have mean 0.
    """
    B, Lcap, Hkv, D = Kc.shape
    nch = -(-Lcap // chunk_size)
    Km = np.zeros((B, Hkv, nch, D))
    valid = np.zeros((B, nch), dtype=bool)
    for b in range(B):
        L = int(prefix_lens[b])
        for c in range(nch):
            lo, hi = c * chunk_size, min((c + 1) * chunk_size, L)
            if hi <= lo:
                continue
            valid[b, c] = True
            Km[b, :, c, :] = Kc[b, lo:hi, :, :].mean(axis=0)
    return Km, valid


def chunk_scores(Q, Kmean, valid):
    """score[b, kvh, c] = qbar . kbar_c, qbar the mean of the block's queries over
    its S tokens and the G query heads of the group.  Invalid chunks: -inf."""
    B, S, Hq, D = Q.shape
    Hkv = Kmean.shape[1]
    G = _group(Hq, Hkv)
    sc = np.full(Kmean.shape[:3], NEG_INF)
    for b in range(B):
        for kvh in range(Hkv):
            qbar = Q[b, :, kvh * G:(kvh + 1) * G, :].reshape(S * G, D).mean(axis=0)
            s = Kmean[b, kvh] @ qbar
            sc[b, kvh] = np.where(valid[b], s, NEG_INF)
    return sc


def select_chunks(Q, Kmean, valid, topk):
    """Top-k chunks per (b, kvh) by score, ties to the lower chunk index.

    Returns idx [B, Hkv, topk] int32 in ascending chunk order, padded with -1
    when fewer than topk chunks are valid.
    """
    sc = chunk_scores(Q, Kmean, valid)
    B, Hkv, nch = sc.shape
    idx = np.full((B, Hkv, topk), -1, dtype=np.int32)
    for b in range(B):
        for kvh in range(Hkv):
            cand = [c for c in range(nch) if valid[b, c]]
            # stable sort on -score keeps lower index first among equal scores
            order = sorted(cand, key=lambda c: (-sc[b, kvh, c], c))
            chosen = sorted(order[:topk])
            idx[b, kvh, :len(chosen)] = chosen
    return idx


# ---------------------------------------------------------------------------
# The cached schedule of one block (Core Mechanism: reuse from the last refresh)
# ---------------------------------------------------------------------------

def cached_block(Qs, Kbs, Vbs, Kc, Vc, prefix_lens, scale, refresh_steps,
                 chunk_idx_fn=None, chunk_size=256):
    """Run one block of denoising steps the FlashBlock way.

    At a refresh step the block-external pair is recomputed with that step's
    queries; on the other steps the pair from the most recent refresh is
    reused and only the in-block partial and the merge are fresh.

    Qs/Kbs/Vbs: lists over steps of [B, S, *, D].  ``chunk_idx_fn(Q)`` returns
    the sparse chunk list for a refresh-step Q (or None for a dense prefix).
    Returns (list of O_s, list of (O_pre, LSE_pre) used at each step).
    """
    outs, pres = [], []
    pre = None
    for s, Q in enumerate(Qs):
        if s in refresh_steps or pre is None:
            idx = None if chunk_idx_fn is None else chunk_idx_fn(Q)
            pre = prefix_partial(Q, Kc, Vc, prefix_lens, scale, idx, chunk_size)
        o, _ = block_step(Q, Kbs[s], Vbs[s], pre[0], pre[1], scale)
        outs.append(o)
        pres.append(pre)
    return outs, pres


def complement_chunks(chunk_idx, valid):
    """The valid chunks a selection leaves out: [B, Hkv, nchunks] int32,
    ascending, padded with -1 (Compatibility with Sparse Attention: the
    unselected keys form the block-external set whose contribution is
    cached)."""
    B, Hkv, _ = chunk_idx.shape
    nch = valid.shape[1]
    comp = np.full((B, Hkv, nch), -1, dtype=np.int32)
    for b in range(B):
        for kvh in range(Hkv):
            chosen = set(int(c) for c in chunk_idx[b, kvh] if c >= 0)
            rest = [c for c in range(nch) if valid[b, c] and c not in chosen]
            comp[b, kvh, :len(rest)] = rest
    return comp


def residual_block(Qs, Kbs, Vbs, Kc, Vc, prefix_lens, scale, refresh_steps, topk, chunk_size=256):
    """One block with sparse attention and residual reuse (Adaptive Reuse
    Strategies, Compatibility with Sparse Attention).

    At a refresh step the top-k chunks are selected with that step's queries
    and the partial over the *unselected* chunks (the residual) is computed
    and cached.  Every step recomputes the partial over the selected chunks
    with its own queries and merges three partials: residual, selected and
    in-block.  Returns the list of O_s.
    """
    outs = []
    res = idx = None
    Km, valid = chunk_means(Kc, prefix_lens, chunk_size)
    for s, Q in enumerate(Qs):
        if s in refresh_steps or res is None:
            idx = select_chunks(Q, Km, valid, topk)
            comp = complement_chunks(idx, valid)
            res = prefix_partial(Q, Kc, Vc, prefix_lens, scale, comp, chunk_size)
        sel = prefix_partial(Q, Kc, Vc, prefix_lens, scale, idx, chunk_size)
        o_pre, l_pre = merge_partials(res[0], np.transpose(res[1], (0, 2, 1)),
                                      sel[0], np.transpose(sel[1], (0, 2, 1)))
        o, _ = block_step(Q, Kbs[s], Vbs[s], o_pre, np.transpose(l_pre, (0, 2, 1)), scale)
        outs.append(o)
    return outs


def unit_query_similarity(Q, Qref, hkv):
    """Cosine similarity per (b, kv head) unit between the block's queries now
    and the queries the unit's cached pair was computed with, over the unit's
    S x G x D values ([B, Hkv])."""
    B, S, Hq, D = Q.shape
    G = _group(Hq, hkv)
    sim = np.zeros((B, hkv))
    for b in range(B):
        for kvh in range(hkv):
            a = Q[b, :, kvh * G:(kvh + 1) * G, :].ravel()
            r = Qref[b, :, kvh * G:(kvh + 1) * G, :].ravel()
            den = np.linalg.norm(a) * np.linalg.norm(r)
            sim[b, kvh] = (a @ r) / den if den > 0 else 1.0
    return sim


def headwise_block(Qs, Kbs, Vbs, Kc, Vc, prefix_lens, scale, gamma):
    """Head-wise selective reuse (Adaptive Reuse Strategies, Head-wise
    Selection): step 0 computes every unit's block-external pair; at a later
    step a (b, kv head) unit reuses its pair only if the similarity of its
    queries to the ones the pair was computed with is at least gamma,
    otherwise its pair is recomputed with the current queries.
    Returns (list of O_s, list of refresh masks [B, Hkv])."""
    B, S, Hq, D = Qs[0].shape
    Hkv = Kc.shape[2]
    G = _group(Hq, Hkv)
    Op, Lp = prefix_partial(Qs[0], Kc, Vc, prefix_lens, scale)
    Qref = Qs[0].copy()
    outs, masks = [], []
    for s, Q in enumerate(Qs):
        if s == 0:
            mask = np.ones((B, Hkv), dtype=bool)
        else:
            mask = unit_query_similarity(Q, Qref, Hkv) < gamma
            if mask.any():
                On, Ln = prefix_partial(Q, Kc, Vc, prefix_lens, scale)
                for b in range(B):
                    for kvh in range(Hkv):
                        if mask[b, kvh]:
                            hs = slice(kvh * G, (kvh + 1) * G)
                            Op[b, :, hs] = On[b, :, hs]
                            Lp[b, hs] = Ln[b, hs]
                            Qref[b, :, hs] = Q[b, :, hs]
        o, _ = block_step(Q, Kbs[s], Vbs[s], Op, Lp, scale)
        outs.append(o)
        masks.append(mask)
    return outs, masks


def updated_tokens(Kprev, Vprev, Know, Vnow, eps):
    """M: per sequence, the block tokens whose key or value moved by more than
    eps (max abs change over heads and dims) since the previous step ([B])."""
    dk = np.abs(Know - Kprev).max(axis=(2, 3))
    dv = np.abs(Vnow - Vprev).max(axis=(2, 3))
    return ((dk > eps) | (dv > eps)).sum(axis=1)


def threshold_block(Qs, Kbs, Vbs, Kc, Vc, prefix_lens, scale, tau, eps):
    """Threshold-based reuse (Adaptive Reuse Strategies): step 0 refreshes;
    at step s + 1 a sequence keeps its block-external pair while its count
    M^{s+1} of tokens changed since step s stays under tau, and recomputes it
    otherwise.
    Returns (list of O_s, list of per-sequence refresh flags [B])."""
    B, S, Hq, D = Qs[0].shape
    Op, Lp = prefix_partial(Qs[0], Kc, Vc, prefix_lens, scale)
    outs, flags = [], []
    for s, Q in enumerate(Qs):
        if s == 0:
            flag = np.ones(B, dtype=bool)
        else:
            flag = updated_tokens(Kbs[s - 1], Vbs[s - 1], Kbs[s], Vbs[s], eps) >= tau
            if flag.any():
                On, Ln = prefix_partial(Q, Kc, Vc, prefix_lens, scale)
                Op[flag] = On[flag]
                Lp[flag] = Ln[flag]
        o, _ = block_step(Q, Kbs[s], Vbs[s], Op, Lp, scale)
        outs.append(o)
        flags.append(flag)
    return outs, flags


def attention_weights(q, k, scale):
    """Explicit softmax weight matrix e^{z - L} of one partial ([R, N])."""
    _, lse = attention_partial(q, k, np.zeros((k.shape[0], 1)), scale)
    z = scale * (np.asarray(q, np.float64) @ np.asarray(k, np.float64).T)
    return np.exp(z - lse[:, None])


__all__ = [
    "NEG_INF", "attention_partial", "merge_partials", "chunk_token_positions",
    "prefix_partial", "inblock_partial", "block_step", "full_attention",
    "chunk_means", "chunk_scores", "select_chunks", "cached_block",
    "complement_chunks", "residual_block", "unit_query_similarity", "headwise_block",
    "updated_tokens", "threshold_block", "attention_weights",
]
