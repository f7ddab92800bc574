"""Pure-Python brute force for tiny inputs: plain loops, math.exp, no max trick.

Used only to pin the oracle (it shares nothing with it beyond the definition of
softmax attention written out term by term).
"""
import math


def partial(q_rows, keys, vals, scale):
    """Rows of softmax attention computed term by term: (o rows, lse list)."""
    outs, lses = [], []
    for q in q_rows:
        ws = []
        for k in keys:
            z = 0.0
            for a, b in zip(q, k):
                z += a * b
            ws.append(math.exp(scale * z))
        if not ws:
            outs.append([0.0] * (len(vals[0]) if vals else 0))
            lses.append(-math.inf)
            continue
        Z = 0.0
        for w in ws:
            Z += w
        o = []
        for d in range(len(vals[0])):
            acc = 0.0
            for w, v in zip(ws, vals):
                acc += w * v[d]
            o.append(acc / Z)
        outs.append(o)
        lses.append(math.log(Z))
    return outs, lses


def tolist(a):
    return [list(map(float, r)) for r in a]


def layer_full(Q, Kc, Vc, lens, Kb, Vb, scale):
    """Brute-force uncached attention over [prefix ; block] for every (b, t, h)."""
    B, S, Hq, D = Q.shape
    Hkv = Kc.shape[2]
    G = Hq // Hkv
    O, LSE = {}, {}
    for b in range(B):
        for h in range(Hq):
            kv = h // G
            keys = tolist(Kc[b, :lens[b], kv]) + tolist(Kb[b, :, kv])
            vals = tolist(Vc[b, :lens[b], kv]) + tolist(Vb[b, :, kv])
            o, l = partial(tolist(Q[b, :, h]), keys, vals, scale)
            for t in range(S):
                O[(b, t, h)] = o[t]
                LSE[(b, h, t)] = l[t]
    return O, LSE


def chunk_select(Q, Kc, lens, chunk, topk):
    """Brute-force chunk means, scores and top-k (ties to the lower index)."""
    B, S, Hq, D = Q.shape
    Lcap, Hkv = Kc.shape[1], Kc.shape[2]
    G = Hq // Hkv
    nch = -(-Lcap // chunk)
    out = {}
    for b in range(B):
        for kv in range(Hkv):
            qbar = [0.0] * D
            for t in range(S):
                for g in range(G):
                    for d in range(D):
                        qbar[d] += float(Q[b, t, kv * G + g, d])
            qbar = [x / (S * G) for x in qbar]
            scored = []
            for c in range(nch):
                lo, hi = c * chunk, min((c + 1) * chunk, int(lens[b]))
                if hi <= lo:
                    continue
                kbar = [0.0] * D
                for j in range(lo, hi):
                    for d in range(D):
                        kbar[d] += float(Kc[b, j, kv, d])
                kbar = [x / (hi - lo) for x in kbar]
                s = 0.0
                for d in range(D):
                    s += qbar[d] * kbar[d]
                scored.append((s, c))
            chosen = []
            for s, c in scored:
                better = 0
                for s2, c2 in scored:
                    if s2 > s or (s2 == s and c2 < c):
                        better += 1
                if better < topk:
                    chosen.append(c)
            out[(b, kv)] = sorted(chosen)
    return out
