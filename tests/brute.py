"""Brute-force restatements for tiny inputs (pure Python loops, fp64).

These enumerate every (query, key) pair and rank with a full sort of
(-score, index) tuples. They are a second, independent route to the same
definitions the oracle vectorises, used only to pin the oracle on small N.
"""
import math


def dot(a, b):
    return sum(x * y for x, y in zip(a, b))


def block_scores_bf(qt, kt, block):
    """{(i, j): max over causal pairs} for every query block i and key block j <= i."""
    n = len(qt)
    nb = n // block
    out = {}
    for i in range(nb):
        for j in range(i + 1):
            best = -math.inf
            for t in range(i * block, (i + 1) * block):
                for u in range(j * block, (j + 1) * block):
                    if u <= t:
                        best = max(best, dot(qt[t], kt[u]))
            out[(i, j)] = best
    return out


def topk_bf(scores_by_index, k):
    """Full sort of (-score, index); the first k indices, ascending."""
    ranked = sorted(scores_by_index.items(), key=lambda kv: (-kv[1], kv[0]))
    return sorted(idx for idx, _ in ranked[:k])


def softmax_attend_bf(q, keys, values, scale):
    logits = [scale * dot(q, kk) for kk in keys]
    m = max(logits)
    w = [math.exp(l - m) for l in logits]
    s = sum(w)
    D = len(values[0])
    return [sum(w[n] * values[n][d] for n in range(len(keys))) / s for d in range(D)]


def prefill_head_bf(q, k, v, qt, kt, topk, window_blocks, sink_blocks, block, scale):
    """Full pipeline for one retrieval head: rows [N][D] lists. Returns (sel, out)."""
    n = len(q)
    nb = n // block
    bs = block_scores_bf(qt, kt, block)
    sel, out = {}, [None] * n
    for i in range(nb):
        cand = {j: bs[(i, j)] for j in range(i + 1)}
        sel[i] = topk_bf(cand, topk)
        att = set(sel[i]) | set(range(min(sink_blocks, i + 1))) | \
            set(range(max(0, i - window_blocks + 1), i + 1))
        for t in range(i * block, (i + 1) * block):
            keys = [u for j in sorted(att) for u in range(j * block, (j + 1) * block) if u <= t]
            out[t] = softmax_attend_bf(q[t], [k[u] for u in keys], [v[u] for u in keys], scale)
    return sel, out


def swa_bf(q, k, v, window, scale):
    out = []
    for t in range(len(q)):
        keys = [u for u in range(len(k)) if t - window < u <= t]
        out.append(softmax_attend_bf(q[t], [k[u] for u in keys], [v[u] for u in keys], scale))
    return out


def decode_bf(q, kc, vc, qt, kt, topk, window, sink, scale):
    L = len(kc)
    scores = {u: dot(qt, kt[u]) for u in range(L)}
    sel = topk_bf(scores, topk)
    att = sorted(set(sel) | set(range(min(sink, L))) | set(range(max(0, L - window), L)))
    return sel, softmax_attend_bf(q, [kc[u] for u in att], [vc[u] for u in att], scale)
