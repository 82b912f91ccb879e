"""Plain fp64 CPU oracle for RTPurbo-style head-wise hybrid attention.

TEST INFRASTRUCTURE. Only ``tests/``, ``__graft_entry__.smoke()`` and the
benchmark's CPU-baseline leg use this module. The CUDA library never imports
it and it shares no code with the CUDA sources.

What it computes, step by step (the sources, by page and paragraph):

* Head-wise split: about 15% of heads are retrieval heads, the rest are
  streaming heads that run sliding-window attention with a window of 8192
  (RTPurboV2 article, th-motor.com: the paragraphs on retrieval vs streaming
  heads and on the Qwen3-Coder-30B-A3B recipe). The split is an input here.
* Indexer: a per-KV-head low-rank projector maps the head dimension D to
  r = 16 (RTPurboV2 article, paragraph on the low-rank projector); it is a
  cheap scout whose scores pick candidates, after which exact attention runs
  at full dimension on the small selected set (RTPurbo digest, Telegram
  channel "Data analysis", post 5185).
* Block score for prefill: the maximum of the projected dot product over the
  (query, key) pairs of a 64 x 64 block pair; each query block keeps its top-k
  causal key blocks plus key block 0 (the sink) plus the window blocks (the
  tiny 2K-token prefill workload statement).
* Decode: token-level top-k over the whole cache by the projected score,
  unioned with the last W tokens and token 0, then exact softmax attention
  (the 128K-context decode workload statement).

Readings taken where the sources are silent (each one is used identically by
the CUDA path, which is written separately from the same text):

* softmax scale ``1/sqrt(D)`` is passed explicitly as ``scale``;
* query head ``h`` reads KV head ``h // (Hq/Hkv)``; its projector is that KV
  head's;
* inputs are taken as already position-encoded (no RoPE is applied);
* prefill top-k ranks *every* causal key block ``j <= i`` (sink and window
  blocks included), and only then is the union with sink and window taken;
* the block score of the diagonal block uses causal pairs only (``u <= t``);
* the retrieval heads' prefill window is block-granular: the ``W/64`` key
  blocks ending at the diagonal block, with the causal mask inside the
  diagonal block;
* the SWA window holds ``W`` keys including the query itself,
  ``t - W < u <= t``;
* keys are a set: a key reached twice (selected and in the window) counts once;
* exact score ties rank the smaller index first;
* the stored key index and the prefill query index are rounded to bf16
  (round-to-nearest-even of the exact sum); the decode query index stays
  unrounded (fp32 on the GPU, fp64 here);
* when fewer candidates than ``k`` exist, all are taken (``-1`` pads the rest).

Parity pins live in ``tests/test_oracle_pins.py``; every function below is
pinned there (no function here is parity unpinned).
"""
from __future__ import annotations

import numpy as np

BLOCK = 64


# ---------------------------------------------------------------------------
# bf16 rounding
# ---------------------------------------------------------------------------
def bf16_round(x) -> np.ndarray:
    """Round fp64 values to the nearest bf16 value, ties to even.

    bf16 keeps 8 significant bits and fp32's exponent range; below 2**-126 the
    spacing is fixed at 2**-133 (subnormals). Returned as fp64.
    """
    x = np.asarray(x, dtype=np.float64)
    out = np.zeros_like(x)
    nz = x != 0
    _, e = np.frexp(x[nz])                       # x = m * 2**e, 0.5 <= |m| < 1
    exp_unbiased = np.maximum(e - 1, -126)       # floor(log2|x|), clamped at the subnormal range
    quantum = np.ldexp(1.0, exp_unbiased - 7)    # spacing of 8 significant bits
    out[nz] = np.rint(x[nz] / quantum) * quantum  # np.rint: round half to even
    return out


def to_f64(t) -> np.ndarray:
    """A torch tensor or array (any float dtype) as fp64 numpy (bf16 -> fp64 is exact)."""
    try:
        import torch
        if isinstance(t, torch.Tensor):
            return t.detach().to("cpu").to(torch.float64).numpy()
    except ImportError:  # pragma: no cover
        pass
    return np.asarray(t, dtype=np.float64)


# ---------------------------------------------------------------------------
# Index projection (low-rank projector D -> r)
# ---------------------------------------------------------------------------
def project(x, P, round_to_bf16: bool = True) -> np.ndarray:
    """x_tilde = x @ P for rows ``x[..., D]`` and one projector ``P[D, r]``.

    The sum is taken in fp64 (every bf16 x bf16 product is exact there), then
    rounded once to bf16 when the result is a stored index.
    """
    y = np.matmul(to_f64(x), to_f64(P))
    return bf16_round(y) if round_to_bf16 else y


# ---------------------------------------------------------------------------
# Prefill selection
# ---------------------------------------------------------------------------
def block_scores(qt, kt, i: int, block: int = BLOCK, key_chunk_blocks: int = 4096) -> np.ndarray:
    """s[j] for j = 0..i: max over causal pairs (t in query block i, u in key
    block j, u <= t) of qt[t] . kt[u].

    ``qt`` [N, r] and ``kt`` [N, r] are one head's projected queries and keys.
    The keys are visited in chunks of ``key_chunk_blocks`` blocks only to bound
    the temporary; a maximum does not depend on the order it is taken in.
    """
    qt = to_f64(qt)
    kt = to_f64(kt)
    qb = qt[i * block:(i + 1) * block]                       # [64, r]
    t_pos = np.arange(i * block, (i + 1) * block)
    out = np.empty(i + 1)
    for j0 in range(0, i + 1, key_chunk_blocks):
        j1 = min(i + 1, j0 + key_chunk_blocks)
        kb = kt[j0 * block:j1 * block]                       # [(j1-j0)*64, r]
        s = qb @ kb.T                                        # [64, (j1-j0)*64]
        u_pos = np.arange(j0 * block, j1 * block)
        s = np.where(u_pos[None, :] <= t_pos[:, None], s, -np.inf)
        out[j0:j1] = s.reshape(block, j1 - j0, block).max(axis=(0, 2))
    return out


def topk_desc(scores, k: int) -> np.ndarray:
    """Indices of the k largest scores (ties: smaller index first), ascending.

    With ``len(scores) <= k`` every index is returned.
    """
    scores = np.asarray(scores, dtype=np.float64)
    n = scores.shape[0]
    if n <= k:
        return np.arange(n, dtype=np.int64)
    order = np.lexsort((np.arange(n), -scores))   # primary: score desc; secondary: index asc
    return np.sort(order[:k])


def select_prefill(qt, kt, topk: int, qblocks=None, block: int = BLOCK):
    """Top-k causal key blocks for each query block of one head.

    Returns ``(sel, scores)``: dicts keyed by query block i, ``sel[i]`` the
    ascending selected block indices (min(k, i+1) of them), ``scores[i]`` the
    block scores s[0..i] used for the ranking.
    """
    N = to_f64(qt).shape[0]
    nb = N // block
    qblocks = range(nb) if qblocks is None else qblocks
    sel, scores = {}, {}
    for i in qblocks:
        s = block_scores(qt, kt, i, block)
        scores[i] = s
        sel[i] = topk_desc(s, topk)
    return sel, scores


def attended_blocks(sel_i, i: int, window_blocks: int, sink_blocks: int) -> np.ndarray:
    """Key blocks attended by query block i: selected, sink blocks and the
    window blocks ending at the diagonal, as an ascending set."""
    win = np.arange(max(0, i - window_blocks + 1), i + 1)
    sink = np.arange(0, min(sink_blocks, i + 1))
    return np.unique(np.concatenate([np.asarray(sel_i, dtype=np.int64), sink, win]))


# ---------------------------------------------------------------------------
# Exact attention
# ---------------------------------------------------------------------------
def attend(q_rows, q_pos, keys, values, key_pos, scale: float, window=None) -> np.ndarray:
    """Softmax attention of each query row over the given keys, keeping only
    keys at positions <= the query's position (and, with ``window``, only keys
    at positions > the query's position - window).

    ``q_rows`` [m, D], ``q_pos`` [m], ``keys``/``values`` [n, D], ``key_pos`` [n].
    fp64 throughout, max-subtracted exponentials.
    """
    q_rows, keys, values = to_f64(q_rows), to_f64(keys), to_f64(values)
    logits = scale * (q_rows @ keys.T)                         # [m, n]
    kp = np.asarray(key_pos)[None, :]
    qp = np.asarray(q_pos)[:, None]
    ok = kp <= qp
    if window is not None:
        ok &= kp > qp - window
    logits = np.where(ok, logits, -np.inf)
    m = logits.max(axis=1, keepdims=True)
    p = np.exp(logits - m)
    p /= p.sum(axis=1, keepdims=True)
    return p @ values


def sparse_attn_prefill_block(q, k, v, i: int, attended, scale: float,
                              block: int = BLOCK) -> np.ndarray:
    """Output rows of query block i of one retrieval head.

    ``q`` [N, D] (that head), ``k``/``v`` [N, D] (its KV head), ``attended``
    the ascending key-block set.
    """
    rows = np.arange(i * block, (i + 1) * block)
    key_pos = np.concatenate([np.arange(j * block, (j + 1) * block) for j in attended])
    return attend(to_f64(q[rows]), rows, to_f64(k[key_pos]), to_f64(v[key_pos]), key_pos, scale)


def swa_rows(q, k, v, rows, window: int, scale: float, q_pos0: int = 0) -> np.ndarray:
    """Sliding-window attention for query rows ``rows`` of one head.

    Query row t sits at position ``q_pos0 + t`` and attends the keys u with
    ``pos - window < u <= pos`` (and u inside the key array).
    """
    rows = np.asarray(rows, dtype=np.int64)
    pos = q_pos0 + rows
    Nk = k.shape[0]
    lo, hi = max(0, int(pos.min()) - window + 1), min(Nk, int(pos.max()) + 1)
    kp = np.arange(lo, hi)
    return attend(to_f64(q[rows]), pos, to_f64(k[lo:hi]), to_f64(v[lo:hi]), kp, scale, window)


# ---------------------------------------------------------------------------
# Decode
# ---------------------------------------------------------------------------
def decode_scores(qt, kt) -> np.ndarray:
    """score_u = qt . kt[u] for every cached token u (qt [r], kt [L, r])."""
    return to_f64(kt) @ to_f64(qt)


def select_decode(qt, kt, topk: int) -> np.ndarray:
    """Token-level top-k over the whole cache (ascending indices)."""
    return topk_desc(decode_scores(qt, kt), topk)


def decode_attended(sel, L: int, window: int, sink: int) -> np.ndarray:
    """Selected tokens, tokens 0..sink-1 and the last ``window`` tokens, as a set."""
    return np.unique(np.concatenate([np.asarray(sel, dtype=np.int64),
                                     np.arange(0, min(sink, L)),
                                     np.arange(max(0, L - window), L)]))


def attend_decode(q, kc, vc, keys_idx, scale: float) -> np.ndarray:
    """One query (at the last position) over the cache rows ``keys_idx``."""
    keys_idx = np.asarray(keys_idx, dtype=np.int64)
    L = kc.shape[0]
    return attend(to_f64(q)[None, :], [L - 1], to_f64(kc[keys_idx]), to_f64(vc[keys_idx]),
                  keys_idx, scale)[0]


# ---------------------------------------------------------------------------
# 8-bit key index
# ---------------------------------------------------------------------------
QGROUP = 64


def quantize_index(kt, group: int = QGROUP):
    """The 8-bit key index: symmetric int8 codes with one fp32 scale per group
    of ``group`` consecutive tokens of one KV head (the "mixed-precision index
    system" section of the Baidu article on layered long-context attention: an
    8-bit quantised indexer; the pages fix no scheme, so this is the plain one).

    ``kt`` [L, r] holds the bf16 index values; only the L // group full groups
    are quantised (a partial last group stays in bf16). Per group, in fp32
    arithmetic (so that both sides take every rounding decision alike):
    amax = max |x|, s = amax / 127 (one fp32 division), and each code is x / s
    (one fp32 division) rounded half to even and clamped to [-127, 127]; an
    all-zero group gets s = 0 and zero codes. Returns (codes [n_full*group, r]
    int8, scales [n_full] float32).
    """
    x = to_f64(kt).astype(np.float32)            # bf16 values are exact in fp32
    n_full = x.shape[0] // group
    r = x.shape[1]
    codes = np.zeros((n_full * group, r), np.int8)
    scales = np.zeros(n_full, np.float32)
    for gi in range(n_full):
        blk = x[gi * group:(gi + 1) * group]
        amax = np.float32(np.abs(blk).max())
        if amax == 0:
            continue
        s_g = np.float32(amax / np.float32(127.0))
        q = np.rint(blk / s_g)                   # float32 / float32: one IEEE division each
        codes[gi * group:(gi + 1) * group] = np.clip(q, -127, 127).astype(np.int8)
        scales[gi] = s_g
    return codes, scales


def decode_scores_q8(qt, codes, scales, kt_tail, group: int = QGROUP) -> np.ndarray:
    """Decode scores over an 8-bit index: score_u = s_g * sum_c qt_c code_{u,c}
    for the tokens of full groups (g = u // group), and qt . kt[u] over the
    bf16 rows of the partial last group (``kt_tail``). Exact in fp64."""
    qt = to_f64(qt)
    full = (codes.astype(np.float64) @ qt) * np.repeat(scales.astype(np.float64), group)
    tail = to_f64(kt_tail) @ qt if len(kt_tail) else np.zeros(0)
    return np.concatenate([full, tail])


# ---------------------------------------------------------------------------
# K-cache clustering: two-level decode selection
# ---------------------------------------------------------------------------
FIX_SCALE = 2.0 ** 20          # fixed-point step of the centroid sums


def kmeans_assign(x32, mu32) -> np.ndarray:
    """Nearest centroid of every row: argmin_i sum_c (x_c - mu_ic)^2, the sum
    taken over c = 0, 1, ... with every subtraction, square and addition
    rounded to fp32 (no fused multiply-add), ties to the smaller index.
    ``x32`` [L, r] and ``mu32`` [C, r] are float32."""
    L, r = x32.shape
    out = np.empty(L, np.int64)
    for u0 in range(0, L, 4096):                              # bounded temporaries
        xs = x32[u0:u0 + 4096]
        d = np.zeros((xs.shape[0], mu32.shape[0]), np.float32)
        for c in range(r):
            diff = xs[:, c:c + 1] - mu32[None, :, c]          # float32, one rounding
            d = d + diff * diff                               # float32 product, then float32 sum
        out[u0:u0 + 4096] = np.argmin(d, axis=1)              # first minimum: smaller index
    return out


def kmeans_update(x32, assign, mu32) -> np.ndarray:
    """New centroids: the mean of each cluster's rows. The sums are exact
    integer sums of trunc(x * 2^20) (so that their value does not depend on
    the order of the additions), then mean = fp32(double(sum) / double(count)
    * 2^-20); a cluster with no rows keeps its centroid."""
    C, r = mu32.shape
    fixed = np.trunc(x32.astype(np.float64) * FIX_SCALE).astype(np.int64)
    sums = np.zeros((C, r), np.int64)
    np.add.at(sums, assign, fixed)
    cnt = np.bincount(assign, minlength=C).astype(np.int64)
    new = mu32.copy()
    nz = cnt > 0
    new[nz] = ((sums[nz].astype(np.float64) / cnt[nz, None].astype(np.float64)) / FIX_SCALE).astype(np.float32)
    return new


def kmeans_index(kt, cluster_size: int = 64, iters: int = 2):
    """K-means over one KV head's key index (RTPurboV2 article: the keys of the
    retrieval heads are clustered in the low-rank space, so that decode can
    skip whole groups of semantically unrelated tokens; the pages give no
    algorithm, so this is plain Lloyd k-means). C = ceil(L / cluster_size)
    centroids start at the rows 0, cluster_size, 2 cluster_size, ...; each of
    ``iters`` iterations assigns every row to its nearest centroid and moves
    the centroids to their clusters' means; a final assignment pairs every
    row with its nearest final centroid. Returns (centroids [C, r] float32,
    assignment [L] int64)."""
    x = to_f64(kt).astype(np.float32)
    L = x.shape[0]
    C = (L + cluster_size - 1) // cluster_size
    mu = x[np.arange(C) * cluster_size].copy()
    for _ in range(iters):
        mu = kmeans_update(x, kmeans_assign(x, mu), mu)
    return mu, kmeans_assign(x, mu)


def select_decode_clustered(qt, kt, centroids, assign, n_probe: int, topk: int):
    """Two-level token selection: the n_probe clusters whose centroids score
    highest against q~ (ties to the smaller cluster), then the top-k tokens by
    q~ . k~ among those clusters' members (ties to the smaller token; all of
    them when fewer). Returns a dict with the ascending selection ``sel`` and
    the intermediate ``cluster_scores``, ``clusters`` (chosen, ascending),
    ``cand`` (ascending candidate tokens) and ``cand_scores``."""
    qt = to_f64(qt)
    cs = to_f64(centroids) @ qt
    chosen = topk_desc(cs, n_probe)
    cand = np.flatnonzero(np.isin(np.asarray(assign), chosen))
    sc = to_f64(kt)[cand] @ qt
    sel = cand[topk_desc(sc, topk)]
    return dict(sel=np.sort(sel), cluster_scores=cs, clusters=chosen, cand=cand, cand_scores=sc)


# ---------------------------------------------------------------------------
# Static patterns on the same attention (presets)
# ---------------------------------------------------------------------------
def triangle_keys(t: int, N: int, sink_blocks: int, window_blocks: int, last_tokens: int,
                  block: int = BLOCK) -> np.ndarray:
    """Keys of query row t under the triangle-shaped mask (TriangleMix
    interview, 36kr, paragraph on the triangle-shaped mask): rows of the last
    Q-K region (t >= N - last_tokens) keep every causal key; every other row
    keeps only the streaming region, the sink blocks and the local band of
    blocks ending at its own block (block-granular, like the retrieval heads'
    window), causal."""
    if t >= N - last_tokens:
        return np.arange(0, t + 1)
    i = t // block
    blocks = np.union1d(np.arange(0, min(sink_blocks, i + 1)), np.arange(max(0, i - window_blocks + 1), i + 1))
    keys = np.concatenate([np.arange(j * block, (j + 1) * block) for j in blocks])
    return keys[keys <= t]


def triangle_rows(q, k, v, rows, sink_blocks: int, window_blocks: int, last_tokens: int,
                  scale: float, block: int = BLOCK) -> np.ndarray:
    """Triangle-mask attention of query rows ``rows`` of one head (q [N, D],
    k/v [N, D] of its KV head), one row at a time."""
    N = k.shape[0]
    q64, k64, v64 = to_f64(q), to_f64(k), to_f64(v)
    out = []
    for t in rows:
        keys = triangle_keys(int(t), N, sink_blocks, window_blocks, last_tokens, block)
        out.append(attend(q64[t:t + 1], [t], k64[keys], v64[keys], keys, scale)[0])
    return np.stack(out)


def dense_decode(q, kc, vc, scale: float) -> np.ndarray:
    """Full attention of one query (at the last position) over the whole
    cache: the cross-attention of an output position in Orthros (Orthros
    article, section on one attention with two working modes; the trained
    Scale-Offset of its query is out of scope, so the query is used as is)."""
    return attend_decode(q, kc, vc, np.arange(kc.shape[0]), scale)


# ---------------------------------------------------------------------------
# Whole-layer drivers
# ---------------------------------------------------------------------------
def kv_of(h: int, Hq: int, Hkv: int) -> int:
    return h // (Hq // Hkv)


def prefill_layer(q, k, v, P, ret_heads, window: int, ret_window: int, topk: int,
                  scale: float, qblocks=None, sink_blocks: int = 1, heads=None,
                  block: int = BLOCK, index=None):
    """One prefill layer for batch element 0-sliced tensors.

    ``q`` [N, Hq, D], ``k``/``v`` [N, Hkv, D], ``P`` [Hkv, D, r] (bf16 values).
    Computes the output rows of the query blocks ``qblocks`` (default: all)
    for ``heads`` (default: all). Returns a dict with ``out`` {(h, i): [64, D]},
    ``sel``/``scores`` {(h, i): ...} for retrieval heads, and ``kt``/``qt``.
    ``index`` may carry already projected ``{"kt": {g: ...}, "qt": {h: ...}}``
    (the output of ``project``) so that a caller sampling a few query blocks
    projects the sequence once.
    """
    P = to_f64(P)
    N, Hq, D = q.shape
    Hkv = k.shape[1]
    nb = N // block
    qblocks = list(range(nb)) if qblocks is None else list(qblocks)
    heads = list(range(Hq)) if heads is None else list(heads)
    ret = set(ret_heads)
    wb = ret_window // block
    kt_cache = dict(index["kt"]) if index else {}
    qt_given = index["qt"] if index else {}
    res = dict(out={}, sel={}, scores={}, kt={}, qt={})
    for h in heads:
        g = kv_of(h, Hq, Hkv)
        if h in ret:
            if g not in kt_cache:
                kt_cache[g] = project(k[:, g, :], P[g])
            kt = kt_cache[g]
            qt = qt_given[h] if h in qt_given else project(q[:, h, :], P[g])
            res["kt"][g], res["qt"][h] = kt, qt
            sel, sc = select_prefill(qt, kt, topk, qblocks, block)
            for i in qblocks:
                att = attended_blocks(sel[i], i, wb, sink_blocks)
                res["sel"][(h, i)] = sel[i]
                res["scores"][(h, i)] = sc[i]
                res["out"][(h, i)] = sparse_attn_prefill_block(q[:, h, :], k[:, g, :], v[:, g, :],
                                                               i, att, scale, block)
        else:
            for i in qblocks:
                rows = np.arange(i * block, (i + 1) * block)
                res["out"][(h, i)] = swa_rows(q[:, h, :], k[:, g, :], v[:, g, :], rows,
                                              window, scale)
    return res


def decode_layer(q, kc, vc, P, ret_heads, window: int, ret_window: int, topk: int,
                 scale: float, sink: int = 1, heads=None, index_bits: int = 16):
    """One decode step for one sequence.

    ``q`` [Hq, D], ``kc``/``vc`` [L, Hkv, D], ``P`` [Hkv, D, r]. The key index
    is the bf16-rounded projection of the cache; the query index is unrounded.
    ``index_bits`` = 8 scores over the 8-bit form of that index
    (``quantize_index``; its partial last group stays bf16).
    Returns ``out`` {h: [D]}, ``sel``/``scores`` {h: ...}.
    """
    q, P = to_f64(q), to_f64(P)
    Hq, D = q.shape
    L, Hkv, _ = kc.shape
    heads = list(range(Hq)) if heads is None else list(heads)
    ret = set(ret_heads)
    res = dict(out={}, sel={}, scores={}, kt={})
    for h in heads:
        g = kv_of(h, Hq, Hkv)
        if h in ret:
            if g not in res["kt"]:
                res["kt"][g] = project(kc[:, g, :], P[g])
            kt = res["kt"][g]
            qt = project(q[h], P[g], round_to_bf16=False)
            if index_bits == 8:
                codes, scales = quantize_index(kt)
                sc = decode_scores_q8(qt, codes, scales, kt[len(codes):])
            else:
                sc = decode_scores(qt, kt)
            sel = topk_desc(sc, topk)
            res["sel"][h], res["scores"][h] = sel, sc
            idx = decode_attended(sel, L, ret_window, sink)
        else:
            idx = np.arange(max(0, L - window), L)
        res["out"][h] = attend_decode(q[h], kc[:, g, :], vc[:, g, :], idx, scale)
    return res


__all__ = [
    "BLOCK", "bf16_round", "to_f64", "project", "block_scores", "topk_desc", "select_prefill",
    "attended_blocks", "attend", "sparse_attn_prefill_block", "swa_rows", "decode_scores",
    "select_decode", "decode_attended", "attend_decode", "kv_of", "prefill_layer",
    "decode_layer", "triangle_keys", "triangle_rows", "dense_decode", "QGROUP", "quantize_index",
    "decode_scores_q8", "FIX_SCALE", "kmeans_assign", "kmeans_update", "kmeans_index",
    "select_decode_clustered",
]
