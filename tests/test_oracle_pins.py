"""Pins for the CPU oracle: each check ties it to something other than itself.

Kinds of pin used here:
  * hand-worked examples (``tests/golden/*.json``, each with its derivation);
  * special cases that reduce to a library routine (torch's float64
    ``scaled_dot_product_attention`` with an explicit mask, torch's bf16 cast);
  * closed forms (window 1 returns the query's own value row; two keys with a
    known logit gap);
  * brute force on tiny inputs (pure-Python loops over every pair and a full
    sort, ``tests/brute.py``);
  * invariants (convex hull, key permutation, counts, causal-only blocks).

The last section plants plausible mistakes in copies of the oracle's
functions and checks that a pin above catches each one.
"""
import json
import math
import os

import numpy as np
import pytest
import torch

import oracle as O
import brute

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")
rng = np.random.default_rng(12345)


def _bf16_arr(shape, scale=1.0, rs=rng):
    return O.bf16_round(rs.standard_normal(shape) * scale)


def _sdpa_masked(q, k, v, mask, scale):
    """torch float64 SDPA for one head: q [m,D], k/v [n,D], mask [m,n] bool (True = attend)."""
    qt = torch.from_numpy(q)[None, None]
    kt = torch.from_numpy(k)[None, None]
    vt = torch.from_numpy(v)[None, None]
    mt = torch.from_numpy(mask)[None, None]
    return torch.nn.functional.scaled_dot_product_attention(qt, kt, vt, attn_mask=mt,
                                                            scale=scale)[0, 0].numpy()


# ---------------------------------------------------------------------------
# bf16 rounding
# ---------------------------------------------------------------------------
def test_bf16_round_known_values():
    one = 1.0
    cases = {
        one: one,
        one + 2.0 ** -8: one,                           # midpoint, ties to even (mantissa 0)
        one + 3 * 2.0 ** -8: one + 2.0 ** -6,           # midpoint between m=1 and m=2 -> even m=2
        one + 2.0 ** -8 + 2.0 ** -20: one + 2.0 ** -7,  # just above the midpoint
        -(one + 3 * 2.0 ** -8): -(one + 2.0 ** -6),
        3.0 * 2.0 ** -134: 2.0 ** -132,                 # subnormal: 1.5 quanta of 2**-133 -> 2 quanta
        2.0 ** -135: 0.0,                               # quarter quantum -> 0
        0.0: 0.0,
    }
    for x, want in cases.items():
        assert O.bf16_round(np.array([x]))[0] == want, x


def test_bf16_round_matches_torch_cast_on_fp32_values():
    x = (rng.standard_normal(200000) * np.exp(rng.uniform(-20, 20, 200000))).astype(np.float32)
    x = np.concatenate([x, np.float32([1e-39, -3e-40, 65504.0, 3.3895e38])])
    want = torch.from_numpy(x).to(torch.bfloat16).to(torch.float64).numpy()
    got = O.bf16_round(x.astype(np.float64))
    np.testing.assert_array_equal(got, want)


# ---------------------------------------------------------------------------
# Projection
# ---------------------------------------------------------------------------
def test_project_identity_columns_exact():
    x = _bf16_arr((300, 128), 3.0)
    P = np.zeros((128, 16))
    P[np.arange(16), np.arange(16)] = 1.0
    np.testing.assert_array_equal(O.project(x, P), x[:, :16])


def test_project_single_entries_closed_form():
    # column c picks 2**-c times component (5c mod 128): every result is exact.
    x = _bf16_arr((64, 128))
    P = np.zeros((128, 16))
    for c in range(16):
        P[(5 * c) % 128, c] = 2.0 ** -c
    want = np.stack([x[:, (5 * c) % 128] * 2.0 ** -c for c in range(16)], axis=1)
    np.testing.assert_array_equal(O.project(x, P), want)


def test_project_rounds_once_to_bf16():
    x = np.zeros((1, 128))
    x[0, 0] = 1.0
    x[0, 1] = 2.0 ** -8          # 1 + 2**-8 is a bf16 tie -> 1.0
    x[0, 2] = 2.0 ** -30         # pushes it above the tie -> 1 + 2**-7
    P = np.zeros((128, 16))
    P[0, 0] = P[1, 0] = 1.0
    P[0, 1] = P[1, 1] = P[2, 1] = 1.0
    y = O.project(x, P)
    assert y[0, 0] == 1.0 and y[0, 1] == 1.0 + 2.0 ** -7
    assert O.project(x, P, round_to_bf16=False)[0, 1] == 1.0 + 2.0 ** -8 + 2.0 ** -30


# ---------------------------------------------------------------------------
# Selection: hand-worked golden examples
# ---------------------------------------------------------------------------
def test_golden_block_selection():
    g = json.load(open(os.path.join(GOLDEN, "block_select_hand.json")))
    qt, kt = np.array(g["qt"], float), np.array(g["kt"], float)
    b = g["block"]
    sel, scores = O.select_prefill(qt, kt, g["topk"], block=b)
    for i in range(len(qt) // b):
        assert list(scores[i]) == g["scores"][str(i)]
        assert list(sel[i]) == g["selected"][str(i)]
        att = O.attended_blocks(sel[i], i, g["window_blocks"], g["sink_blocks"])
        assert list(att) == g["attended"][str(i)]


def test_golden_decode_selection():
    g = json.load(open(os.path.join(GOLDEN, "decode_select_hand.json")))
    qt, kt = np.array(g["qt"], float), np.array(g["kt"], float)
    assert list(O.decode_scores(qt, kt)) == g["scores"]
    sel = O.select_decode(qt, kt, g["topk"])
    assert list(sel) == g["selected"]
    assert list(O.decode_attended(sel, len(kt), g["window"], g["sink"])) == g["attended"]


# ---------------------------------------------------------------------------
# Selection: brute force and the r = D reduction
# ---------------------------------------------------------------------------
def _clustered(n, D, centres, rs):
    c = rs.standard_normal((centres, D))
    c = 3 * c / np.linalg.norm(c, axis=1, keepdims=True)
    return O.bf16_round(c[rs.integers(0, centres, n)] + rs.standard_normal((n, D)))


@pytest.mark.parametrize("N,block,topk", [(64, 8, 3), (96, 16, 2), (128, 32, 1)])
def test_block_scores_brute_force(N, block, topk):
    rs = np.random.default_rng(N)
    qt = O.bf16_round(rs.standard_normal((N, 4)))
    kt = O.bf16_round(rs.standard_normal((N, 4)))
    bs = brute.block_scores_bf(qt.tolist(), kt.tolist(), block)
    sel, scores = O.select_prefill(qt, kt, topk, block=block)
    for i in range(N // block):
        for j in range(i + 1):
            assert scores[i][j] == pytest.approx(bs[(i, j)], abs=1e-12)
        assert list(sel[i]) == brute.topk_bf({j: bs[(i, j)] for j in range(i + 1)}, topk)


def test_selection_with_identity_projector_is_exact_qk_topk():
    """r = D, P = I: the projected score is the exact q.k, so the selection is
    the top-k of the exact max-over-pairs q.k, found here by brute force."""
    rs = np.random.default_rng(7)
    N, D, block, topk = 256, 128, 64, 2
    q = _clustered(N, D, 8, rs)
    k = _clustered(N, D, 8, rs)
    P = np.eye(D)
    qt, kt = O.project(q, P), O.project(k, P)
    np.testing.assert_array_equal(qt, q)
    sel, _ = O.select_prefill(qt, kt, topk, block=block)
    bs = brute.block_scores_bf(q.tolist(), k.tolist(), block)
    for i in range(N // block):
        assert list(sel[i]) == brute.topk_bf({j: bs[(i, j)] for j in range(i + 1)}, topk)


def test_topk_ties_and_short_lists():
    s = np.array([1.0, 3.0, 3.0, 2.0, 3.0])
    assert list(O.topk_desc(s, 2)) == [1, 2]
    assert list(O.topk_desc(s, 4)) == [1, 2, 3, 4]
    assert list(O.topk_desc(s, 5)) == [0, 1, 2, 3, 4]
    assert list(O.topk_desc(s, 9)) == [0, 1, 2, 3, 4]
    rs = np.random.default_rng(3)
    for _ in range(50):
        s = rs.integers(0, 6, 40).astype(float)   # many ties
        k = int(rs.integers(1, 40))
        assert list(O.topk_desc(s, k)) == brute.topk_bf(dict(enumerate(s)), k)


def test_prefill_selection_invariants():
    rs = np.random.default_rng(11)
    N, block, topk = 1024, 64, 4
    qt = O.bf16_round(rs.standard_normal((N, 16)))
    kt = O.bf16_round(rs.standard_normal((N, 16)))
    sel, _ = O.select_prefill(qt, kt, topk, block=block)
    for i, s in sel.items():
        assert len(s) == min(topk, i + 1)
        assert np.all(np.diff(s) > 0) and s.min() >= 0 and s.max() <= i
        att = O.attended_blocks(s, i, 3, 1)
        assert 0 in att and i in att and max(0, i - 2) in att
        assert np.all(np.diff(att) > 0)


# ---------------------------------------------------------------------------
# Attention: library-routine reductions, closed forms, invariants
# ---------------------------------------------------------------------------
def test_attend_two_keys_closed_form():
    q = np.array([[1.0, 0.0]])
    k = np.array([[0.0, 0.0], [math.log(3.0), 5.0]])
    v = np.array([[4.0, -8.0], [0.0, 8.0]])
    o = O.attend(q, [1], k, v, [0, 1], 1.0)
    np.testing.assert_allclose(o[0], [1.0, 4.0], rtol=0, atol=1e-14)   # weights 1/4, 3/4


def test_sparse_prefill_with_all_blocks_is_dense_causal():
    """k >= number of blocks: every query attends every earlier key, i.e.
    dense causal attention (torch float64 SDPA, is_causal)."""
    rs = np.random.default_rng(5)
    N, D, block = 320, 128, 64
    q, k, v = _bf16_arr((N, D), 1, rs), _bf16_arr((N, D), 1, rs), _bf16_arr((N, D), 1, rs)
    scale = 1 / math.sqrt(D)
    qt = O.bf16_round(rs.standard_normal((N, 16)))
    kt = O.bf16_round(rs.standard_normal((N, 16)))
    sel, _ = O.select_prefill(qt, kt, N // block, block=block)
    ref = torch.nn.functional.scaled_dot_product_attention(
        torch.from_numpy(q)[None, None], torch.from_numpy(k)[None, None],
        torch.from_numpy(v)[None, None], is_causal=True, scale=scale)[0, 0].numpy()
    for i in range(N // block):
        att = O.attended_blocks(sel[i], i, 1, 1)
        assert list(att) == list(range(i + 1))
        o = O.sparse_attn_prefill_block(q, k, v, i, att, scale, block)
        np.testing.assert_allclose(o, ref[i * block:(i + 1) * block], rtol=0, atol=1e-12)


def test_sparse_prefill_matches_masked_sdpa():
    """General sparse sets: the same attention as torch SDPA given the mask
    'key block in the attended set and u <= t'."""
    rs = np.random.default_rng(6)
    N, D, block = 512, 64, 64
    q, k, v = _bf16_arr((N, D), 1, rs), _bf16_arr((N, D), 1, rs), _bf16_arr((N, D), 1, rs)
    scale = 0.125
    for i, att in [(7, [0, 2, 5, 6, 7]), (3, [0, 3]), (5, [1, 4, 5])]:
        rows = np.arange(i * block, (i + 1) * block)
        mask = np.zeros((block, N), bool)
        for j in att:
            mask[:, j * block:(j + 1) * block] = True
        mask &= np.arange(N)[None, :] <= rows[:, None]
        ref = _sdpa_masked(q[rows], k, v, mask, scale)
        o = O.sparse_attn_prefill_block(q, k, v, i, np.array(att), scale, block)
        np.testing.assert_allclose(o, ref, rtol=0, atol=1e-12)


def test_swa_wide_window_is_full_causal():
    rs = np.random.default_rng(8)
    N, D = 200, 128
    q, k, v = _bf16_arr((N, D), 1, rs), _bf16_arr((N, D), 1, rs), _bf16_arr((N, D), 1, rs)
    scale = 1 / math.sqrt(D)
    ref = torch.nn.functional.scaled_dot_product_attention(
        torch.from_numpy(q)[None, None], torch.from_numpy(k)[None, None],
        torch.from_numpy(v)[None, None], is_causal=True, scale=scale)[0, 0].numpy()
    for W in (N, N + 77):
        np.testing.assert_allclose(O.swa_rows(q, k, v, np.arange(N), W, scale), ref,
                                   rtol=0, atol=1e-12)


def test_swa_window_one_returns_own_value():
    rs = np.random.default_rng(9)
    q, k, v = _bf16_arr((50, 32), 1, rs), _bf16_arr((50, 32), 1, rs), _bf16_arr((50, 32), 1, rs)
    np.testing.assert_array_equal(O.swa_rows(q, k, v, np.arange(50), 1, 0.3), v)


@pytest.mark.parametrize("W", [2, 17, 64])
def test_swa_matches_band_masked_sdpa(W):
    rs = np.random.default_rng(W)
    N, D = 150, 64
    q, k, v = _bf16_arr((N, D), 1, rs), _bf16_arr((N, D), 1, rs), _bf16_arr((N, D), 1, rs)
    t = np.arange(N)
    mask = (t[None, :] <= t[:, None]) & (t[None, :] > t[:, None] - W)
    ref = _sdpa_masked(q, k, v, mask, 0.2)
    np.testing.assert_allclose(O.swa_rows(q, k, v, t, W, 0.2), ref, rtol=0, atol=1e-12)


def test_swa_decode_position_offset():
    """A single query at position L-1 over an L-key cache: last W keys."""
    rs = np.random.default_rng(10)
    L, D, W = 300, 64, 40
    q, k, v = _bf16_arr((1, D), 1, rs), _bf16_arr((L, D), 1, rs), _bf16_arr((L, D), 1, rs)
    mask = np.zeros((1, L), bool)
    mask[0, L - W:] = True
    ref = _sdpa_masked(q, k, v, mask, 0.1)
    np.testing.assert_allclose(O.swa_rows(q, k, v, [0], W, 0.1, q_pos0=L - 1), ref,
                               rtol=0, atol=1e-12)


def test_attention_invariants_hull_and_permutation():
    rs = np.random.default_rng(12)
    D = 128
    q = _bf16_arr((4, D), 1, rs)
    k, v = _bf16_arr((90, D), 1, rs), _bf16_arr((90, D), 1, rs)
    pos = np.arange(90)
    o = O.attend(q, [89] * 4, k, v, pos, 0.09)
    assert np.all(o <= v.max(axis=0) + 1e-12) and np.all(o >= v.min(axis=0) - 1e-12)
    perm = rs.permutation(90)
    o2 = O.attend(q, [89] * 4, k[perm], v[perm], pos[perm], 0.09)
    np.testing.assert_allclose(o, o2, rtol=0, atol=1e-13)


def test_decode_all_tokens_is_dense_attention():
    rs = np.random.default_rng(13)
    L, D = 500, 128
    q, kc, vc = _bf16_arr((D,), 1, rs), _bf16_arr((L, D), 1, rs), _bf16_arr((L, D), 1, rs)
    qt, kt = rs.standard_normal(16), O.bf16_round(rs.standard_normal((L, 16)))
    sel = O.select_decode(qt, kt, L)
    att = O.decode_attended(sel, L, 8, 1)
    assert list(att) == list(range(L))
    o = O.attend_decode(q, kc, vc, att, 1 / math.sqrt(D))
    ref = _sdpa_masked(q[None], kc, vc, np.ones((1, L), bool), 1 / math.sqrt(D))[0]
    np.testing.assert_allclose(o, ref, rtol=0, atol=1e-12)


def test_decode_identity_projector_selects_needles():
    """With P = I the decode score is the exact q.k; keys planted as 8*unit(q)
    (score 8|q|, far above the clustered background's q.k) are all selected."""
    rs = np.random.default_rng(14)
    L, D, n_needle = 4096, 128, 32
    kc = _clustered(L, D, 64, rs)
    q = _clustered(1, D, 64, rs)[0]
    pos = np.sort(rs.choice(L, n_needle, replace=False))
    kc[pos] = O.bf16_round(8 * q / np.linalg.norm(q))
    sel = O.select_decode(O.project(q, np.eye(D), round_to_bf16=False), O.project(kc, np.eye(D)),
                          n_needle)
    assert list(sel) == list(pos)


def test_decode_brute_force_pipeline():
    rs = np.random.default_rng(15)
    L, D, Hkv, Hq = 96, 16, 2, 4
    kc = _bf16_arr((L, Hkv, D), 1, rs)
    vc = _bf16_arr((L, Hkv, D), 1, rs)
    q = _bf16_arr((Hq, D), 1, rs)
    P = _bf16_arr((Hkv, D, 4), 0.25, rs)
    res = O.decode_layer(q, kc, vc, P, ret_heads=[1, 2], window=10, ret_window=7, topk=5,
                         scale=0.25, sink=1)
    for h in range(Hq):
        g = h // 2
        if h in (1, 2):
            qt = (q[h] @ P[g]).tolist()
            kt = O.bf16_round(kc[:, g, :] @ P[g]).tolist()
            sel, o = brute.decode_bf(q[h].tolist(), kc[:, g].tolist(), vc[:, g].tolist(), qt, kt,
                                     5, 7, 1, 0.25)
            assert list(res["sel"][h]) == sel
        else:
            o = brute.swa_bf([q[h].tolist()] * L, kc[:, g].tolist(), vc[:, g].tolist(), 10,
                             0.25)[L - 1]
        np.testing.assert_allclose(res["out"][h], o, rtol=0, atol=1e-12)


def test_prefill_brute_force_pipeline():
    """N = 256 prefill layer, every head, against the pure-Python definition."""
    rs = np.random.default_rng(16)
    N, D, Hq, Hkv, block = 256, 32, 4, 2, 64
    q = _bf16_arr((N, Hq, D), 1, rs)
    k = _bf16_arr((N, Hkv, D), 1, rs)
    v = _bf16_arr((N, Hkv, D), 1, rs)
    P = _bf16_arr((Hkv, D, 4), 0.3, rs)
    res = O.prefill_layer(q, k, v, P, ret_heads=[0, 3], window=70, ret_window=64, topk=1,
                          scale=0.2)
    for h in range(Hq):
        g = h // 2
        if h in (0, 3):
            qt = O.bf16_round(q[:, h] @ P[g]).tolist()
            kt = O.bf16_round(k[:, g] @ P[g]).tolist()
            sel, out = brute.prefill_head_bf(q[:, h].tolist(), k[:, g].tolist(), v[:, g].tolist(),
                                             qt, kt, 1, 1, 1, block, 0.2)
            for i in range(N // block):
                assert list(res["sel"][(h, i)]) == sel[i]
        else:
            out = brute.swa_bf(q[:, h].tolist(), k[:, g].tolist(), v[:, g].tolist(), 70, 0.2)
        for i in range(N // block):
            np.testing.assert_allclose(res["out"][(h, i)], np.array(out[i * block:(i + 1) * block]),
                                       rtol=0, atol=1e-12)


# ---------------------------------------------------------------------------
# Planted mistakes: each mutant of an oracle step must fail a pin above.
# ---------------------------------------------------------------------------
def _golden_selection_ok(block_scores_fn, topk_fn):
    g = json.load(open(os.path.join(GOLDEN, "block_select_hand.json")))
    qt, kt = np.array(g["qt"], float), np.array(g["kt"], float)
    for i in range(4):
        s = block_scores_fn(qt, kt, i, g["block"])
        if list(topk_fn(s, g["topk"])) != g["selected"][str(i)]:
            return False
    return True


def test_planted_mistakes_are_caught():
    assert _golden_selection_ok(O.block_scores, O.topk_desc)

    def non_causal_scores(qt, kt, i, block):       # diagonal block scored on every pair
        qb = qt[i * block:(i + 1) * block]
        s = qb @ kt[:(i + 1) * block].T
        return s.reshape(block, i + 1, block).max(axis=(0, 2))

    def ties_to_larger(scores, k):                  # reversed tie-break
        n = len(scores)
        if n <= k:
            return np.arange(n)
        order = np.lexsort((-np.arange(n), -np.asarray(scores)))
        return np.sort(order[:k])

    def sum_instead_of_max(qt, kt, i, block):       # block score as a mean, not a max
        s = O.block_scores(qt, kt, i, block)
        qb = qt[i * block:(i + 1) * block]
        return np.array([(qb @ kt[j * block:(j + 1) * block].T).mean() for j in range(i + 1)])

    assert not _golden_selection_ok(non_causal_scores, O.topk_desc)
    assert not _golden_selection_ok(O.block_scores, ties_to_larger)
    assert not _golden_selection_ok(sum_instead_of_max, O.topk_desc)

    # SWA with the window off by one must fail the band-mask library check.
    rs = np.random.default_rng(21)
    N, D, W = 80, 32, 9
    q, k, v = _bf16_arr((N, D), 1, rs), _bf16_arr((N, D), 1, rs), _bf16_arr((N, D), 1, rs)
    t = np.arange(N)
    mask = (t[None, :] <= t[:, None]) & (t[None, :] > t[:, None] - W)
    ref = _sdpa_masked(q, k, v, mask, 0.2)
    assert np.abs(O.swa_rows(q, k, v, t, W + 1, 0.2) - ref).max() > 1e-3

    # Attention with a wrong scale must fail the two-key closed form.
    qq = np.array([[1.0, 0.0]])
    kk = np.array([[0.0, 0.0], [math.log(3.0), 5.0]])
    vv = np.array([[4.0, -8.0], [0.0, 8.0]])
    assert np.abs(O.attend(qq, [1], kk, vv, [0, 1], 0.5)[0] - [1.0, 4.0]).max() > 0.1

    # Window blocks counted from the wrong end must fail the golden attended sets.
    g = json.load(open(os.path.join(GOLDEN, "block_select_hand.json")))
    wrong = np.unique(np.concatenate([np.array(g["selected"]["3"]), [0], np.arange(0, 1)]))
    assert list(wrong) != g["attended"]["3"]


# ---------------------------------------------------------------------------
# Static patterns: triangle-shaped mask, dense (full cross-attention) decode
# ---------------------------------------------------------------------------
def _ranges_to_keys(ranges):
    return np.concatenate([np.arange(a, b + 1) for a, b in ranges])


def _golden_triangle_ok(keys_fn):
    g = json.load(open(os.path.join(GOLDEN, "triangle_mask_hand.json")))
    for c in g["cases"]:
        got = keys_fn(c["t"], g["N"], c["sink_blocks"], c["window_blocks"], c["last_tokens"], g["block"])
        if not np.array_equal(np.asarray(got), _ranges_to_keys(c["ranges"])):
            return False
    return True


def test_golden_triangle_key_sets():
    assert _golden_triangle_ok(O.triangle_keys)


def test_triangle_uniform_attention_averages_the_key_set():
    """q = 0 makes every logit equal, so each output row is the plain mean of
    the attended value rows: with v_u = e_u the row is 1/|set| on the set."""
    g = json.load(open(os.path.join(GOLDEN, "triangle_mask_hand.json")))
    N, D = g["N"], g["N"]
    q = np.zeros((N, D))
    k = _bf16_arr((N, D), 1, np.random.default_rng(30))
    v = np.eye(N)
    for c in g["cases"]:
        o = O.triangle_rows(q, k, v, [c["t"]], c["sink_blocks"], c["window_blocks"], c["last_tokens"], 0.3)[0]
        want = np.zeros(N)
        keys = _ranges_to_keys(c["ranges"])
        want[keys] = 1.0 / len(keys)
        np.testing.assert_allclose(o, want, rtol=0, atol=1e-15)


def test_triangle_whole_last_region_is_dense_causal():
    rs = np.random.default_rng(31)
    N, D = 256, 128
    q, k, v = _bf16_arr((N, D), 1, rs), _bf16_arr((N, D), 1, rs), _bf16_arr((N, D), 1, rs)
    scale = 1 / math.sqrt(D)
    ref = torch.nn.functional.scaled_dot_product_attention(
        torch.from_numpy(q)[None, None], torch.from_numpy(k)[None, None],
        torch.from_numpy(v)[None, None], is_causal=True, scale=scale)[0, 0].numpy()
    rows = np.arange(N)
    np.testing.assert_allclose(O.triangle_rows(q, k, v, rows, 1, 1, N, scale), ref, rtol=0, atol=1e-12)
    # no last region but a band covering every block: dense causal as well
    np.testing.assert_allclose(O.triangle_rows(q, k, v, rows, 0, N // 64, 0, scale), ref, rtol=0, atol=1e-12)


def test_triangle_matches_masked_sdpa():
    rs = np.random.default_rng(32)
    N, D, block = 384, 64, 64
    q, k, v = _bf16_arr((N, D), 1, rs), _bf16_arr((N, D), 1, rs), _bf16_arr((N, D), 1, rs)
    sink, wb, last = 1, 2, 128
    t = np.arange(N)
    kb, qb = t[None, :] // block, t[:, None] // block
    # mask from the golden's wording: last rows see every causal key; others
    # see sink blocks and the band of wb blocks ending at their own block
    mask = (t[None, :] <= t[:, None]) & ((t[:, None] >= N - last) | (kb < sink) | (kb > qb - wb))
    ref = _sdpa_masked(q, k, v, mask, 0.125)
    np.testing.assert_allclose(O.triangle_rows(q, k, v, t, sink, wb, last, 0.125), ref, rtol=0, atol=1e-12)


def test_dense_decode_is_full_attention():
    rs = np.random.default_rng(33)
    L, D = 700, 128
    q, kc, vc = _bf16_arr((D,), 1, rs), _bf16_arr((L, D), 1, rs), _bf16_arr((L, D), 1, rs)
    ref = _sdpa_masked(q[None], kc, vc, np.ones((1, L), bool), 1 / math.sqrt(D))[0]
    np.testing.assert_allclose(O.dense_decode(q, kc, vc, 1 / math.sqrt(D)), ref, rtol=0, atol=1e-12)


def test_planted_triangle_mistakes_are_caught():
    def last_region_off_by_one(t, N, sink, wb, last, block):     # '>' instead of '>='
        if t > N - last:
            return np.arange(0, t + 1)
        return O.triangle_keys(t, N, sink, wb, 0, block)

    def band_without_own_block(t, N, sink, wb, last, block):     # band ends one block early
        if t >= N - last:
            return np.arange(0, t + 1)
        i = t // block
        blocks = np.union1d(np.arange(0, min(sink, i + 1)), np.arange(max(0, i - wb), i))
        keys = np.concatenate([np.arange(j * block, (j + 1) * block) for j in blocks]) if len(blocks) else \
            np.arange(0)
        return keys[keys <= t]

    assert not _golden_triangle_ok(last_region_off_by_one)
    assert not _golden_triangle_ok(band_without_own_block)


# ---------------------------------------------------------------------------
# 8-bit key index
# ---------------------------------------------------------------------------
def _golden_q8_ok(quant):
    import struct
    g = json.load(open(os.path.join(GOLDEN, "index_q8_hand.json")))
    kt = np.array(g["kt"])
    codes, scales = quant(kt, g["group"])
    if codes.tolist() != g["codes"]:
        return False
    hexes = [hex(struct.unpack("<I", struct.pack("<f", float(x)))[0]) for x in scales]
    if [int(h, 16) for h in hexes] != [int(h, 16) for h in g["scales_f32_hex"]]:
        return False
    sc = O.decode_scores_q8(g["q"], codes, scales, kt[len(codes):], g["group"])
    return all(sc[int(r)] == v for r, v in g["scores_by_row"].items()) and \
        sc[2] / float(scales[1]) == g["score_row2_over_s1"]


def test_golden_index_q8():
    assert _golden_q8_ok(O.quantize_index)


def test_index_q8_reconstruction_bound_and_extremes():
    """Each code times its scale lies within half a step (s/2) of the bf16
    value, plus what the fp32 division x / s may move the quotient by (half
    an fp32 ulp of a quotient below 128: 2^-17 code units), and a group's
    largest magnitude maps to +-127."""
    rs = np.random.default_rng(40)
    kt = O.bf16_round(rs.standard_normal((64 * 37 + 13, 16)) * rs.uniform(0.01, 30, (64 * 37 + 13, 1)))
    codes, scales = O.quantize_index(kt)
    assert codes.shape == (64 * 37, 16) and scales.shape == (37,)
    rec = codes.astype(np.float64) * np.repeat(scales.astype(np.float64), 64)[:, None]
    err = np.abs(rec - kt[:64 * 37])
    assert np.all(err <= np.repeat(scales.astype(np.float64), 64)[:, None] * (0.5 + 2.0 ** -17))
    for gi in range(37):
        blk = codes[gi * 64:(gi + 1) * 64]
        assert np.abs(blk).max() == 127


def test_index_q8_scores_track_the_bf16_scores():
    """The 8-bit scores differ from the bf16 ones by at most sum_c |q_c| (s/2
    + the fp32 quotient rounding, 2^-17 s)."""
    rs = np.random.default_rng(41)
    kt = O.bf16_round(rs.standard_normal((4096, 16)))
    q = rs.standard_normal(16)
    codes, scales = O.quantize_index(kt)
    sc8 = O.decode_scores_q8(q, codes, scales, kt[len(codes):])
    sc16 = O.decode_scores(q, kt)
    bound = np.abs(q).sum() * np.repeat(scales.astype(np.float64), 64) * (0.5 + 2.0 ** -17)
    assert np.all(np.abs(sc8 - sc16) <= bound)


def test_planted_q8_mistakes_are_caught():
    def truncating(kt, group):                     # round toward zero instead of half to even
        x = O.to_f64(kt).astype(np.float32)
        n = x.shape[0] // group
        codes = np.zeros((n * group, x.shape[1]), np.int8)
        scales = np.zeros(n, np.float32)
        for gi in range(n):
            blk = x[gi * group:(gi + 1) * group]
            a = np.float32(np.abs(blk).max())
            if a == 0:
                continue
            s_g = np.float32(a / np.float32(127.0))
            codes[gi * group:(gi + 1) * group] = np.clip(np.trunc(blk / s_g), -127, 127).astype(np.int8)
            scales[gi] = s_g
        return codes, scales

    def scale_by_128(kt, group):                   # step amax/128: the largest value overflows
        x = O.to_f64(kt).astype(np.float32)
        n = x.shape[0] // group
        codes = np.zeros((n * group, x.shape[1]), np.int8)
        scales = np.zeros(n, np.float32)
        for gi in range(n):
            blk = x[gi * group:(gi + 1) * group]
            a = np.float32(np.abs(blk).max())
            if a == 0:
                continue
            s_g = np.float32(a / np.float32(128.0))
            codes[gi * group:(gi + 1) * group] = np.clip(np.rint(blk / s_g), -127, 127).astype(np.int8)
            scales[gi] = s_g
        return codes, scales

    assert not _golden_q8_ok(truncating)
    assert not _golden_q8_ok(scale_by_128)


# ---------------------------------------------------------------------------
# K-cache clustering (two-level decode selection)
# ---------------------------------------------------------------------------
def _golden_kcluster_ok(kmeans, select):
    g = json.load(open(os.path.join(GOLDEN, "kcluster_hand.json")))
    kt = np.array(g["kt"], np.float64)
    mu, a = kmeans(kt, g["cluster_size"], g["iters"])
    if not (np.array_equal(mu, np.array(g["centroids"], np.float32)) and list(a) == g["assign"]):
        return False
    for c in g["selections"]:
        r = select(np.array(g["q"], np.float64), kt, mu, a, c["n_probe"], c["topk"])
        if list(r["clusters"]) != c["clusters"] or list(r["sel"]) != c["sel"]:
            return False
    return True


def test_golden_kcluster():
    assert _golden_kcluster_ok(O.kmeans_index, O.select_decode_clustered)


def test_kcluster_reduces_to_flat_topk():
    """Every token its own cluster, or every cluster probed: the two-level
    selection is the flat top-k over the whole cache."""
    rs = np.random.default_rng(50)
    L = 700
    kt = O.bf16_round(rs.standard_normal((L, 16)) * 2)
    q = rs.standard_normal(16)
    flat = O.select_decode(q, kt, 64)
    mu, a = O.kmeans_index(kt, 1, 1)
    assert list(a) == list(range(L))                          # distinct rows: each its own centroid
    assert list(O.select_decode_clustered(q, kt, mu, a, 64, 64)["sel"]) == list(flat)
    mu, a = O.kmeans_index(kt, 64, 2)
    assert list(O.select_decode_clustered(q, kt, mu, a, len(mu), 64)["sel"]) == list(flat)


def test_kmeans_objective_does_not_increase():
    """Lloyd's iterations never raise the within-cluster sum of squares, and
    every row ends at its nearest final centroid."""
    rs = np.random.default_rng(51)
    c = rs.standard_normal((12, 16)) * 4
    kt = O.bf16_round(c[rs.integers(0, 12, 3000)] + rs.standard_normal((3000, 16)) * 0.5)
    x = kt.astype(np.float32)
    prev = None
    for it in range(4):
        mu, a = O.kmeans_index(kt, 256, it)
        obj = float(((x.astype(np.float64) - mu[a].astype(np.float64)) ** 2).sum())
        d = ((x[:, None, :].astype(np.float64) - mu[None].astype(np.float64)) ** 2).sum(-1)
        assert np.all(d[np.arange(len(a)), a] <= d.min(1) * (1 + 1e-6) + 1e-9)
        if prev is not None:
            assert obj <= prev * (1 + 1e-6)
        prev = obj


def test_planted_kcluster_mistakes_are_caught():
    def far_assign(x32, mu32):                       # argmax instead of argmin
        d = ((x32[:, None, :] - mu32[None]) ** 2).sum(-1)
        return np.argmax(d, axis=1)

    def kmeans_far(kt, cs, iters):
        x = O.to_f64(kt).astype(np.float32)
        C = (len(x) + cs - 1) // cs
        mu = x[np.arange(C) * cs].copy()
        for _ in range(iters):
            mu = O.kmeans_update(x, far_assign(x, mu), mu)
        return mu, far_assign(x, mu)

    def kmeans_ties_high(kt, cs, iters):             # ties to the larger centroid index
        x = O.to_f64(kt).astype(np.float32)
        C = (len(x) + cs - 1) // cs
        mu = x[np.arange(C) * cs].copy()

        def asg(mu_):
            d = np.zeros((len(x), len(mu_)), np.float32)
            for c in range(x.shape[1]):
                diff = x[:, c:c + 1] - mu_[None, :, c]
                d = d + diff * diff
            return len(mu_) - 1 - np.argmin(d[:, ::-1], axis=1)
        for _ in range(iters):
            mu = O.kmeans_update(x, asg(mu), mu)
        return mu, asg(mu)

    def select_lowest_clusters(q, kt, mu, a, n_probe, topk):   # probes the lowest-scoring clusters
        r = O.select_decode_clustered(-np.asarray(q), kt, mu, a, n_probe, topk)
        cand = r["cand"]
        sc = O.to_f64(kt)[cand] @ np.asarray(q, np.float64)
        return dict(r, sel=np.sort(cand[O.topk_desc(sc, topk)]))

    assert not _golden_kcluster_ok(kmeans_far, O.select_decode_clustered)
    assert not _golden_kcluster_ok(kmeans_ties_high, O.select_decode_clustered)
    assert not _golden_kcluster_ok(O.kmeans_index, select_lowest_clusters)
