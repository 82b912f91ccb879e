"""GPU parity: every C-ABI call against the fp64 oracle, stage by stage, then
end to end, at sizes the oracle finishes in seconds (several tiles plus a
ragged tail), with the method's edge cases.

Stage isolation: a GPU stage is fed the oracle's own inputs for that stage
(the oracle's projected index, the oracle's selected lists), never the other
way round.
"""
import math

import numpy as np
import pytest
import torch

import oracle as O
import synth
from helpers import assert_attn_close, assert_f32_index_close, assert_index_close, band_check

pytestmark = pytest.mark.gpu

rtp = pytest.importorskip("long_context_hybrid_b200")


def _f64(t):
    return t.detach().float().cpu().numpy().astype(np.float64)


def _randn_bf16(shape, seed, scale=1.0):
    g = torch.Generator().manual_seed(seed)
    return (torch.randn(*shape, generator=g) * scale).to(torch.bfloat16)


def _clustered_bf16(shape, seed, centres=16):
    g = torch.Generator().manual_seed(seed)
    D = shape[-1]
    c = torch.randn(centres, D, generator=g)
    c = 3 * c / c.norm(dim=1, keepdim=True)
    n = int(np.prod(shape[:-1]))
    a = torch.randint(0, centres, (n,), generator=g)
    return (c[a] + torch.randn(n, D, generator=g)).reshape(shape).to(torch.bfloat16)


@pytest.fixture(scope="module", autouse=True)
def _built():
    from long_context_hybrid_b200 import build
    build.build()
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    rtp.lib()


DEV = "cuda"


# ---------------------------------------------------------------------------
# Projection
# ---------------------------------------------------------------------------
@pytest.mark.parametrize("N", [1, 17, 1000])
def test_index_project_bf16_and_f32(N):
    x = _clustered_bf16((2, N, 5, 128), 1)
    P = _randn_bf16((3, 128, 16), 2, 1 / math.sqrt(128))
    heads, proj = [0, 3, 4], [0, 2, 1]
    xd, Pd = x.to(DEV), P.to(DEV)
    out = rtp.index_project(xd, Pd, heads, proj)
    out32 = rtp.index_project(xd, Pd, heads, proj, out_dtype=torch.float32)
    torch.cuda.synchronize()
    for j, (h, p) in enumerate(zip(heads, proj)):
        for b in range(2):
            assert_index_close(_f64(out[b, j]), x[b, :, h], P[p])
            assert_f32_index_close(_f64(out32[b, j]), x[b, :, h], P[p])


def test_index_project_strided_input():
    """A head slice of a wider tensor (non-packed strides)."""
    big = _clustered_bf16((1, 300, 6, 128), 3)
    x = big[:, :, 1:5, :]                    # strides (300*6*128, 6*128, 128, 1)
    P = _randn_bf16((1, 128, 16), 4, 1 / math.sqrt(128))
    out = rtp.index_project(big.to(DEV)[:, :, 1:5, :], P.to(DEV), [2], [0])
    torch.cuda.synchronize()
    assert_index_close(_f64(out[0, 0]), x[0, :, 2], P[0])


# ---------------------------------------------------------------------------
# Decode selection
# ---------------------------------------------------------------------------
# 24577: one token past a 24576-token slice; 196608 and 200003: rows longer
# than the largest bench workload
@pytest.mark.parametrize("L,topk", [(5003, 64), (40, 64), (1, 1), (2048, 2048), (70000, 2048), (24577, 100),
                                    (196608, 2048), (200003, 2048)])
def test_select_decode_matches_oracle(L, topk):
    B, Hkv, kv = 2, 2, [0, 0, 1]
    kindex = _clustered_bf16((B, Hkv, L, 16), 10 + L)
    if L > 200:   # planted identical keys: exact score ties
        kindex[:, :, 100:140] = kindex[:, :, 99:100]
    g = torch.Generator().manual_seed(L)
    qt = torch.randn(B, len(kv), 16, generator=g) * 2
    idx = rtp.select_decode(qt.to(DEV), kindex.to(DEV), kv, topk)
    torch.cuda.synchronize()
    idx = idx.cpu().numpy()
    for b in range(B):
        for j, gk in enumerate(kv):
            sc = O.decode_scores(qt[b, j].double().numpy(), kindex[b, gk])
            sel = O.topk_desc(sc, topk)
            got = idx[b, j]
            n = min(topk, L)
            assert np.all(got[n:] == -1)
            assert np.all(np.diff(got[:n]) > 0), "ascending"
            ok, amb, msg = band_check(got[:n], sel, sc, topk)
            assert ok, f"b{b} j{j}: {msg}"


@pytest.mark.parametrize("L", [1500, 3000, 6000, 60000, 250000])
def test_select_decode_ties_pick_lowest_index(L):
    """All keys equal: the lowest k indices must be chosen (the tied bin fits
    in shared memory at L = 1500; it does not at 3000 and beyond, and at
    60000 and 250000 it spans several filter blocks)."""
    topk = 100
    kindex = torch.ones(1, 1, L, 16, dtype=torch.bfloat16)
    qt = torch.ones(1, 1, 16)
    idx = rtp.select_decode(qt.to(DEV), kindex.to(DEV), [0], topk).cpu().numpy()
    assert list(idx[0, 0]) == list(range(topk))


def test_select_decode_candidate_overflow_falls_back_exactly():
    """More equal scores in the k-th score's bin than the candidate list holds:
    the full radix select must still pick the lowest indices; a second row with
    distinct scores in the same call takes the normal path."""
    L, topk = 20000, 300
    kindex = torch.ones(1, 2, L, 16, dtype=torch.bfloat16)
    kindex[0, 1] = _clustered_bf16((1, 1, L, 16), 77)[0, 0]
    qt = torch.ones(1, 2, 16)
    idx = rtp.select_decode(qt.to(DEV), kindex.to(DEV), [0, 1], topk).cpu().numpy()
    assert list(idx[0, 0]) == list(range(topk))
    sc = O.decode_scores(qt[0, 1].double().numpy(), kindex[0, 1])
    ok, amb, msg = band_check(idx[0, 1], O.topk_desc(sc, topk), sc, topk)
    assert ok, msg


# ---------------------------------------------------------------------------
# Prefill selection
# ---------------------------------------------------------------------------
# 192 and 2368: an odd number of query blocks (the last CTA has one); 9600:
# more than 16 full key tiles per CTA, so the staged row maxima are folded
# several times
@pytest.mark.parametrize("N,topk", [(1536, 5), (256, 8), (64, 1), (4096, 16), (192, 2), (2368, 9), (9600, 20)])
def test_select_prefill_matches_oracle(N, topk):
    B, Hkv, kv = 1, 2, [0, 1, 1]
    kt = _clustered_bf16((B, Hkv, N, 16), 20 + N)
    qt = _clustered_bf16((B, len(kv), N, 16), 30 + N)
    if N >= 1024:   # identical needle blocks: exact block-score ties
        kt[:, :, 3 * 64:4 * 64] = kt[:, :, 7 * 64:8 * 64] = kt[:, :, 11 * 64:11 * 64 + 1]
    blocks, counts = rtp.select_prefill(qt.to(DEV), kt.to(DEV), kv, topk)
    torch.cuda.synchronize()
    blocks, counts = blocks.cpu().numpy(), counts.cpu().numpy()
    nb = N // 64
    for j, gk in enumerate(kv):
        sel, scores = O.select_prefill(qt[0, j], kt[0, gk], topk)
        for i in range(nb):
            n = min(topk, i + 1)
            assert counts[0, j, i] == n
            got = blocks[0, j, i]
            assert np.all(got[n:] == -1)
            assert np.all(np.diff(got[:n]) > 0) and got[:n].max() <= i
            ok, amb, msg = band_check(got[:n], sel[i], scores[i], topk)
            assert ok, f"head {j} block {i}: {msg}"


# ---------------------------------------------------------------------------
# Prefill attention
# ---------------------------------------------------------------------------
def _qkv(B, N, Hq, Hkv, seed):
    return (_clustered_bf16((B, N, Hq, 128), seed), _clustered_bf16((B, N, Hkv, 128), seed + 1),
            _randn_bf16((B, N, Hkv, 128), seed + 2))


@pytest.mark.parametrize("N,window", [(640, 1), (640, 100), (640, 256), (640, 1000), (1024, 513)])
def test_swa_prefill_matches_oracle(N, window):
    B, Hq, Hkv = 2, 4, 2
    q, k, v = _qkv(B, N, Hq, Hkv, 40)
    heads = [1, 2, 3]
    o = torch.zeros(B, N, Hq, 128, dtype=torch.bfloat16, device=DEV)
    ws = torch.zeros(256, dtype=torch.uint8, device=DEV)
    rtp.swa(q.to(DEV), k.to(DEV), v.to(DEV), o, heads, window, ws=ws)
    assert rtp.workspace_status(ws) == 0
    o = o.cpu()
    scale = 1 / math.sqrt(128)
    for b in range(B):
        for h in heads:
            g = h // 2
            ref = O.swa_rows(q[b, :, h], k[b, :, g], v[b, :, g], np.arange(N), window, scale)
            assert_attn_close(_f64(o[b, :, h]), ref, f"b{b} h{h}")
    assert torch.all(o[:, :, 0] == 0), "unlisted head written"


def test_sparse_attn_prefill_matches_oracle():
    B, N, Hq, Hkv, topk = 1, 1024, 8, 2, 4
    nb = N // 64
    q, k, v = _qkv(B, N, Hq, Hkv, 50)
    heads = [0, 5]
    rs = np.random.default_rng(0)
    blocks = -np.ones((B, len(heads), nb, topk), np.int32)
    counts = np.zeros((B, len(heads), nb), np.int32)
    for j in range(len(heads)):
        for i in range(nb):
            n = min(topk, i + 1)
            sel = np.sort(rs.choice(i + 1, n, replace=False))
            blocks[0, j, i, :n] = sel
            counts[0, j, i] = n
    # one list deliberately unsorted with a duplicate: the set is what counts
    blocks[0, 1, 12, :4] = [9, 2, 9, 0]
    o = torch.zeros(B, N, Hq, 128, dtype=torch.bfloat16, device=DEV)
    rtp.sparse_attn_prefill(q.to(DEV), k.to(DEV), v.to(DEV), o, heads, torch.from_numpy(blocks).to(DEV),
                            torch.from_numpy(counts).to(DEV), window_blocks=3, sink_blocks=1)
    torch.cuda.synchronize()
    o = o.cpu()
    scale = 1 / math.sqrt(128)
    for j, h in enumerate(heads):
        g = h * Hkv // Hq
        for i in range(nb):
            att = O.attended_blocks(blocks[0, j, i, :counts[0, j, i]], i, 3, 1)
            ref = O.sparse_attn_prefill_block(q[0, :, h], k[0, :, g], v[0, :, g], i, att, scale)
            assert_attn_close(_f64(o[0, i * 64:(i + 1) * 64, h]), ref, f"h{h} i{i}")


def test_sparse_attn_prefill_all_blocks_is_dense_causal():
    B, N, Hq, Hkv = 1, 512, 2, 1
    nb = N // 64
    q, k, v = _qkv(B, N, Hq, Hkv, 60)
    blocks = torch.full((1, 1, nb, nb), -1, dtype=torch.int32)
    counts = torch.zeros(1, 1, nb, dtype=torch.int32)
    for i in range(nb):
        blocks[0, 0, i, :i + 1] = torch.arange(i + 1)
        counts[0, 0, i] = i + 1
    o = torch.zeros(B, N, Hq, 128, dtype=torch.bfloat16, device=DEV)
    rtp.sparse_attn_prefill(q.to(DEV), k.to(DEV), v.to(DEV), o, [1], blocks.to(DEV), counts.to(DEV),
                            window_blocks=1, sink_blocks=0)
    ref = torch.nn.functional.scaled_dot_product_attention(
        q[:, :, 1:2].double().transpose(1, 2), k.double().transpose(1, 2), v.double().transpose(1, 2),
        is_causal=True)[0, 0].numpy()
    assert_attn_close(_f64(o[0, :, 1].cpu()), ref, "dense causal")


# ---------------------------------------------------------------------------
# Decode attention
# ---------------------------------------------------------------------------
@pytest.mark.parametrize("L,window", [(3000, 512), (100, 512), (1, 8), (5000, 1)])
def test_swa_decode_matches_oracle(L, window):
    B, Hq, Hkv = 2, 8, 2
    q = _clustered_bf16((B, Hq, 128), 70)
    kc, vc = _clustered_bf16((B, L, Hkv, 128), 71), _randn_bf16((B, L, Hkv, 128), 72)
    heads = [1, 2, 3, 6]
    o = torch.zeros(B, Hq, 128, dtype=torch.bfloat16, device=DEV)
    rtp.swa(q.to(DEV).unsqueeze(1), kc.to(DEV), vc.to(DEV), o.unsqueeze(1), heads, window, q_pos0=L - 1)
    torch.cuda.synchronize()
    o = o.cpu()
    for b in range(B):
        for h in heads:
            g = h // 4
            idx = np.arange(max(0, L - window), L)
            ref = O.attend_decode(q[b, h], kc[b, :, g], vc[b, :, g], idx, 1 / math.sqrt(128))
            assert_attn_close(_f64(o[b, h]), ref[None], f"b{b} h{h}")


@pytest.mark.parametrize("L,topk,window,sink", [(4000, 256, 512, 1), (600, 256, 512, 1),
                                                (3000, 100, 64, 0), (3000, 300, 64, 4)])
def test_sparse_attn_decode_matches_oracle(L, topk, window, sink):
    B, Hq, Hkv = 2, 8, 2
    q = _clustered_bf16((B, Hq, 128), 80)
    kc, vc = _clustered_bf16((B, L, Hkv, 128), 81), _randn_bf16((B, L, Hkv, 128), 82)
    heads = [0, 5, 6]
    rs = np.random.default_rng(L + topk)
    idx = -np.ones((B, len(heads), topk), np.int32)
    special = [0, 1, 2, L - 1]          # sink tokens and the newest token: also reached otherwise
    for b in range(B):
        for j in range(len(heads)):
            n = min(topk, L) - (3 if topk < L else 0)   # some -1 padding
            pool = np.setdiff1d(np.arange(L), special)
            pick = rs.choice(pool, n - len(special), replace=False)
            idx[b, j, :n] = np.sort(np.concatenate([pick, special]))
    o = torch.zeros(B, Hq, 128, dtype=torch.bfloat16, device=DEV)
    rtp.sparse_attn_decode(q.to(DEV), kc.to(DEV), vc.to(DEV), o, heads, torch.from_numpy(idx).to(DEV),
                           window, sink)
    torch.cuda.synchronize()
    o = o.cpu()
    for b in range(B):
        for j, h in enumerate(heads):
            g = h // 4
            sel = idx[b, j][idx[b, j] >= 0]
            att = O.decode_attended(sel, L, window, sink)
            ref = O.attend_decode(q[b, h], kc[b, :, g], vc[b, :, g], att, 1 / math.sqrt(128))
            assert_attn_close(_f64(o[b, h]), ref[None], f"b{b} h{h}")


# ---------------------------------------------------------------------------
# End to end
# ---------------------------------------------------------------------------
def _prefill_e2e(cfg, data, qblocks, heads=None, check_kt=True):
    """Run the layer on the GPU, the oracle on the given query blocks; compare."""
    q, k, v, P = data["q"], data["k"], data["v"], data["P"]
    B, N = q.shape[0], q.shape[1]
    dev = q.device
    layer = rtp.PrefillLayer(B, N, cfg.Hq, cfg.Hkv, cfg.ret_heads, cfg.window, cfg.ret_window, cfg.topk,
                             dev)
    o = torch.zeros(B, N, cfg.Hq, 128, dtype=torch.bfloat16, device=dev)
    layer(q, k, v, P, o)
    assert layer.device_status() == 0
    qc, kc, vc, Pc = q[0].cpu(), k[0].cpu(), v[0].cpu(), P.cpu()
    res = O.prefill_layer(qc, kc, vc, Pc, cfg.ret_heads, cfg.window, cfg.ret_window, cfg.topk,
                          1 / math.sqrt(128), qblocks=qblocks, heads=heads)
    if check_kt:
        for slot, g in enumerate(layer.kv_used):
            if g in res["kt"]:
                assert_index_close(_f64(layer.kt[0, slot]), kc[:, g, :], Pc[g])
    blocks = layer.blocks.cpu().numpy() if layer.ret else None
    n_amb_rows, worst = 0, (0.0, 0.0)
    outs, refs = [], []
    for (h, i), ref in res["out"].items():
        if h in cfg.ret_heads:
            j = layer.ret.index(h)
            n = min(cfg.topk, i + 1)
            ok, amb, msg = band_check(blocks[0, j, i, :n], res["sel"][(h, i)], res["scores"][(h, i)],
                                      cfg.topk)
            assert ok, f"selection h{h} i{i}: {msg}"
            if not np.array_equal(np.sort(blocks[0, j, i, :n]), res["sel"][(h, i)]):
                # a tolerated near-tie changed the set: the oracle recomputes the
                # row's attention over the GPU's set
                n_amb_rows += 1
                g = O.kv_of(h, cfg.Hq, cfg.Hkv)
                att = O.attended_blocks(blocks[0, j, i, :n], i, cfg.ret_window // 64, cfg.sink_blocks)
                ref = O.sparse_attn_prefill_block(qc[:, h, :], kc[:, g, :], vc[:, g, :], i, att,
                                                  1 / math.sqrt(128))
        outs.append(_f64(o[0, i * 64:(i + 1) * 64, h].cpu()))
        refs.append(ref)
    worst = assert_attn_close(np.stack(outs), np.stack(refs), cfg.name)
    return worst, n_amb_rows


def test_prefill_layer_graph_replay_matches_eager():
    """The layer captured as one CUDA graph reads its inputs at replay: a new
    query gives the same output as an eager call on that query."""
    cfg = synth.TINY_PREFILL
    data = synth.make_prefill(cfg, device=DEV)
    q, k, v, P = data["q"], data["k"], data["v"], data["P"]
    B, N = q.shape[0], q.shape[1]
    layer = rtp.PrefillLayer(B, N, cfg.Hq, cfg.Hkv, cfg.ret_heads, cfg.window, cfg.ret_window, cfg.topk, DEV)
    o_graph = torch.zeros(B, N, cfg.Hq, 128, dtype=torch.bfloat16, device=DEV)
    layer(q, k, v, P, o_graph)
    torch.cuda.synchronize()
    g = layer.graph(q, k, v, P, o_graph)
    q2 = synth.make_prefill(cfg, device=DEV, seed=cfg.seed + 99)["q"]
    q.copy_(q2)
    o_graph.zero_()
    g.replay()
    o_eager = torch.zeros_like(o_graph)
    layer2 = rtp.PrefillLayer(B, N, cfg.Hq, cfg.Hkv, cfg.ret_heads, cfg.window, cfg.ret_window, cfg.topk, DEV)
    layer2(q2, k, v, P, o_eager)
    torch.cuda.synchronize()
    assert layer.device_status() == 0
    assert torch.equal(o_graph, o_eager)


def test_e2e_tiny_prefill_full_oracle():
    cfg = synth.TINY_PREFILL
    data = synth.make_prefill(cfg, device="cpu")
    data = {k: (v.to(DEV) if isinstance(v, torch.Tensor) else v) for k, v in data.items()}
    (max_abs, rel), n_amb = _prefill_e2e(cfg, data, qblocks=None)
    assert n_amb <= 2


def test_e2e_decode_reduced():
    cfg = synth.DECODE_128K
    B, L = 2, 16384
    data = synth.make_decode(cfg, device=DEV, B=B, L=L)
    q, kc, vc, P = data["q"], data["kc"], data["vc"], data["P"]
    step = rtp.DecodeStep(B, L, cfg.Hq, cfg.Hkv, cfg.ret_heads, cfg.window, cfg.ret_window, cfg.topk, DEV)
    kindex = torch.empty(B, cfg.Hkv, L, 16, dtype=torch.bfloat16, device=DEV)
    rtp.index_project(kc, P, list(range(cfg.Hkv)), list(range(cfg.Hkv)), out=kindex)
    o = torch.zeros(B, cfg.Hq, 128, dtype=torch.bfloat16, device=DEV)
    step(q, kc, vc, kindex, P, o)
    torch.cuda.synchronize()
    idx = step.idx.cpu().numpy()
    outs, refs = [], []
    for b in range(B):
        res = O.decode_layer(q[b].cpu(), kc[b].cpu(), vc[b].cpu(), P.cpu(), cfg.ret_heads, cfg.window,
                             cfg.ret_window, cfg.topk, 1 / math.sqrt(128))
        for g in res["kt"]:
            assert_index_close(_f64(kindex[b, g]), kc[b, :, g, :].cpu(), P[g].cpu())
        for h in range(cfg.Hq):
            if h in cfg.ret_heads:
                j = cfg.ret_heads.index(h)
                ok, amb, msg = band_check(idx[b, j], res["sel"][h], res["scores"][h], cfg.topk)
                assert ok, f"b{b} h{h}: {msg}"
                ref = res["out"][h]
                if not np.array_equal(np.sort(idx[b, j]), res["sel"][h]):
                    # tolerated near-tie: the oracle's attention over the GPU's set
                    g = O.kv_of(h, cfg.Hq, cfg.Hkv)
                    att = O.decode_attended(idx[b, j][idx[b, j] >= 0], L, cfg.ret_window, cfg.sink)
                    ref = O.attend_decode(q[b, h].cpu(), kc[b, :, g].cpu(), vc[b, :, g].cpu(), att,
                                          1 / math.sqrt(128))
            else:
                ref = res["out"][h]
            outs.append(_f64(o[b, h].cpu()))
            refs.append(ref)
    assert_attn_close(np.stack(outs), np.stack(refs), "decode")
    # the same step captured as a CUDA graph and replayed with a new query
    o_eager = o.clone()
    g = step.graph(q, kc, vc, kindex, P, o)
    o.zero_()
    g.replay()
    torch.cuda.synchronize()
    assert torch.equal(o, o_eager), "graph replay differs from the eager step"
    q2 = synth.make_decode(cfg, device=DEV, B=B, L=L, seed=cfg.seed + 1)["q"]
    q.copy_(q2)
    g.replay()
    o2 = torch.zeros_like(o)
    step(q2, kc, vc, kindex, P, o2)
    torch.cuda.synchronize()
    assert torch.equal(o, o2), "graph replay with a new query differs from the eager step"


def test_decode_step_equals_the_three_calls():
    """rtp_decode_step (projection, selection and attention in one call, the
    attention starting before the selection ends) gives what the three calls
    give one after another: the same selection bit for bit, and outputs
    within 2^-10 + 2^-6 |o| (the step runs its attention on as many CTAs as
    fit beside the filter, so its partials group the keys differently: each
    partial rounds its probabilities to bf16 against its own running max, and
    the fp32 sums round differently)."""
    cfg = synth.DECODE_128K
    B, L = 3, 20000
    data = synth.make_decode(cfg, device=DEV, B=B, L=L, seed=cfg.seed + 5)
    q, kc, vc, P = data["q"], data["kc"], data["vc"], data["P"]
    kindex = rtp.index_project(kc, P, list(range(cfg.Hkv)), list(range(cfg.Hkv)))
    ret = list(cfg.ret_heads)
    swa_heads = [h for h in range(cfg.Hq) if h not in ret]
    kv_ret = [rtp.kv_of(h, cfg.Hq, cfg.Hkv) for h in ret]
    for window in (8192, 1000):
        o1 = torch.zeros(B, cfg.Hq, 128, dtype=torch.bfloat16, device=DEV)
        idx1 = torch.empty(B, len(ret), cfg.topk, dtype=torch.int32, device=DEV)
        rtp.decode_step(q, P, kindex, kc, vc, o1, ret, idx1, window, swa_heads, window, cfg.topk, sink=1)
        qt = rtp.index_project(q.unsqueeze(1), P, ret, kv_ret, out_dtype=torch.float32).view(B, len(ret), 16)
        idx2 = rtp.select_decode(qt, kindex, kv_ret, cfg.topk)
        o2 = torch.zeros_like(o1)
        rtp.decode_attn_hybrid(q, kc, vc, o2, ret, idx2, window, swa_heads, window, 1)
        torch.cuda.synchronize()
        assert torch.equal(idx1, idx2)
        a, b = o1.float(), o2.float()
        tol = 2.0 ** -10 + torch.maximum(a.abs(), b.abs()) * 2.0 ** -6
        assert bool(((a - b).abs() <= tol).all()), float((a - b).abs().max())


@pytest.mark.parametrize("L,ret_window,swa_window,topk", [(6000, 512, 256, 300), (6000, 256, 1024, 129),
                                                          (700, 4096, 4096, 100), (20000, 8192, 8192, 2048)])
def test_decode_attn_hybrid_matches_oracle(L, ret_window, swa_window, topk):
    """Retrieval and streaming heads in one launch, windows of different sizes."""
    B, Hq, Hkv = 2, 16, 2
    q = _clustered_bf16((B, Hq, 128), 90)
    kc, vc = _clustered_bf16((B, L, Hkv, 128), 91), _randn_bf16((B, L, Hkv, 128), 92)
    ret = [0, 3, 9]
    swa_heads = [h for h in range(Hq) if h not in ret]
    rs = np.random.default_rng(L + topk)
    idx = -np.ones((B, len(ret), topk), np.int32)
    for b in range(B):
        for j in range(len(ret)):
            n = min(topk, L)
            idx[b, j, :n] = np.sort(rs.choice(L, n, replace=False))
    o = torch.zeros(B, Hq, 128, dtype=torch.bfloat16, device=DEV)
    rtp.decode_attn_hybrid(q.to(DEV), kc.to(DEV), vc.to(DEV), o, ret, torch.from_numpy(idx).to(DEV), ret_window,
                           swa_heads, swa_window, sink=1)
    torch.cuda.synchronize()
    o = o.cpu()
    scale = 1 / math.sqrt(128)
    outs, refs = [], []
    for b in range(B):
        for h in range(Hq):
            g = h // (Hq // Hkv)
            if h in ret:
                sel = idx[b, ret.index(h)]
                att = O.decode_attended(sel[sel >= 0], L, ret_window, 1)
            else:
                att = np.arange(max(0, L - swa_window), L)
            outs.append(_f64(o[b, h]))
            refs.append(O.attend_decode(q[b, h], kc[b, :, g], vc[b, :, g], att, scale))
    assert_attn_close(np.stack(outs), np.stack(refs), "hybrid decode")
