"""K-cache clustering and the two-level decode selection, against the oracle.

Build: every centroid and every assignment bit for bit (both sides compute
the distances op by op in fp32 and sum the centroids exactly in fixed point),
and the member lists exactly the clusters' rows. Selection, stage by stage:
the GPU's probed clusters under the band rule against the oracle's centroid
scores; then the GPU's tokens under the band rule against the oracle's top-k
over the members of the GPU's clusters; then the attention over the GPU's
tokens within the attention tolerance.

Sources: RTPurboV2 article, the sequence-dimension compression paragraph and
the Qwen3-Coder-30B-A3B recipe (the retrieval heads' K cache is clustered).
"""
import math

import numpy as np
import pytest
import torch

import oracle as O
import synth
from helpers import assert_attn_close, band_check

pytestmark = pytest.mark.gpu

rtp = pytest.importorskip("long_context_hybrid_b200")
DEV = "cuda"


@pytest.fixture(scope="module", autouse=True)
def _built():
    from long_context_hybrid_b200 import build
    build.build()
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    rtp.lib()


def _clustered_index(B, Hkv, L, seed, centres=40):
    g = torch.Generator().manual_seed(seed)
    c = torch.randn(centres, 16, generator=g) * 3
    kt = c[torch.randint(0, centres, (B * Hkv * L,), generator=g)] + torch.randn(B * Hkv * L, 16, generator=g) * 0.7
    kt = kt.view(B, Hkv, L, 16).to(torch.bfloat16)
    if L > 300:
        kt[:, :, 200:230] = kt[:, :, 100:101]               # identical rows: exact distance ties
    return kt


@pytest.mark.parametrize("L,S,iters", [(5003, 64, 2), (2560, 64, 0), (2560, 32, 3), (700, 1, 1), (97, 64, 2)])
def test_kcluster_build_matches_oracle_bit_for_bit(L, S, iters):
    B, Hkv = 2, 2
    kt = _clustered_index(B, Hkv, L, L + S)
    cap = L + 11
    kindex = torch.zeros(B, Hkv, cap, 16, dtype=torch.bfloat16, device=DEV)
    kindex[:, :, :L] = kt.to(DEV)
    cl = rtp.kcluster_build(kindex, L, S, iters)
    torch.cuda.synchronize()
    cen, asg = cl.centroids.cpu().numpy(), cl.assign.cpu().numpy()
    off, mem = cl.offsets.cpu().numpy(), cl.members.cpu().numpy()
    for b in range(B):
        for h in range(Hkv):
            mu, a = O.kmeans_index(kt[b, h], S, iters)
            assert np.array_equal(cen[b, h].view(np.uint32), mu.view(np.uint32)), f"centroids b{b} h{h}"
            assert np.array_equal(asg[b, h], a), f"assignment b{b} h{h}"
            assert off[b, h, 0] == 0 and off[b, h, -1] == L and np.all(np.diff(off[b, h]) >= 0)
            for i in range(len(mu)):
                got = np.sort(mem[b, h, off[b, h, i]:off[b, h, i + 1]])
                assert np.array_equal(got, np.flatnonzero(a == i)), f"members b{b} h{h} cluster {i}"


@pytest.mark.parametrize("L0,L,n_probe,topk", [(8192, 8192, 16, 256), (8000, 8100, 8, 300), (4096, 4096, 4, 2048),
                                               (3000, 3000, 200, 64)])
def test_select_decode_clustered_matches_oracle(L0, L, n_probe, topk):
    B, Hkv, kv = 2, 2, [0, 1, 1]
    kt = _clustered_index(B, Hkv, L, L0 + L)
    kindex = kt.to(DEV)
    cl = rtp.kcluster_build(kindex, L0, 64, 2)
    g = torch.Generator().manual_seed(L0)
    qt = torch.randn(B, len(kv), 16, generator=g) * 2
    idx = rtp.select_decode_clustered(qt.to(DEV), kindex, cl, kv, n_probe, topk, L=L).cpu().numpy()
    cen, asg = cl.centroids.cpu().numpy(), cl.assign.cpu().numpy()
    for b in range(B):
        for j, gk in enumerate(kv):
            q = qt[b, j].double().numpy()
            # stage 1: the probed clusters (the GPU's own choice is recovered from
            # its candidates: every selected token's cluster must be probed)
            cs = cen[b, gk].astype(np.float64) @ q
            want = O.topk_desc(cs, n_probe)
            # stage 2: the oracle's top-k over the members of the oracle's clusters
            # plus the appended rows; the band rule on the tokens (the cluster
            # scores themselves are checked through the selection: a cluster that
            # a near-tie swapped would show as a non-ambiguous token difference)
            cand = np.union1d(np.flatnonzero(np.isin(asg[b, gk], want)), np.arange(L0, L))
            sc = kt[b, gk, cand].double().numpy() @ q
            sel = cand[O.topk_desc(sc, topk)]
            got = idx[b, j]
            n = min(topk, len(cand))
            assert np.all(got[n:] == -1) and np.all(np.diff(got[:n]) > 0)
            # compare in candidate-local indices (the band is over candidate scores)
            pos = {u: i for i, u in enumerate(cand)}
            if not all(u in pos for u in got[:n]):
                raise AssertionError(f"b{b} j{j}: a selected token outside the probed clusters")
            ok, amb, msg = band_check([pos[u] for u in got[:n]], [pos[u] for u in sel], sc, topk)
            assert ok, f"b{b} j{j}: {msg}"


def test_clustered_decode_step_attention_matches_oracle():
    cfg = synth.DECODE_128K
    B, L = 2, 16384
    d = synth.make_decode(cfg, device=DEV, B=B, L=L, seed=cfg.seed + 21)
    q, kc, vc, P = d["q"], d["kc"], d["vc"], d["P"]
    kindex = rtp.index_project(kc, P, list(range(cfg.Hkv)), list(range(cfg.Hkv)))
    cl = rtp.kcluster_build(kindex, L, 64, 2)
    ret = list(cfg.ret_heads)
    kv_ret = [h // 8 for h in ret]
    qt = rtp.index_project(q.unsqueeze(1), P, ret, kv_ret, out_dtype=torch.float32).view(B, len(ret), 16)
    idx = rtp.select_decode_clustered(qt, kindex, cl, kv_ret, 32, cfg.topk)
    flat = rtp.select_decode(qt, kindex, kv_ret, cfg.topk)
    swa_heads = [h for h in range(cfg.Hq) if h not in ret]
    o = torch.zeros(B, cfg.Hq, 128, dtype=torch.bfloat16, device=DEV)
    rtp.decode_attn_hybrid(q, kc, vc, o, ret, idx, cfg.ret_window, swa_heads, cfg.window, 1)
    torch.cuda.synchronize()
    idx, flat = idx.cpu().numpy(), flat.cpu().numpy()
    scale = 1 / math.sqrt(128)
    outs, refs, recall = [], [], []
    for b in range(B):
        for j, h in enumerate(ret):
            g = kv_ret[j]
            sel = idx[b, j][idx[b, j] >= 0]
            att = O.decode_attended(sel, L, cfg.ret_window, 1)
            refs.append(O.attend_decode(q[b, h].cpu(), kc[b, :, g].cpu(), vc[b, :, g].cpu(), att, scale))
            outs.append(o[b, h].float().cpu().numpy())
            recall.append(len(np.intersect1d(sel, flat[b, j])) / cfg.topk)
    assert_attn_close(np.stack(outs), np.stack(refs), "clustered decode attention")
    print(f"recall of the flat top-{cfg.topk} by 32 probed clusters of 64: mean {np.mean(recall):.3f}")


def test_clustered_decode_step_call_matches_the_calls_and_the_oracle():
    """rtp_decode_step_clustered (projection, two-level selection and the
    attention streaming its window while the selection runs) selects exactly
    what the separate calls select; its outputs agree with theirs within
    2^-10 + 2^-6 |o| (its attention runs on fewer CTAs, so its partials group
    the keys differently) and with the oracle over its selection."""
    cfg = synth.DECODE_128K
    B, L, L0 = 2, 16384, 16000
    d = synth.make_decode(cfg, device=DEV, B=B, L=L, seed=cfg.seed + 23)
    q, kc, vc, P = d["q"], d["kc"], d["vc"], d["P"]
    kindex = rtp.index_project(kc, P, list(range(cfg.Hkv)), list(range(cfg.Hkv)))
    cl = rtp.kcluster_build(kindex, L0, 64, 2)
    ret = list(cfg.ret_heads)
    kv_ret = [h // 8 for h in ret]
    swa_heads = [h for h in range(cfg.Hq) if h not in ret]
    n_probe = 16
    o1 = torch.zeros(B, cfg.Hq, 128, dtype=torch.bfloat16, device=DEV)
    idx1 = torch.empty(B, len(ret), cfg.topk, dtype=torch.int32, device=DEV)
    rtp.decode_step_clustered(q, P, kindex, cl, kc, vc, o1, ret, idx1, cfg.ret_window, swa_heads, cfg.window,
                              cfg.topk, n_probe, sink=1)
    qt = rtp.index_project(q.unsqueeze(1), P, ret, kv_ret, out_dtype=torch.float32).view(B, len(ret), 16)
    idx2 = rtp.select_decode_clustered(qt, kindex, cl, kv_ret, n_probe, cfg.topk, L=L)
    o2 = torch.zeros_like(o1)
    rtp.decode_attn_hybrid(q, kc, vc, o2, ret, idx2, cfg.ret_window, swa_heads, cfg.window, 1)
    torch.cuda.synchronize()
    assert torch.equal(idx1, idx2)
    a, b = o1.float(), o2.float()
    tol = 2.0 ** -10 + torch.maximum(a.abs(), b.abs()) * 2.0 ** -6
    assert bool(((a - b).abs() <= tol).all()), float((a - b).abs().max())
    idx1 = idx1.cpu().numpy()
    scale = 1 / math.sqrt(128)
    outs, refs = [], []
    for bb in range(B):
        for j, h in enumerate(ret):
            g = kv_ret[j]
            att = O.decode_attended(idx1[bb, j][idx1[bb, j] >= 0], L, cfg.ret_window, 1)
            refs.append(O.attend_decode(q[bb, h].cpu(), kc[bb, :, g].cpu(), vc[bb, :, g].cpu(), att, scale))
            outs.append(o1[bb, h].float().cpu().numpy())
        for h in swa_heads[:4]:
            g = h // 8
            att = np.arange(max(0, L - cfg.window), L)
            refs.append(O.attend_decode(q[bb, h].cpu(), kc[bb, :, g].cpu(), vc[bb, :, g].cpu(), att, scale))
            outs.append(o1[bb, h].float().cpu().numpy())
    assert_attn_close(np.stack(outs), np.stack(refs), "clustered decode step")
