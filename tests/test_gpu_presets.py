"""Static patterns on the same kernels, against the oracle.

* TriangleMix's triangle-shaped mask (TriangleMix interview, 36kr, paragraph
  on the triangle-shaped mask): rtp_triangle_prefill;
* Orthros' two working modes (Orthros article, section on one attention with
  two working modes): sliding-window attention for every token and a full
  cross-attention for the position that predicts the next token
  (OrthrosStep, on rtp_swa);
* a token top-k as large as the cache (k >= L: the selection keeps every
  token, and the decode step becomes a full cross-attention), and top-k
  values beyond 4096.
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


def _f64(t):
    return t.detach().float().cpu().numpy().astype(np.float64)


def _qkv(B, N, Hq, Hkv, seed):
    cfg = synth.PrefillConfig("preset", B=B, N=N, Hq=Hq, Hkv=Hkv, ret_heads=(), window=64, ret_window=64, topk=1,
                              centres=64, seed=seed)
    d = synth.make_prefill(cfg, device="cpu")
    return d["q"], d["k"], d["v"]


# N = 576: an odd number of query blocks; last_tokens = 64: a last region
# shorter than one tile of the banded kernel
@pytest.mark.parametrize("N,sink,wb,last", [(1024, 1, 2, 256), (576, 1, 1, 64), (640, 0, 3, 0), (512, 2, 1, 512),
                                            (1536, 1, 4, 320)])
def test_triangle_prefill_matches_oracle(N, sink, wb, last):
    B, Hq, Hkv = 2, 8, 2
    q, k, v = _qkv(B, N, Hq, Hkv, 2000 + N + last)
    heads = [0, 3, 5, 6]
    o = torch.zeros(B, N, Hq, 128, dtype=torch.bfloat16, device=DEV)
    ws = torch.zeros(256, dtype=torch.uint8, device=DEV)
    rtp.triangle_prefill(q.to(DEV), k.to(DEV), v.to(DEV), o, heads, sink, wb, last, ws=ws)
    assert rtp.workspace_status(ws) == 0
    o = o.cpu()
    scale = 1 / math.sqrt(128)
    rows = np.arange(N)
    for b in range(B):
        for h in heads:
            g = h // (Hq // Hkv)
            ref = O.triangle_rows(q[b, :, h], k[b, :, g], v[b, :, g], rows, sink, wb, last, scale)
            assert_attn_close(_f64(o[b, :, h]), ref, f"b{b} h{h}")
    assert torch.all(o[:, :, [1, 2, 4, 7]] == 0), "unlisted head written"


def test_triangle_prefill_last_region_everywhere_is_dense_causal():
    B, N, Hq, Hkv = 1, 768, 4, 1
    q, k, v = _qkv(B, N, Hq, Hkv, 2100)
    o = torch.zeros(B, N, Hq, 128, dtype=torch.bfloat16, device=DEV)
    rtp.triangle_prefill(q.to(DEV), k.to(DEV), v.to(DEV), o, [2], 1, 1, N)
    ref = torch.nn.functional.scaled_dot_product_attention(
        q[:, :, 2:3].double().transpose(1, 2), k.double().transpose(1, 2), v.double().transpose(1, 2),
        is_causal=True)[0, 0].numpy()
    assert_attn_close(_f64(o[0, :, 2]), ref, "dense causal")


def test_orthros_prefill_and_decode_match_oracle():
    B, N, Hq, Hkv, W, steps = 2, 3072, 32, 4, 512, 4
    q, k, v = _qkv(B, N + steps, Hq, Hkv, 2200)
    qd, kd, vd = q.to(DEV), k.to(DEV), v.to(DEV)
    st = rtp.OrthrosStep(B, N + steps, Hq, Hkv, W, DEV)
    o = torch.zeros(B, N, Hq, 128, dtype=torch.bfloat16, device=DEV)
    o_ca = torch.zeros(B, Hq, 128, dtype=torch.bfloat16, device=DEV)
    st.prefill(qd[:, :N], kd[:, :N], vd[:, :N], o, o_ca)
    torch.cuda.synchronize()
    scale = 1 / math.sqrt(128)
    rows = np.array([0, 1, 511, 512, 1999, N - 1])
    for b in range(B):
        for h in range(0, Hq, 5):
            g = h // (Hq // Hkv)
            ref = O.swa_rows(q[b, :N, h], k[b, :N, g], v[b, :N, g], rows, W, scale)
            assert_attn_close(_f64(o[b, rows, h].cpu()), ref, f"SWA b{b} h{h}")
        outs = [_f64(o_ca[b, h]) for h in range(Hq)]
        refs = [O.dense_decode(q[b, N - 1, h], k[b, :N, h // 8], v[b, :N, h // 8], scale) for h in range(Hq)]
        assert_attn_close(np.stack(outs), np.stack(refs), f"prefill cross-attention b{b}")
    for t in range(steps):
        L = N + t + 1
        od = torch.zeros(B, Hq, 128, dtype=torch.bfloat16, device=DEV)
        oc = torch.zeros_like(od)
        st.decode(qd[:, L - 1].contiguous(), kd, vd, od, oc, L=L)
        torch.cuda.synchronize()
        for b in range(B):
            for h in range(Hq):
                g = h // (Hq // Hkv)
                ref_w = O.attend_decode(q[b, L - 1, h], k[b, :L, g], v[b, :L, g], np.arange(L - W, L), scale)
                ref_c = O.dense_decode(q[b, L - 1, h], k[b, :L, g], v[b, :L, g], scale)
                assert_attn_close(_f64(od[b, h])[None], ref_w[None], f"step {t} SWA b{b} h{h}")
                assert_attn_close(_f64(oc[b, h])[None], ref_c[None], f"step {t} cross-attention b{b} h{h}")


@pytest.mark.parametrize("L,topk", [(20000, 6000), (3000, 3000), (3000, 5000), (70000, 9000)])
def test_select_decode_large_topk(L, topk):
    B, Hkv, kv = 2, 2, [0, 1, 1]
    g = torch.Generator().manual_seed(L + topk)
    kindex = (torch.randn(B, Hkv, L, 16, generator=g)).to(torch.bfloat16)
    qt = torch.randn(B, len(kv), 16, generator=g) * 2
    idx = rtp.select_decode(qt.to(DEV), kindex.to(DEV), kv, topk).cpu().numpy()
    n = min(topk, L)
    for b in range(B):
        for j, gk in enumerate(kv):
            got = idx[b, j]
            assert np.all(got[n:] == -1) and np.all(np.diff(got[:n]) > 0)
            sc = O.decode_scores(qt[b, j].double().numpy(), kindex[b, gk])
            ok, amb, msg = band_check(got[:n], O.topk_desc(sc, topk), sc, topk)
            assert ok, f"b{b} j{j}: {msg}"


def test_decode_step_with_topk_as_large_as_the_cache_is_full_attention():
    """k >= L: every token is selected, so each retrieval head's output is the
    full cross-attention over the cache (the dense preset of the selection)."""
    cfg = synth.DECODE_128K
    B, L = 2, 5000
    d = synth.make_decode(cfg, device=DEV, B=B, L=L, seed=cfg.seed + 9)
    q, kc, vc, P = d["q"], d["kc"], d["vc"], d["P"]
    kindex = rtp.index_project(kc, P, list(range(cfg.Hkv)), list(range(cfg.Hkv)))
    ret = list(cfg.ret_heads)
    step = rtp.DecodeStep(B, L, cfg.Hq, cfg.Hkv, ret, 256, 256, L + 100, DEV)
    o = torch.zeros(B, cfg.Hq, 128, dtype=torch.bfloat16, device=DEV)
    step(q, kc, vc, kindex, P, o)
    torch.cuda.synchronize()
    idx = step.idx.cpu().numpy()
    scale = 1 / math.sqrt(128)
    for b in range(B):
        for j, h in enumerate(ret):
            assert np.array_equal(idx[b, j, :L], np.arange(L)) and np.all(idx[b, j, L:] == -1)
            g = h // (cfg.Hq // cfg.Hkv)
            ref = O.dense_decode(q[b, h].cpu(), kc[b, :, g].cpu(), vc[b, :, g].cpu(), scale)
            assert_attn_close(_f64(o[b, h])[None], ref[None], f"b{b} h{h}")
