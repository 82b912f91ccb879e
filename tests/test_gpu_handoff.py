"""Prefill -> decode handoff and decode index maintenance, against the oracle.

A 4096-token prompt runs through the prefill layer, which writes the key index
of every KV head into a decode cache index with headroom (rtp_index_append at
row 0) and selects its key blocks from there. Then 16 decode steps follow, the
cache growing by one token per step: the new token's K/V row is written into
the cache, its key index row appended (rtp_index_append at row L-1), and one
rtp_decode_step runs over the L tokens. Every step's selections and outputs
are compared with the oracle's decode over the same L tokens (band rule for
the sets; tolerated near-tie rows recomputed by the oracle over the GPU's
set), and the final index with the oracle's projection of the whole cache.

Sources: RTPurboV2 article (the sparse indexer runs in the decode stage of
the Qwen3-Coder-30B-A3B recipe; keys projected to r = 16); the 128K decode
workload statement (a 16-d key index beside the cache).
"""
import math

import numpy as np
import pytest
import torch

import oracle as O
import synth
from helpers import assert_attn_close, assert_index_close, band_check

pytestmark = pytest.mark.gpu

rtp = pytest.importorskip("long_context_hybrid_b200")
DEV = "cuda"

PROMPT = synth.PrefillConfig("prefill_4k_then_decode", B=2, N=4096, Hq=32, Hkv=4,
                             ret_heads=(0, 7, 13, 19, 26), window=1024, ret_window=1024, topk=16,
                             centres=512, seed=1006)
STEPS = 16
DECODE_TOPK = 256


@pytest.fixture(scope="module", autouse=True)
def _built():
    from long_context_hybrid_b200 import build
    build.build()
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    rtp.lib()


def _f64(t):
    return t.detach().float().cpu().numpy().astype(np.float64)


def test_prefill_then_growing_decode_on_one_index():
    cfg = PROMPT
    B, N, Hq, Hkv, D = cfg.B, cfg.N, cfg.Hq, cfg.Hkv, 128
    scale = 1 / math.sqrt(D)
    d = synth.make_prefill(cfg, device=DEV)
    q, k, v, P = d["q"], d["k"], d["v"], d["P"]
    new = synth.make_prefill(cfg, device=DEV, seed=cfg.seed + 1, N=STEPS)   # the decoded tokens' q, k, v
    cap = N + STEPS + 5                                                       # headroom beyond the last step
    kc = torch.zeros(B, cap, Hkv, D, dtype=torch.bfloat16, device=DEV)
    vc = torch.zeros_like(kc)
    kc[:, :N] = k
    vc[:, :N] = v
    kindex = torch.full((B, Hkv, cap, 16), float("nan"), dtype=torch.bfloat16, device=DEV)

    # prefill writing the decode index; the same layer without it must agree bit for bit
    layer = rtp.PrefillLayer(B, N, Hq, Hkv, cfg.ret_heads, cfg.window, cfg.ret_window, cfg.topk, DEV)
    o = torch.zeros(B, N, Hq, D, dtype=torch.bfloat16, device=DEV)
    layer(q, k, v, P, o, index_out=kindex)
    assert layer.device_status() == 0
    blocks_handoff = layer.blocks.clone()
    o2 = torch.zeros_like(o)
    layer(q, k, v, P, o2)
    torch.cuda.synchronize()
    assert torch.equal(blocks_handoff, layer.blocks)
    assert torch.equal(o, o2)
    # rows past the prompt are untouched until a decode step appends them
    assert torch.isnan(kindex[:, :, N:].float()).all()

    ret = list(cfg.ret_heads)
    step = rtp.DecodeStep(B, cap, Hq, Hkv, ret, cfg.window, cfg.ret_window, DECODE_TOPK, DEV)
    n_tol = 0
    for t in range(STEPS):
        L = N + t + 1
        kc[:, L - 1] = new["k"][:, t]
        vc[:, L - 1] = new["v"][:, t]
        rtp.index_append(new["k"][:, t:t + 1], P, kindex, L - 1)
        qd = new["q"][:, t].contiguous()
        od = torch.zeros(B, Hq, D, dtype=torch.bfloat16, device=DEV)
        step(qd, kc, vc, kindex, P, od, L=L)
        torch.cuda.synchronize()
        idx = step.idx.cpu().numpy()
        outs, refs = [], []
        for b in range(B):
            kcb, vcb = kc[b, :L].cpu(), vc[b, :L].cpu()
            res = O.decode_layer(qd[b].cpu(), kcb, vcb, P.cpu(), ret, cfg.window, cfg.ret_window, DECODE_TOPK,
                                 scale)
            for h in range(Hq):
                ref = res["out"][h]
                if h in ret:
                    j = ret.index(h)
                    ok, amb, msg = band_check(idx[b, j], res["sel"][h], res["scores"][h], DECODE_TOPK)
                    assert ok, f"step {t} b{b} h{h}: {msg}"
                    if not np.array_equal(np.sort(idx[b, j]), res["sel"][h]):
                        n_tol += 1
                        g = h // (Hq // Hkv)
                        att = O.decode_attended(idx[b, j][idx[b, j] >= 0], L, cfg.ret_window, 1)
                        ref = O.attend_decode(qd[b, h].cpu(), kcb[:, g], vcb[:, g], att, scale)
                outs.append(_f64(od[b, h]))
                refs.append(ref)
        assert_attn_close(np.stack(outs), np.stack(refs), f"decode step {t} (L={L})")
    assert n_tol <= STEPS * B * len(ret) // 10
    # the maintained index: every row the oracle's projection of the cache
    L = N + STEPS
    for b in range(B):
        for g in range(Hkv):
            assert_index_close(_f64(kindex[b, g, :L]), kc[b, :L, g].cpu(), P[g].cpu())
    assert torch.isnan(kindex[:, :, L:].float()).all()


def test_index_append_rows_match_index_project():
    """Rows appended as blocks (the tensor-core projection) equal what
    rtp_index_project computes for the whole sequence bit for bit; rows
    appended one at a time (a decode step's row, the small-row kernel, whose
    fp32 summation order differs) lie in their rounding interval of the
    oracle's exact projection; rows past those written stay untouched."""
    g = torch.Generator().manual_seed(5)
    B, n, Hkv = 3, 300, 4
    k = (torch.randn(B, n, Hkv, 128, generator=g) * 1.5).to(torch.bfloat16).to(DEV)
    P = (torch.randn(Hkv, 128, 16, generator=g) / math.sqrt(128)).to(torch.bfloat16).to(DEV)
    full = rtp.index_project(k, P, list(range(Hkv)), list(range(Hkv)))
    cap = n + 7
    kindex = torch.zeros(B, Hkv, cap, 16, dtype=torch.bfloat16, device=DEV)
    rtp.index_append(k[:, :100], P, kindex, 0)          # a block (tensor-core kernel)
    for t in range(100, 140):                           # single rows (decode steps)
        rtp.index_append(k[:, t:t + 1], P, kindex, t)
    rtp.index_append(k[:, 140:], P, kindex, 140)        # the rest
    torch.cuda.synchronize()
    assert torch.equal(kindex[:, :, :100], full[:, :, :100])
    assert torch.equal(kindex[:, :, 140:n], full[:, :, 140:])
    for b in range(B):
        for h in range(Hkv):
            assert_index_close(_f64(kindex[b, h, 100:140]), k[b, 100:140, h].cpu(), P[h].cpu())
    assert torch.all(kindex[:, :, n:] == 0)
