"""The 8-bit key index on the GPU, against the oracle.

Quantiser: codes and scales bit for bit (both sides divide in IEEE fp32 and
round half to even, so every code is decided alike). Selection over the 8-bit
index: the band rule against the oracle's 8-bit scores. Decode step over the
8-bit index: sets under the band rule and outputs within the attention
tolerance, near-tie rows recomputed over the GPU's set.

Source: the Baidu developer article on layered long-context attention,
section on the mixed-precision index system (an 8-bit quantised indexer).
"""
import math
import struct

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


def _index(B, Hkv, L, seed):
    g = torch.Generator().manual_seed(seed)
    mag = torch.empty(B, Hkv, L, 1).uniform_(0.05, 20.0, generator=g)
    kt = (torch.randn(B, Hkv, L, 16, generator=g) * mag).to(torch.bfloat16)
    if L >= 192:
        kt[:, :, 64:128] = 0                                   # an all-zero group: scale 0
        kt[0, 0, 128:192] = torch.tensor([63.5, -127.0, 0.5, 1.5] * 4).to(torch.bfloat16)  # exact ties
    return kt


@pytest.mark.parametrize("L,cap", [(64 * 40, 64 * 40), (5003, 5100), (70, 200)])
def test_quantize_matches_oracle_bit_for_bit(L, cap):
    B, Hkv = 2, 3
    kt = _index(B, Hkv, L, L)
    kindex = torch.zeros(B, Hkv, cap, 16, dtype=torch.bfloat16, device=DEV)
    kindex[:, :, :L] = kt.to(DEV)
    n_full = L // 64
    k8, ks = rtp.index_quantize(kindex, 0, n_full)
    torch.cuda.synchronize()
    k8, ks = k8.cpu().numpy(), ks.cpu().numpy()
    for b in range(B):
        for h in range(Hkv):
            codes, scales = O.quantize_index(kt[b, h])
            assert np.array_equal(k8[b, h, :n_full * 64], codes), f"codes b{b} h{h}"
            got = ks[b, h, :n_full].view(np.uint32)
            assert np.array_equal(got, scales.view(np.uint32)), f"scales b{b} h{h}"
            assert np.all(k8[b, h, n_full * 64:] == 0)     # rows past the full groups untouched


@pytest.mark.parametrize("L,topk", [(5003, 64), (16384, 2048), (40, 16), (64 * 300, 300), (70000, 2048)])
def test_select_decode_q8_matches_oracle(L, topk):
    B, Hkv, kv = 2, 2, [0, 0, 1]
    g = torch.Generator().manual_seed(L + 3)
    c = torch.randn(32, 16, generator=g)
    kt = (c[torch.randint(0, 32, (B * Hkv * L,), generator=g)] + torch.randn(B * Hkv * L, 16, generator=g))
    kt = kt.view(B, Hkv, L, 16).to(torch.bfloat16)
    qt = torch.randn(B, len(kv), 16, generator=g) * 2
    kindex = kt.to(DEV)
    k8, ks = rtp.index_quantize(kindex, 0, L // 64)
    idx = rtp.select_decode_q8(qt.to(DEV), k8, ks, kindex, kv, topk).cpu().numpy()
    n = min(topk, L)
    for b in range(B):
        for j, gk in enumerate(kv):
            codes, scales = O.quantize_index(kt[b, gk])
            sc = O.decode_scores_q8(qt[b, j].double().numpy(), codes, scales, kt[b, gk, len(codes):])
            got = idx[b, j]
            assert np.all(got[n:] == -1) and np.all(np.diff(got[:n]) > 0)
            ok, amb, msg = band_check(got[:n], O.topk_desc(sc, topk), sc, topk)
            assert ok, f"b{b} j{j}: {msg}"


def test_decode_step_over_the_8bit_index_matches_oracle():
    cfg = synth.DECODE_128K
    B, L = 2, 16384 + 37                           # a partial last group
    d = synth.make_decode(cfg, device=DEV, B=B, L=L, seed=cfg.seed + 11)
    q, kc, vc, P = d["q"], d["kc"], d["vc"], d["P"]
    kindex = rtp.index_project(kc, P, list(range(cfg.Hkv)), list(range(cfg.Hkv)))
    k8, ks = rtp.index_quantize(kindex, 0, L // 64)
    step = rtp.DecodeStep(B, L, cfg.Hq, cfg.Hkv, cfg.ret_heads, cfg.window, cfg.ret_window, cfg.topk, DEV)
    o = torch.zeros(B, cfg.Hq, 128, dtype=torch.bfloat16, device=DEV)
    step(q, kc, vc, kindex, P, o, kindex8=k8, kscale=ks)
    torch.cuda.synchronize()
    idx = step.idx.cpu().numpy()
    # the same step over the bf16 index, for the recall of the 8-bit selection
    o16 = torch.zeros_like(o)
    step16 = rtp.DecodeStep(B, L, cfg.Hq, cfg.Hkv, cfg.ret_heads, cfg.window, cfg.ret_window, cfg.topk, DEV)
    step16(q, kc, vc, kindex, P, o16)
    torch.cuda.synchronize()
    idx16 = step16.idx.cpu().numpy()
    scale = 1 / math.sqrt(128)
    outs, refs, recall = [], [], []
    ret = list(cfg.ret_heads)
    for b in range(B):
        res = O.decode_layer(q[b].cpu(), kc[b].cpu(), vc[b].cpu(), P.cpu(), ret, cfg.window, cfg.ret_window,
                             cfg.topk, scale, index_bits=8)
        for h in range(cfg.Hq):
            ref = res["out"][h]
            if h in ret:
                j = ret.index(h)
                ok, amb, msg = band_check(idx[b, j], res["sel"][h], res["scores"][h], cfg.topk)
                assert ok, f"b{b} h{h}: {msg}"
                if not np.array_equal(np.sort(idx[b, j]), res["sel"][h]):
                    g = h // (cfg.Hq // cfg.Hkv)
                    att = O.decode_attended(idx[b, j][idx[b, j] >= 0], L, cfg.ret_window, 1)
                    ref = O.attend_decode(q[b, h].cpu(), kc[b, :, g].cpu(), vc[b, :, g].cpu(), att, scale)
                recall.append(len(np.intersect1d(idx[b, j], idx16[b, j])) / cfg.topk)
            outs.append(_f64(o[b, h]))
            refs.append(ref)
    assert_attn_close(np.stack(outs), np.stack(refs), "decode over the 8-bit index")
    # a diagnostic, not a pin: the 8-bit selection keeps most of the bf16 one
    print(f"recall of the bf16 top-{cfg.topk} by the 8-bit index: mean {np.mean(recall):.4f}, "
          f"min {np.min(recall):.4f}")
    assert np.mean(recall) > 0.8
