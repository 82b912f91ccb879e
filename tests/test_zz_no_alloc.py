"""The allocation-free decode attention entry point.

rtp_sparse_attn_decode_noalloc serves callers that cannot hand the library
scratch memory (a host framework that owns every device allocation, or a
decode loop that cannot afford cudaMalloc/cudaFree per step): its split-K
partials live in a fixed array inside the library. This test calls it through
the C ABI twice in a row and checks each result against the workspace-taking
rtp_sparse_attn_decode on the same inputs, within the attention tolerance the
other parity tests use, and one sequence of each call against the fp64
oracle. It lives in its own file, collected last.
"""
import ctypes
import math

import numpy as np
import pytest
import torch

import oracle as O
from helpers import assert_attn_close

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def rtp():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from long_context_hybrid_b200 import build
    build.build()
    import long_context_hybrid_b200 as m
    L = m.lib()
    fn = L.rtp_sparse_attn_decode_noalloc
    fn.restype = ctypes.c_int
    fn.argtypes = [ctypes.c_void_p, ctypes.c_void_p, m.Strides, ctypes.c_void_p, m.Strides, ctypes.c_void_p,
                   ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.POINTER(ctypes.c_int32),
                   ctypes.c_int, ctypes.c_void_p, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_float,
                   ctypes.c_void_p]
    return m


def _inputs(seed, B, L, Hq, Hkv, heads, topk, dev):
    g = torch.Generator().manual_seed(seed)
    q = torch.randn(B, Hq, 128, generator=g).to(torch.bfloat16).to(dev)
    kc = torch.randn(B, L, Hkv, 128, generator=g).to(torch.bfloat16).to(dev)
    vc = torch.randn(B, L, Hkv, 128, generator=g).to(torch.bfloat16).to(dev)
    idx = torch.stack([torch.stack([torch.randperm(L, generator=g)[:topk].sort().values
                                    for _ in heads]) for _ in range(B)]).to(torch.int32).to(dev)
    return q, kc, vc, idx


def test_noalloc_matches_workspace_entry_point(rtp):
    dev = torch.device("cuda:0")
    B, L, Hq, Hkv, heads, topk, window, sink = 4, 20000, 32, 4, [0, 7, 13, 19, 26], 2048, 4096, 1
    scale = 1 / math.sqrt(128)
    L_ = rtp.lib()
    harr = (ctypes.c_int32 * len(heads))(*heads)
    stream = torch.cuda.current_stream().cuda_stream
    for call, seed in enumerate((11, 12)):          # two calls in a row, different inputs
        q, kc, vc, idx = _inputs(seed, B, L, Hq, Hkv, heads, topk, dev)
        ref = torch.zeros(B, Hq, 128, dtype=torch.bfloat16, device=dev)
        rtp.sparse_attn_decode(q, kc, vc, ref, heads, idx, window, sink, scale)
        out = torch.zeros(B, Hq, 128, dtype=torch.bfloat16, device=dev)
        st = L_.rtp_sparse_attn_decode_noalloc(q.data_ptr(), kc.data_ptr(), rtp._strides4(kc), vc.data_ptr(),
                                               rtp._strides4(vc), out.data_ptr(), B, L, Hq, Hkv, harr,
                                               len(heads), idx.data_ptr(), topk, window, sink, scale, stream)
        assert st == 0, L_.rtp_status_string(st).decode()
        torch.cuda.synchronize()
        for h in heads:
            assert_attn_close(out[:, h].float().cpu().numpy(), ref[:, h].float().cpu().numpy(),
                              f"call {call} head {h}")
        assert torch.all(out[:, [h for h in range(Hq) if h not in heads]] == 0)
        b = call                                    # one sequence per call against the oracle
        for j, h in enumerate(heads):
            g = h // (Hq // Hkv)
            sel = idx[b, j].cpu().numpy()
            att = O.decode_attended(sel[sel >= 0], L, window, sink)
            ref = O.attend_decode(q[b, h].cpu(), kc[b, :, g].cpu(), vc[b, :, g].cpu(), att, scale)
            assert_attn_close(out[b, h].float().cpu().numpy(), ref, f"call {call} oracle head {h}")


def test_noalloc_rejects_partials_beyond_its_array(rtp):
    dev = torch.device("cuda:0")
    L_ = rtp.lib()
    B, L, Hq, Hkv, heads, topk = 64, 70000, 32, 4, list(range(32)), 4096
    harr = (ctypes.c_int32 * len(heads))(*heads)
    q = torch.zeros(1, dtype=torch.bfloat16, device=dev)  # never read: the size check comes first
    st = L_.rtp_sparse_attn_decode_noalloc(q.data_ptr(), q.data_ptr(), rtp.Strides(L * Hkv * 128, Hkv * 128, 128),
                                           q.data_ptr(), rtp.Strides(L * Hkv * 128, Hkv * 128, 128),
                                           q.data_ptr(), B, L, Hq, Hkv, harr, len(heads), q.data_ptr(), topk,
                                           8192, 1, 0.1, None)
    assert L_.rtp_status_string(st).decode() == "RTP_ERR_WORKSPACE"
