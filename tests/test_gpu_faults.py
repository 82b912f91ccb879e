"""Failure detection on the GPU without faulting it.

Every wait inside the tensor-core kernels is bounded. The test hook
rtp_debug_prefill_timeout_probe launches one CTA whose producer withholds the
query tile, so nothing ever completes the barrier the MMA warp waits on: the
wait must run out, the CTA must drain and free its tensor memory, and the
status word must read RTP_ERR_TIMEOUT. The context must stay usable.
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
    fn = m.lib().rtp_debug_prefill_timeout_probe
    fn.restype = ctypes.c_int
    fn.argtypes = [ctypes.c_void_p] * 5 + [ctypes.c_size_t, ctypes.c_void_p]
    return m


def test_withheld_tile_times_out_and_device_stays_usable(rtp):
    dev = torch.device("cuda:0")
    bufs = [torch.zeros(1, 128, 1, 128, dtype=torch.bfloat16, device=dev) for _ in range(4)]
    ws = torch.zeros(256, dtype=torch.uint8, device=dev)
    st = rtp.lib().rtp_debug_prefill_timeout_probe(*(b.data_ptr() for b in bufs), ws.data_ptr(), 256,
                                                   torch.cuda.current_stream().cuda_stream)
    assert st == 0
    assert rtp.lib().rtp_status_string(rtp.workspace_status(ws)).decode() == "RTP_ERR_TIMEOUT"

    # the same kernel, run normally afterwards, is correct
    g = torch.Generator().manual_seed(3)
    q = torch.randn(1, 256, 2, 128, generator=g).to(torch.bfloat16)
    k = torch.randn(1, 256, 1, 128, generator=g).to(torch.bfloat16)
    v = torch.randn(1, 256, 1, 128, generator=g).to(torch.bfloat16)
    o = torch.zeros(1, 256, 2, 128, dtype=torch.bfloat16, device=dev)
    ws2 = torch.zeros(256, dtype=torch.uint8, device=dev)
    rtp.swa(q.to(dev), k.to(dev), v.to(dev), o, [0, 1], 100, ws=ws2)
    assert rtp.workspace_status(ws2) == 0
    for h in (0, 1):
        ref = O.swa_rows(q[0, :, h], k[0, :, 0], v[0, :, 0], np.arange(256), 100, 1 / math.sqrt(128))
        assert_attn_close(o[0, :, h].float().cpu().numpy(), ref, f"head {h}")
