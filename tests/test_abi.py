"""CPU checks of the C ABI: the library builds, loads, exports every call the
header declares, and rejects bad arguments on the host before any launch."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "rtp.h")
TEST_HEADER = os.path.join(ROOT, "include", "rtp_testing.h")


@pytest.fixture(scope="module")
def L():
    from long_context_hybrid_b200 import build
    build.build()
    import long_context_hybrid_b200 as rtp
    return rtp.lib()


def declared_symbols(header=HEADER):
    text = open(header).read()
    return sorted(set(re.findall(r"RTP_API\s+[\w\s\*]+?\b(rtp_\w+)\s*\(", text)))


def test_header_declares_the_six_calls():
    syms = declared_symbols()
    for name in ("rtp_index_project", "rtp_select_prefill", "rtp_select_decode",
                 "rtp_sparse_attn_prefill", "rtp_sparse_attn_decode", "rtp_swa"):
        assert name in syms


def test_every_declared_symbol_is_exported(L):
    for name in declared_symbols() + declared_symbols(TEST_HEADER):
        assert hasattr(L, name), name


def test_test_hooks_stay_out_of_the_public_header():
    assert not any("debug" in n for n in declared_symbols())
    assert declared_symbols(TEST_HEADER) == ["rtp_debug_prefill_timeout_probe"]


def test_version_and_status_strings(L):
    assert L.rtp_version() == 1
    for s, name in enumerate(["RTP_OK", "RTP_ERR_INVALID_ARG", "RTP_ERR_UNSUPPORTED", "RTP_ERR_CUDA",
                              "RTP_ERR_TIMEOUT", "RTP_ERR_WORKSPACE"]):
        assert L.rtp_status_string(s).decode() == name
    assert L.rtp_status_string(99).decode() == "RTP_ERR_UNKNOWN"


def test_workspace_sizes(L):
    # Decode selection keeps one fp32 score per (sequence, retrieval head, token).
    assert L.rtp_workspace_size_select_decode(8, 131072, 5, 2048) >= 8 * 5 * 131072 * 4
    assert L.rtp_workspace_size_sparse_attn_decode(8, 131072, 32, 5, 2048, 8192) > 0
    assert L.rtp_workspace_size_swa(8, 1, 131072, 27, 8192) > 0
    assert L.rtp_workspace_size_swa(1, 4096, 4096, 27, 1024) == 256   # status word only


def _heads(vals):
    return (ctypes.c_int32 * len(vals))(*vals)


def test_rejects_bad_arguments_without_launching(L):
    import long_context_hybrid_b200 as rtp
    S = rtp.Strides
    fake = 0x10000   # never dereferenced: validation fails first
    INVALID, UNSUP, WS = 1, 2, 5
    st = S(8192, 512, 128)
    # null pointer
    assert L.rtp_index_project(None, st, 1, 64, 4, fake, 1, 16, _heads([0]), _heads([0]), 1, fake, 0, None) == INVALID
    # r != 16
    assert L.rtp_index_project(fake, st, 1, 64, 4, fake, 1, 8, _heads([0]), _heads([0]), 1, fake, 0, None) == UNSUP
    # head out of range, duplicate heads
    assert L.rtp_index_project(fake, st, 1, 64, 4, fake, 1, 16, _heads([4]), _heads([0]), 1, fake, 0, None) == INVALID
    assert L.rtp_index_project(fake, st, 1, 64, 4, fake, 1, 16, _heads([1, 1]), _heads([0, 0]), 2, fake, 0, None) == INVALID
    # misaligned pointer / stride
    assert L.rtp_index_project(fake + 2, st, 1, 64, 4, fake, 1, 16, _heads([0]), _heads([0]), 1, fake, 0, None) == INVALID
    assert L.rtp_index_project(fake, S(8192, 516, 128), 1, 64, 4, fake, 1, 16, _heads([0]), _heads([0]), 1, fake, 0, None) == INVALID
    # N not a multiple of 64 for prefill selection
    assert L.rtp_select_prefill(fake, fake, 100, 1, 100, 1, 1, 16, _heads([0]), 4, fake, fake, None, 0, None) == UNSUP
    # kv head out of range
    assert L.rtp_select_prefill(fake, fake, 128, 1, 128, 1, 1, 16, _heads([1]), 4, fake, fake, None, 0, None) == INVALID
    # index capacity below the rows used
    assert L.rtp_select_prefill(fake, fake, 64, 1, 128, 1, 1, 16, _heads([0]), 4, fake, fake, fake, 256, None) == INVALID
    assert L.rtp_select_decode(fake, fake, 999, 1, 1000, 1, 1, 16, _heads([0]), 8, fake, fake, 1 << 30, None) == INVALID
    assert L.rtp_decode_step(fake, fake, fake, 639, None, None, fake, S(640 * 256, 256, 128), fake, S(640 * 256, 256, 128), fake,
                             1, 640, 8, 2, _heads([0]), 1, 16, 64, 1, _heads([1]), 1, 64, ctypes.c_float(0.1),
                             fake, fake, 1 << 24, None) == INVALID
    # 8-bit index: groups past the capacity, reversed range, one of codes/scales missing
    assert L.rtp_index_quantize(fake, 128, 1, 2, 0, 3, fake, fake, None) == INVALID
    assert L.rtp_index_quantize(fake, 128, 1, 2, 2, 1, fake, fake, None) == INVALID
    assert L.rtp_select_decode_q8(fake, None, fake, fake, 1000, 1, 1000, 1, 1, 16, _heads([0]), 8, fake, fake,
                                  1 << 30, None) == INVALID
    assert L.rtp_decode_step(fake, fake, fake, 640, fake, None, fake, S(640 * 256, 256, 128), fake,
                             S(640 * 256, 256, 128), fake, 1, 640, 8, 2, _heads([0]), 1, 16, 64, 1, _heads([1]), 1,
                             64, ctypes.c_float(0.1), fake, fake, 1 << 24, None) == INVALID
    # index append: rows past the capacity, r != 16, negative position
    ka = S(4 * 2 * 128, 2 * 128, 128)
    assert L.rtp_index_append(fake, ka, 1, 4, 2, fake, 16, fake, 100, 97, None) == INVALID
    assert L.rtp_index_append(fake, ka, 1, 4, 2, fake, 8, fake, 100, 0, None) == UNSUP
    assert L.rtp_index_append(fake, ka, 1, 4, 2, fake, 16, fake, 100, -1, None) == INVALID
    assert L.rtp_index_append(None, ka, 1, 4, 2, fake, 16, fake, 100, 0, None) == INVALID
    # decode selection without a workspace
    assert L.rtp_select_decode(fake, fake, 1000, 1, 1000, 1, 1, 16, _heads([0]), 8, fake, None, 0, None) == WS
    assert L.rtp_select_decode(fake, fake, 1000, 1, 1000, 1, 1, 16, _heads([0]), 8, fake, fake, 10, None) == WS
    assert L.rtp_select_decode(fake, fake, 1000, 1, 1000, 1, 1, 16, _heads([0]), (1 << 22) + 1, fake, fake, 1 << 30, None) == UNSUP
    # more than 16 KV groups, or more than 16 retrieval heads on one group
    assert L.rtp_select_decode(fake, fake, 1000, 1, 1000, 1, 17, 16, _heads([0]), 8, fake, fake, 1 << 30, None) == UNSUP
    assert L.rtp_select_decode(fake, fake, 1000, 1, 1000, 17, 2, 16, _heads([0] * 17), 8, fake, fake, 1 << 30,
                               None) == UNSUP
    # sparse prefill: bad window / scale / GQA ratio
    qs = S(64 * 8 * 128, 8 * 128, 128)
    ks = S(64 * 2 * 128, 2 * 128, 128)
    assert L.rtp_sparse_attn_prefill(fake, qs, fake, ks, fake, ks, fake, qs, 1, 64, 8, 2, _heads([0]), 1,
                                     fake, fake, 4, 0, 1, ctypes.c_float(0.1), None, 0, None) == INVALID
    assert L.rtp_sparse_attn_prefill(fake, qs, fake, ks, fake, ks, fake, qs, 1, 64, 8, 2, _heads([0]), 1,
                                     fake, fake, 4, 1, 1, ctypes.c_float(-1.0), None, 0, None) == INVALID
    assert L.rtp_sparse_attn_prefill(fake, qs, fake, ks, fake, ks, fake, qs, 1, 64, 8, 3, _heads([0]), 1,
                                     fake, fake, 4, 1, 1, ctypes.c_float(0.1), None, 0, None) == INVALID
    # SWA: query positions past the keys, prefill Nq not a multiple of 64
    assert L.rtp_swa(fake, qs, fake, ks, fake, ks, fake, qs, 1, 64, 64, 1, 8, 2, _heads([1]), 1, 16,
                     ctypes.c_float(0.1), None, 0, None) == INVALID
    assert L.rtp_swa(fake, qs, fake, ks, fake, ks, fake, qs, 1, 65, 65, 0, 8, 2, _heads([1]), 1, 16,
                     ctypes.c_float(0.1), None, 0, None) == UNSUP
    # decode SWA needs a workspace
    assert L.rtp_swa(fake, qs, fake, ks, fake, ks, fake, qs, 1, 1, 640, 639, 8, 2, _heads([1]), 1, 16,
                     ctypes.c_float(0.1), None, 0, None) == WS
    # decode sparse attention: idx null
    assert L.rtp_sparse_attn_decode(fake, fake, ks, fake, ks, fake, 1, 640, 8, 2, _heads([0]), 1, None,
                                    16, 64, 1, ctypes.c_float(0.1), fake, 1 << 20, None) == INVALID
    # fused decode step: retrieval heads need P, the index and idx; workspace checked; sink bound
    f = ctypes.c_float(0.1)
    assert L.rtp_decode_step(fake, None, fake, 640, None, None, fake, ks, fake, ks, fake, 1, 640, 8, 2, _heads([0]), 1, 16, 64, 1,
                             _heads([1]), 1, 64, f, fake, fake, 1 << 24, None) == INVALID
    assert L.rtp_decode_step(fake, fake, fake, 640, None, None, fake, ks, fake, ks, fake, 1, 640, 8, 2, _heads([0]), 1, 16, 64, 1,
                             _heads([1]), 1, 64, f, fake, None, 0, None) == WS
    assert L.rtp_decode_step(fake, fake, fake, 640, None, None, fake, ks, fake, ks, fake, 1, 640, 8, 2, _heads([0]), 1, 16, 64, 65,
                             _heads([1]), 1, 64, f, fake, fake, 1 << 24, None) == INVALID
    assert L.rtp_decode_step(fake, fake, fake, 640, None, None, fake, ks, fake, ks, fake, 1, 640, 8, 2, _heads([0]), 1, (1 << 22) + 1, 64, 1,
                             _heads([1]), 1, 64, f, fake, fake, 1 << 30, None) == UNSUP
    # clustered decode step: clusters required, L0 within L, the clustered
    # selection's token limit, workspace checked
    def step_cl(centroids=fake, L0=100, n=640, cap=640, ws=fake, ws_bytes=1 << 24):
        return L.rtp_decode_step_clustered(fake, fake, fake, cap, centroids, fake, fake, L0, 4, 2, fake, ks, fake, ks,
                                           fake, 1, n, 8, 2, _heads([0]), 1, 16, 64, 1, _heads([1]), 1, 64, f, fake,
                                           ws, ws_bytes, None)
    assert step_cl(centroids=None) == INVALID
    assert step_cl(L0=700) == INVALID
    assert step_cl(cap=600) == INVALID
    assert step_cl(n=300000, cap=300000) == UNSUP
    assert step_cl(ws=None, ws_bytes=0) == WS
    whole = L.rtp_workspace_size_decode_step_clustered(4, 20000, 32, 5, 313, 32, 2048, 4096)
    assert whole >= (L.rtp_workspace_size_decode_attn_hybrid(4, 20000, 32, 2048, 4096)
                     + L.rtp_workspace_size_select_decode_clustered(4, 5, 313, 32, 20000) + 4 * 5 * 16 * 4)
    # its workspace holds the three calls' workspaces
    B, Lc, Hq, Hr, k, w = 4, 20000, 32, 5, 2048, 4096
    whole = L.rtp_workspace_size_decode_step(B, Lc, Hq, Hr, k, w)
    parts = (L.rtp_workspace_size_decode_attn_hybrid(B, Lc, Hq, k, w)
             + L.rtp_workspace_size_select_decode(B, Lc, Hr, k) + B * Hr * 16 * 4)
    assert parts <= whole <= parts + 3 * 256


def test_binding_raises_without_library(tmp_path, monkeypatch):
    import long_context_hybrid_b200 as rtp
    monkeypatch.setattr(rtp, "LIB_PATH", str(tmp_path / "missing.so"))
    monkeypatch.setattr(rtp, "_lib", None)
    with pytest.raises(rtp.RtpError):
        rtp.lib()


def test_timeout_probe_validates_before_launch(L):
    import long_context_hybrid_b200 as rtp
    fn = L.rtp_debug_prefill_timeout_probe
    fn.restype = ctypes.c_int
    fn.argtypes = [ctypes.c_void_p] * 5 + [ctypes.c_size_t, ctypes.c_void_p]
    fake = 0x10000
    assert fn(None, fake, fake, fake, fake, 256, None) == 1          # null input
    assert fn(fake, fake, fake, fake, fake, 16, None) == 5           # workspace too small
