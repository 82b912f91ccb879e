"""Python binding of librtp.so, the head-wise hybrid attention library.

Argument marshalling only: every step of the computation runs in the CUDA
kernels behind the C ABI (``include/rtp.h``). Tensors are torch CUDA tensors
(PyTorch provides device memory and streams); each function passes raw
pointers, element strides and the current stream to the matching C call and
raises ``RtpError`` on any status other than RTP_OK. There is no fallback: if
the library is missing, the first call raises.
"""
from __future__ import annotations

import ctypes
import math
import os
from typing import Optional, Sequence

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "librtp.so")

RTP_OK, RTP_BF16, RTP_F32 = 0, 0, 1
D_HEAD, R_INDEX, BLOCK = 128, 16, 64


class RtpError(RuntimeError):
    pass


class Strides(ctypes.Structure):
    _fields_ = [("b", ctypes.c_int64), ("n", ctypes.c_int64), ("h", ctypes.c_int64)]


_lib = None
_c_i32p = ctypes.POINTER(ctypes.c_int32)
_P = ctypes.c_void_p
_I = ctypes.c_int
_F = ctypes.c_float
_SZ = ctypes.c_size_t
_L = ctypes.c_int64

_SIGNATURES = {
    "rtp_status_string": (ctypes.c_char_p, [_I]),
    "rtp_version": (_I, []),
    "rtp_get_device_status": (_I, [_P, _P, ctypes.POINTER(ctypes.c_int)]),
    "rtp_index_project": (_I, [_P, Strides, _I, _I, _I, _P, _I, _I, _c_i32p, _c_i32p, _I, _P, _I, _P]),
    "rtp_workspace_size_select_prefill": (_SZ, [_I, _I, _I, _I]),
    "rtp_index_append": (_I, [_P, Strides, _I, _I, _I, _P, _I, _P, _L, _I, _P]),
    "rtp_select_prefill": (_I, [_P, _P, _L, _I, _I, _I, _I, _I, _c_i32p, _I, _P, _P, _P, _SZ, _P]),
    "rtp_workspace_size_select_decode": (_SZ, [_I, _I, _I, _I]),
    "rtp_select_decode": (_I, [_P, _P, _L, _I, _I, _I, _I, _I, _c_i32p, _I, _P, _P, _SZ, _P]),
    "rtp_index_quantize": (_I, [_P, _L, _I, _I, _I, _I, _P, _P, _P]),
    "rtp_workspace_size_kcluster_build": (_SZ, [_I, _I, _I, _I]),
    "rtp_kcluster_build": (_I, [_P, _L, _I, _I, _I, _I, _I, _P, _P, _P, _P, _P, _SZ, _P]),
    "rtp_workspace_size_select_decode_clustered": (_SZ, [_I, _I, _I, _I, _I]),
    "rtp_select_decode_clustered": (_I, [_P, _P, _L, _P, _P, _P, _I, _I, _I, _I, _I, _I, _c_i32p, _I, _I, _P, _P, _SZ,
                                         _P]),
    "rtp_select_decode_q8": (_I, [_P, _P, _P, _P, _L, _I, _I, _I, _I, _I, _c_i32p, _I, _P, _P, _SZ, _P]),
    "rtp_workspace_size_sparse_attn_prefill": (_SZ, [_I, _I, _I, _I]),
    "rtp_sparse_attn_prefill": (_I, [_P, Strides, _P, Strides, _P, Strides, _P, Strides, _I, _I, _I,
                                     _I, _c_i32p, _I, _P, _P, _I, _I, _I, _F, _P, _SZ, _P]),
    "rtp_workspace_size_triangle_prefill": (_SZ, []),
    "rtp_triangle_prefill": (_I, [_P, Strides, _P, Strides, _P, Strides, _P, Strides, _I, _I, _I, _I, _c_i32p, _I,
                                  _I, _I, _I, _F, _P, _SZ, _P]),
    "rtp_workspace_size_sparse_attn_decode": (_SZ, [_I, _I, _I, _I, _I, _I]),
    "rtp_sparse_attn_decode": (_I, [_P, _P, Strides, _P, Strides, _P, _I, _I, _I, _I, _c_i32p, _I,
                                    _P, _I, _I, _I, _F, _P, _SZ, _P]),
    "rtp_workspace_size_decode_attn_hybrid": (_SZ, [_I, _I, _I, _I, _I]),
    "rtp_decode_attn_hybrid": (_I, [_P, _P, Strides, _P, Strides, _P, _I, _I, _I, _I, _c_i32p, _I, _P, _I,
                                    _I, _I, _c_i32p, _I, _I, _F, _P, _SZ, _P]),
    "rtp_workspace_size_decode_step": (_SZ, [_I, _I, _I, _I, _I, _I]),
    "rtp_decode_step": (_I, [_P, _P, _P, _L, _P, _P, _P, Strides, _P, Strides, _P, _I, _I, _I, _I, _c_i32p, _I, _I,
                             _I, _I,
                             _c_i32p, _I, _I, _F, _P, _P, _SZ, _P]),
    "rtp_workspace_size_decode_step_clustered": (_SZ, [_I, _I, _I, _I, _I, _I, _I, _I]),
    "rtp_decode_step_clustered": (_I, [_P, _P, _P, _L, _P, _P, _P, _I, _I, _I, _P, Strides, _P, Strides, _P, _I, _I,
                                       _I, _I, _c_i32p, _I, _I, _I, _I, _c_i32p, _I, _I, _F, _P, _P, _SZ, _P]),
    "rtp_workspace_size_swa": (_SZ, [_I, _I, _I, _I, _I]),
    "rtp_swa": (_I, [_P, Strides, _P, Strides, _P, Strides, _P, Strides, _I, _I, _I, _I, _I, _I,
                     _c_i32p, _I, _I, _F, _P, _SZ, _P]),
}


def lib() -> ctypes.CDLL:
    """The loaded librtp.so (raises if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RtpError(f"{LIB_PATH} is missing: build it with "
                           "`python -m long_context_hybrid_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in _SIGNATURES.items():
            fn = getattr(L, name)
            fn.restype, fn.argtypes = res, args
        _lib = L
    return _lib


def _check(status: int, what: str) -> None:
    if status != RTP_OK:
        raise RtpError(f"{what}: {lib().rtp_status_string(status).decode()}")


def _i32(values: Sequence[int]):
    arr = (ctypes.c_int32 * len(values))(*[int(v) for v in values])
    return arr


def _strides4(t: torch.Tensor) -> Strides:
    assert t.dim() == 4 and t.stride(3) == 1, "expected [B, N, H, D] with contiguous D"
    return Strides(t.stride(0), t.stride(1), t.stride(2))


def _stream(stream: Optional[torch.cuda.Stream]) -> int:
    s = stream if stream is not None else torch.cuda.current_stream()
    return s.cuda_stream


def _ws(nbytes: int, device, ws: Optional[torch.Tensor]):
    if nbytes == 0:
        return None, 0
    if ws is not None and ws.numel() * ws.element_size() >= nbytes:
        return ws.data_ptr(), ws.numel() * ws.element_size()
    buf = torch.empty(nbytes, dtype=torch.uint8, device=device)
    return buf, nbytes


def _wsptr(buf):
    if buf is None:
        return None
    return buf if isinstance(buf, int) else buf.data_ptr()


def workspace_status(ws: torch.Tensor, stream=None) -> int:
    """Synchronises the stream and returns the status word the last call that
    used ``ws`` left there (0 = RTP_OK, 4 = RTP_ERR_TIMEOUT)."""
    out = ctypes.c_int(0)
    _check(lib().rtp_get_device_status(ws.data_ptr(), _stream(stream), ctypes.byref(out)),
           "rtp_get_device_status")
    return out.value


def kv_of(h: int, Hq: int, Hkv: int) -> int:
    return h // (Hq // Hkv)


# ---------------------------------------------------------------------------
# The six calls
# ---------------------------------------------------------------------------
def index_project(x: torch.Tensor, P: torch.Tensor, heads: Sequence[int], proj_of: Sequence[int],
                  out_dtype=torch.bfloat16, out: Optional[torch.Tensor] = None, stream=None):
    """x [B,N,Hx,D] bf16, P [Hp,D,r] bf16 -> out [B, len(heads), N, r]."""
    B, N, Hx, _ = x.shape
    Hp, _, r = P.shape
    if out is None:
        out = torch.empty(B, len(heads), N, r, dtype=out_dtype, device=x.device)
    dt = RTP_F32 if out.dtype == torch.float32 else RTP_BF16
    _check(lib().rtp_index_project(x.data_ptr(), _strides4(x), B, N, Hx, P.data_ptr(), Hp, r,
                                   _i32(heads), _i32(proj_of), len(heads), out.data_ptr(), dt,
                                   _stream(stream)), "rtp_index_project")
    return out


def index_append(k: torch.Tensor, P: torch.Tensor, kindex: torch.Tensor, pos: int, stream=None):
    """Projects the keys k [B, n_new, Hkv, D] (every KV head, P [Hkv, D, r])
    into rows pos .. pos + n_new - 1 of the key index kindex [B, Hkv, cap, r]."""
    B, n_new, Hkv, _ = k.shape
    assert kindex.is_contiguous() and kindex.shape[:2] == (B, Hkv)
    _check(lib().rtp_index_append(k.data_ptr(), _strides4(k), B, n_new, Hkv, P.data_ptr(), P.shape[2],
                                  kindex.data_ptr(), kindex.shape[2], pos, _stream(stream)), "rtp_index_append")
    return kindex


def select_prefill(qt: torch.Tensor, kt: torch.Tensor, kv_of_ret: Sequence[int], topk: int,
                   blocks: Optional[torch.Tensor] = None, counts: Optional[torch.Tensor] = None,
                   ws: Optional[torch.Tensor] = None, stream=None):
    """qt [B,Hr,N,r], kt [B,Hkv,cap,r] bf16 (rows 0..N-1 used, cap >= N)
    -> (blocks [B,Hr,N/64,k], counts [B,Hr,N/64])."""
    B, Hr, N, r = qt.shape
    Hkv = kt.shape[1]
    assert kt.is_contiguous()
    nb = N // BLOCK
    if blocks is None:
        blocks = torch.empty(B, Hr, nb, topk, dtype=torch.int32, device=qt.device)
    if counts is None:
        counts = torch.empty(B, Hr, nb, dtype=torch.int32, device=qt.device)
    need = lib().rtp_workspace_size_select_prefill(B, N, Hr, topk)
    buf, nbytes = _ws(need, qt.device, ws)
    _check(lib().rtp_select_prefill(qt.data_ptr(), kt.data_ptr(), kt.shape[2], B, N, Hr, Hkv, r, _i32(kv_of_ret),
                                    topk, blocks.data_ptr(), counts.data_ptr(), _wsptr(buf), nbytes,
                                    _stream(stream)), "rtp_select_prefill")
    return blocks, counts


def select_decode(qt: torch.Tensor, kindex: torch.Tensor, kv_of_ret: Sequence[int], topk: int,
                  idx: Optional[torch.Tensor] = None, ws: Optional[torch.Tensor] = None, stream=None,
                  L: Optional[int] = None):
    """qt [B,Hr,r] fp32, kindex [B,Hkv,cap,r] bf16 (rows 0..L-1 used; L
    defaults to cap) -> idx [B,Hr,k] int32 ascending."""
    B, Hr, r = qt.shape
    Hkv = kindex.shape[1]
    L = kindex.shape[2] if L is None else L
    assert kindex.is_contiguous()
    if idx is None:
        idx = torch.empty(B, Hr, topk, dtype=torch.int32, device=qt.device)
    need = lib().rtp_workspace_size_select_decode(B, L, Hr, topk)
    buf, nbytes = _ws(need, qt.device, ws)
    _check(lib().rtp_select_decode(qt.data_ptr(), kindex.data_ptr(), kindex.shape[2], B, L, Hr, Hkv, r,
                                   _i32(kv_of_ret), topk, idx.data_ptr(), _wsptr(buf), nbytes,
                                   _stream(stream)), "rtp_select_decode")
    return idx


def index_quantize(kindex: torch.Tensor, g0: int, g1: int, kindex8: Optional[torch.Tensor] = None,
                   kscale: Optional[torch.Tensor] = None, stream=None):
    """8-bit codes and per-64-token scales of groups g0..g1-1 of the bf16 key
    index kindex [B,Hkv,cap,r] -> (kindex8 int8 [B,Hkv,cap,r], kscale fp32
    [B,Hkv,ceil(cap/64)])."""
    B, Hkv, cap, r = kindex.shape
    assert kindex.is_contiguous()
    if kindex8 is None:
        kindex8 = torch.zeros(B, Hkv, cap, r, dtype=torch.int8, device=kindex.device)
    if kscale is None:
        kscale = torch.zeros(B, Hkv, (cap + 63) // 64, dtype=torch.float32, device=kindex.device)
    _check(lib().rtp_index_quantize(kindex.data_ptr(), cap, B, Hkv, g0, g1, kindex8.data_ptr(), kscale.data_ptr(),
                                    _stream(stream)), "rtp_index_quantize")
    return kindex8, kscale


def select_decode_q8(qt: torch.Tensor, kindex8: torch.Tensor, kscale: torch.Tensor, kindex: torch.Tensor,
                     kv_of_ret: Sequence[int], topk: int, idx: Optional[torch.Tensor] = None,
                     ws: Optional[torch.Tensor] = None, stream=None, L: Optional[int] = None):
    """Token top-k over the 8-bit key index (full 64-token groups) and the bf16
    rows of the partial last group -> idx [B,Hr,k] int32 ascending."""
    B, Hr, r = qt.shape
    Hkv = kindex.shape[1]
    L = kindex.shape[2] if L is None else L
    if idx is None:
        idx = torch.empty(B, Hr, topk, dtype=torch.int32, device=qt.device)
    need = lib().rtp_workspace_size_select_decode(B, L, Hr, topk)
    buf, nbytes = _ws(need, qt.device, ws)
    _check(lib().rtp_select_decode_q8(qt.data_ptr(), kindex8.data_ptr(), kscale.data_ptr(), kindex.data_ptr(),
                                      kindex.shape[2], B, L, Hr, Hkv, r, _i32(kv_of_ret), topk, idx.data_ptr(),
                                      _wsptr(buf), nbytes, _stream(stream)), "rtp_select_decode_q8")
    return idx


class KeyClusters:
    """The clustered key index of a cache (rtp_kcluster_build): centroids
    [B,Hkv,C,r] fp32, assign [B,Hkv,L0], and the members of every cluster as
    offsets [B,Hkv,C+1] / members [B,Hkv,L0] (int32), over the first L0 rows."""

    def __init__(self, centroids, assign, offsets, members, L0):
        self.centroids, self.assign, self.offsets, self.members, self.L0 = centroids, assign, offsets, members, L0

    @property
    def C(self):
        return self.centroids.shape[2]


def kcluster_build(kindex: torch.Tensor, L: int, cluster_size: int = 64, iters: int = 2, ws=None,
                   stream=None) -> KeyClusters:
    """Lloyd k-means over rows 0..L-1 of every (sequence, KV head) of the key
    index kindex [B,Hkv,cap,r]."""
    B, Hkv, cap, r = kindex.shape
    assert kindex.is_contiguous()
    C = (L + cluster_size - 1) // cluster_size
    dev = kindex.device
    cen = torch.empty(B, Hkv, C, r, dtype=torch.float32, device=dev)
    asg = torch.empty(B, Hkv, L, dtype=torch.int32, device=dev)
    off = torch.empty(B, Hkv, C + 1, dtype=torch.int32, device=dev)
    mem = torch.empty(B, Hkv, L, dtype=torch.int32, device=dev)
    need = lib().rtp_workspace_size_kcluster_build(B, Hkv, L, cluster_size)
    buf, nbytes = _ws(need, dev, ws)
    _check(lib().rtp_kcluster_build(kindex.data_ptr(), cap, B, Hkv, L, cluster_size, iters, cen.data_ptr(),
                                    asg.data_ptr(), off.data_ptr(), mem.data_ptr(), _wsptr(buf), nbytes,
                                    _stream(stream)), "rtp_kcluster_build")
    return KeyClusters(cen, asg, off, mem, L)


def select_decode_clustered(qt: torch.Tensor, kindex: torch.Tensor, clusters: KeyClusters,
                            kv_of_ret: Sequence[int], n_probe: int, topk: int, L: Optional[int] = None,
                            idx: Optional[torch.Tensor] = None, ws: Optional[torch.Tensor] = None, stream=None):
    """Two-level token top-k: the n_probe best clusters by centroid score, then
    the top-k tokens among their members and the rows appended after the
    build (clusters.L0 .. L-1) -> idx [B,Hr,topk] int32 ascending."""
    B, Hr, r = qt.shape
    Hkv, cap = kindex.shape[1], kindex.shape[2]
    L = cap if L is None else L
    if idx is None:
        idx = torch.empty(B, Hr, topk, dtype=torch.int32, device=qt.device)
    need = lib().rtp_workspace_size_select_decode_clustered(B, Hr, clusters.C, n_probe, L)
    buf, nbytes = _ws(need, qt.device, ws)
    _check(lib().rtp_select_decode_clustered(qt.data_ptr(), kindex.data_ptr(), cap, clusters.centroids.data_ptr(),
                                             clusters.offsets.data_ptr(), clusters.members.data_ptr(), B,
                                             clusters.L0, L, Hr, Hkv, clusters.C, _i32(kv_of_ret), n_probe, topk,
                                             idx.data_ptr(), _wsptr(buf), nbytes, _stream(stream)),
           "rtp_select_decode_clustered")
    return idx


def sparse_attn_prefill(q, k, v, o, heads: Sequence[int], blocks, counts, window_blocks: int,
                        sink_blocks: int = 1, scale: Optional[float] = None,
                        ws: Optional[torch.Tensor] = None, stream=None):
    """Retrieval-head prefill attention; writes o[:, :, heads, :]."""
    B, N, Hq, D = q.shape
    Hkv = k.shape[2]
    topk = blocks.shape[-1]
    scale = 1.0 / math.sqrt(D) if scale is None else scale
    need = lib().rtp_workspace_size_sparse_attn_prefill(B, N, len(heads), topk)
    buf, nbytes = _ws(need, q.device, ws)
    _check(lib().rtp_sparse_attn_prefill(q.data_ptr(), _strides4(q), k.data_ptr(), _strides4(k),
                                         v.data_ptr(), _strides4(v), o.data_ptr(), _strides4(o),
                                         B, N, Hq, Hkv, _i32(heads), len(heads), blocks.data_ptr(),
                                         counts.data_ptr(), topk, window_blocks, sink_blocks, scale,
                                         _wsptr(buf), nbytes, _stream(stream)),
           "rtp_sparse_attn_prefill")
    return o


def triangle_prefill(q, k, v, o, heads: Sequence[int], sink_blocks: int, window_blocks: int, last_tokens: int,
                     scale: Optional[float] = None, ws: Optional[torch.Tensor] = None, stream=None):
    """Triangle-shaped-mask prefill attention (streaming region: sink and band
    blocks; last Q-K region: the last ``last_tokens`` rows see every key);
    writes o[:, :, heads, :]. q/o [B,N,Hq,D], k/v [B,N,Hkv,D]."""
    B, N, Hq, D = q.shape
    Hkv = k.shape[2]
    scale = 1.0 / math.sqrt(D) if scale is None else scale
    buf, nbytes = _ws(lib().rtp_workspace_size_triangle_prefill(), q.device, ws)
    _check(lib().rtp_triangle_prefill(q.data_ptr(), _strides4(q), k.data_ptr(), _strides4(k), v.data_ptr(),
                                      _strides4(v), o.data_ptr(), _strides4(o), B, N, Hq, Hkv, _i32(heads),
                                      len(heads), sink_blocks, window_blocks, last_tokens, scale, _wsptr(buf),
                                      nbytes, _stream(stream)), "rtp_triangle_prefill")
    return o


def sparse_attn_decode(q, kc, vc, o, heads: Sequence[int], idx, window: int, sink: int = 1,
                       scale: Optional[float] = None, ws: Optional[torch.Tensor] = None, stream=None):
    """Retrieval-head decode attention. q/o [B,Hq,D], kc/vc [B,L,Hkv,D]."""
    B, Hq, D = q.shape
    L, Hkv = kc.shape[1], kc.shape[2]
    topk = idx.shape[-1]
    scale = 1.0 / math.sqrt(D) if scale is None else scale
    need = lib().rtp_workspace_size_sparse_attn_decode(B, L, Hq, len(heads), topk, window)
    buf, nbytes = _ws(need, q.device, ws)
    _check(lib().rtp_sparse_attn_decode(q.data_ptr(), kc.data_ptr(), _strides4(kc), vc.data_ptr(),
                                        _strides4(vc), o.data_ptr(), B, L, Hq, Hkv, _i32(heads),
                                        len(heads), idx.data_ptr(), topk, window, sink, scale,
                                        _wsptr(buf), nbytes, _stream(stream)),
           "rtp_sparse_attn_decode")
    return o


def decode_attn_hybrid(q, kc, vc, o, ret_heads: Sequence[int], idx, ret_window: int,
                       swa_heads: Sequence[int], swa_window: int, sink: int = 1,
                       scale: Optional[float] = None, ws: Optional[torch.Tensor] = None, stream=None):
    """Decode attention of retrieval heads (idx + sink + window) and streaming
    heads (window) in one launch. q/o [B,Hq,D], kc/vc [B,L,Hkv,D]."""
    B, Hq, D = q.shape
    L, Hkv = kc.shape[1], kc.shape[2]
    topk = idx.shape[-1] if idx is not None else 0
    scale = 1.0 / math.sqrt(D) if scale is None else scale
    wmax = max(ret_window if ret_heads else 0, swa_window if swa_heads else 0)
    need = lib().rtp_workspace_size_decode_attn_hybrid(B, L, Hq, topk, wmax)
    buf, nbytes = _ws(need, q.device, ws)
    _check(lib().rtp_decode_attn_hybrid(q.data_ptr(), kc.data_ptr(), _strides4(kc), vc.data_ptr(), _strides4(vc),
                                        o.data_ptr(), B, L, Hq, Hkv, _i32(ret_heads), len(ret_heads),
                                        idx.data_ptr() if idx is not None else None, topk, ret_window, sink,
                                        _i32(swa_heads), len(swa_heads), swa_window, scale, _wsptr(buf), nbytes,
                                        _stream(stream)), "rtp_decode_attn_hybrid")
    return o


def decode_step(q, P, kindex, kc, vc, o, ret_heads: Sequence[int], idx, ret_window: int,
                swa_heads: Sequence[int], swa_window: int, topk: int, sink: int = 1,
                scale: Optional[float] = None, ws: Optional[torch.Tensor] = None, stream=None,
                L: Optional[int] = None, kindex8: Optional[torch.Tensor] = None,
                kscale: Optional[torch.Tensor] = None):
    """One decode step in one call: q~ projection, top-k selection into idx and
    the attention of retrieval and streaming heads. q/o [B,Hq,D], P [Hkv,D,r],
    kindex [B,Hkv,cap,r], kc/vc [B,cap,Hkv,D] (rows 0..L-1 are the cache; L
    defaults to kc's length), idx [B,Hr,topk] int32 (written)."""
    B, Hq, D = q.shape
    Hkv = kc.shape[2]
    L = kc.shape[1] if L is None else L
    if ret_heads:
        assert kindex.is_contiguous() and kindex.shape[2] >= L
    scale = 1.0 / math.sqrt(D) if scale is None else scale
    wmax = max(ret_window if ret_heads else 0, swa_window if swa_heads else 0)
    need = lib().rtp_workspace_size_decode_step(B, L, Hq, len(ret_heads), topk, wmax)
    buf, nbytes = _ws(need, q.device, ws)
    _check(lib().rtp_decode_step(q.data_ptr(), P.data_ptr() if ret_heads else None,
                                 kindex.data_ptr() if ret_heads else None, kindex.shape[2] if ret_heads else 0,
                                 kindex8.data_ptr() if kindex8 is not None else None,
                                 kscale.data_ptr() if kscale is not None else None,
                                 kc.data_ptr(), _strides4(kc),
                                 vc.data_ptr(), _strides4(vc), o.data_ptr(), B, L, Hq, Hkv, _i32(ret_heads),
                                 len(ret_heads), topk, ret_window, sink, _i32(swa_heads), len(swa_heads),
                                 swa_window, scale, idx.data_ptr() if ret_heads else None, _wsptr(buf), nbytes,
                                 _stream(stream)), "rtp_decode_step")
    return o


def decode_step_clustered(q, P, kindex, clusters: "KeyClusters", kc, vc, o, ret_heads: Sequence[int], idx,
                          ret_window: int, swa_heads: Sequence[int], swa_window: int, topk: int, n_probe: int,
                          sink: int = 1, scale: Optional[float] = None, ws: Optional[torch.Tensor] = None,
                          stream=None, L: Optional[int] = None):
    """One decode step in one call with the two-level clustered selection:
    q~ projection, the n_probe best clusters then the top-k tokens among
    their members and the rows appended after the build (into idx), and the
    attention of retrieval and streaming heads. Shapes as decode_step;
    clusters from kcluster_build over the first clusters.L0 rows."""
    B, Hq, D = q.shape
    Hkv = kc.shape[2]
    L = kc.shape[1] if L is None else L
    assert kindex.is_contiguous() and kindex.shape[2] >= L
    scale = 1.0 / math.sqrt(D) if scale is None else scale
    wmax = max(ret_window, swa_window if swa_heads else 0)
    need = lib().rtp_workspace_size_decode_step_clustered(B, L, Hq, len(ret_heads), clusters.C, n_probe, topk, wmax)
    buf, nbytes = _ws(need, q.device, ws)
    _check(lib().rtp_decode_step_clustered(q.data_ptr(), P.data_ptr(), kindex.data_ptr(), kindex.shape[2],
                                           clusters.centroids.data_ptr(), clusters.offsets.data_ptr(),
                                           clusters.members.data_ptr(), clusters.L0, clusters.C, n_probe,
                                           kc.data_ptr(), _strides4(kc), vc.data_ptr(), _strides4(vc), o.data_ptr(),
                                           B, L, Hq, Hkv, _i32(ret_heads), len(ret_heads), topk, ret_window, sink,
                                           _i32(swa_heads), len(swa_heads), swa_window, scale, idx.data_ptr(),
                                           _wsptr(buf), nbytes, _stream(stream)), "rtp_decode_step_clustered")
    return o


def swa(q, k, v, o, heads: Sequence[int], window: int, q_pos0: int = 0,
        scale: Optional[float] = None, ws: Optional[torch.Tensor] = None, stream=None):
    """Streaming-head sliding-window attention. q/o [B,Nq,Hq,D], k/v [B,Nk,Hkv,D]."""
    B, Nq, Hq, D = q.shape
    Nk, Hkv = k.shape[1], k.shape[2]
    scale = 1.0 / math.sqrt(D) if scale is None else scale
    need = lib().rtp_workspace_size_swa(B, Nq, Nk, len(heads), window)
    buf, nbytes = _ws(need, q.device, ws)
    _check(lib().rtp_swa(q.data_ptr(), _strides4(q), k.data_ptr(), _strides4(k), v.data_ptr(),
                         _strides4(v), o.data_ptr(), _strides4(o), B, Nq, Nk, q_pos0, Hq, Hkv,
                         _i32(heads), len(heads), window, scale, _wsptr(buf), nbytes,
                         _stream(stream)), "rtp_swa")
    return o


# ---------------------------------------------------------------------------
# One layer, composed from the six calls
# ---------------------------------------------------------------------------
class PrefillLayer:
    """One prefill layer: indexer projection, block selection, sparse attention
    on retrieval heads and SWA on streaming heads, with buffers kept across calls."""

    def __init__(self, B, N, Hq, Hkv, ret_heads, window, ret_window, topk, device,
                 sink_blocks=1, scale=None):
        self.B, self.N, self.Hq, self.Hkv = B, N, Hq, Hkv
        self.ret = list(ret_heads)
        self.swa_heads = [h for h in range(Hq) if h not in set(self.ret)]
        self.window, self.topk, self.sink_blocks = window, topk, sink_blocks
        self.window_blocks = ret_window // BLOCK
        self.scale = 1.0 / math.sqrt(D_HEAD) if scale is None else scale
        self.kv_ret = [kv_of(h, Hq, Hkv) for h in self.ret]
        self.kv_used = sorted(set(self.kv_ret))
        self.kv_slot = [self.kv_used.index(g) for g in self.kv_ret]
        nb = N // BLOCK
        self.ws_sparse = torch.zeros(lib().rtp_workspace_size_sparse_attn_prefill(B, N, max(1, len(self.ret)), topk),
                                     dtype=torch.uint8, device=device)
        self.ws_swa = torch.zeros(lib().rtp_workspace_size_swa(B, N, N, max(1, len(self.swa_heads)), window),
                                  dtype=torch.uint8, device=device)
        self.ws_sel = torch.zeros(lib().rtp_workspace_size_select_prefill(B, N, max(1, len(self.ret)), topk),
                                  dtype=torch.uint8, device=device)
        if self.ret:
            self.kt = torch.empty(B, len(self.kv_used), N, R_INDEX, dtype=torch.bfloat16, device=device)
            self.qt = torch.empty(B, len(self.ret), N, R_INDEX, dtype=torch.bfloat16, device=device)
            self.blocks = torch.empty(B, len(self.ret), nb, topk, dtype=torch.int32, device=device)
            self.counts = torch.empty(B, len(self.ret), nb, dtype=torch.int32, device=device)

    def __call__(self, q, k, v, P, o, stream=None, index_out: Optional[torch.Tensor] = None):
        """q/o [B,N,Hq,D], k/v [B,N,Hkv,D], P [Hkv,D,r].

        ``index_out`` (optional, bf16 [B, Hkv, cap, r] with cap >= N) is the
        decode key index of the cache this prefill fills: the layer then
        projects the keys of every KV head into its rows 0..N-1
        (``index_append``) and the block selection reads them from there, so
        decode steps continue on the same index (appending one row per new
        token) without a second projection."""
        if index_out is not None:
            index_append(k, P, index_out, 0, stream=stream)
        if self.ret:
            if index_out is None:
                index_project(k, P, self.kv_used, self.kv_used, out=self.kt, stream=stream)
                kt, kv = self.kt, self.kv_slot
            else:
                kt, kv = index_out, self.kv_ret
            index_project(q, P, self.ret, self.kv_ret, out=self.qt, stream=stream)
            select_prefill(self.qt, kt, kv, self.topk, self.blocks, self.counts,
                           ws=self.ws_sel, stream=stream)
            sparse_attn_prefill(q, k, v, o, self.ret, self.blocks, self.counts, self.window_blocks,
                                self.sink_blocks, self.scale, ws=self.ws_sparse, stream=stream)
        if self.swa_heads:
            swa(q, k, v, o, self.swa_heads, self.window, 0, self.scale, ws=self.ws_swa, stream=stream)
        return o

    def graph(self, q, k, v, P, o, index_out: Optional[torch.Tensor] = None) -> "torch.cuda.CUDAGraph":
        """Captures the layer on these buffers into a CUDA graph.

        ``graph.replay()`` then runs every kernel of the layer with one launch
        from the host (for short sequences the per-call launches dominate),
        reading ``q``, ``k``, ``v``, ``P`` as they are at replay and writing
        ``o``. Run the layer once eagerly before capturing, so that every
        kernel attribute is set."""
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            self(q, k, v, P, o, index_out=index_out)
        return g

    def device_status(self, stream=None) -> int:
        """Synchronises and returns the worst status word of the attention calls."""
        return max(workspace_status(self.ws_sparse, stream), workspace_status(self.ws_swa, stream),
                   workspace_status(self.ws_sel, stream))


class OrthrosStep:
    """The two working modes of one Orthros attention on the existing calls
    (Orthros article, section on one attention with two working modes): every
    token runs sliding-window attention, and only the position that predicts
    the next token also runs a full cross-attention over the whole cache.

    ``prefill(q, k, v, o, o_ca)``: SWA over every prompt row (all heads, one
    rtp_swa call) and the full cross-attention of the last prompt row
    (``o_ca`` [B, Hq, D]: the decode form of rtp_swa at position N-1 with a
    window as long as the prompt). ``decode(q, kc, vc, o, o_ca, L)``: for the
    new token at position L-1, its SWA row into ``o`` [B, Hq, D] and its full
    cross-attention over the L cached tokens into ``o_ca``. The trained
    Scale-Offset that tells the two queries apart is out of scope: both use
    the same query."""

    def __init__(self, B, L, Hq, Hkv, window, device, scale=None):
        self.B, self.L, self.Hq, self.Hkv, self.window = B, L, Hq, Hkv, window
        self.heads = list(range(Hq))
        self.scale = 1.0 / math.sqrt(D_HEAD) if scale is None else scale
        self.ws_swa = torch.zeros(lib().rtp_workspace_size_swa(B, 1, L, Hq, window), dtype=torch.uint8, device=device)
        self.ws_ca = torch.zeros(lib().rtp_workspace_size_swa(B, 1, L, Hq, L), dtype=torch.uint8, device=device)
        self.ws_pre = torch.zeros(256, dtype=torch.uint8, device=device)

    def prefill(self, q, k, v, o, o_ca, stream=None):
        N = q.shape[1]
        swa(q, k, v, o, self.heads, self.window, 0, self.scale, ws=self.ws_pre, stream=stream)
        swa(q[:, N - 1:N], k, v, o_ca.unsqueeze(1), self.heads, N, N - 1, self.scale, ws=self.ws_ca, stream=stream)
        return o, o_ca

    def decode(self, q, kc, vc, o, o_ca, L: Optional[int] = None, stream=None):
        L = kc.shape[1] if L is None else L
        assert L <= self.L
        kv, vv = kc[:, :L], vc[:, :L]
        swa(q.unsqueeze(1), kv, vv, o.unsqueeze(1), self.heads, self.window, L - 1, self.scale, ws=self.ws_swa,
            stream=stream)
        swa(q.unsqueeze(1), kv, vv, o_ca.unsqueeze(1), self.heads, L, L - 1, self.scale, ws=self.ws_ca, stream=stream)
        return o, o_ca


class DecodeStep:
    """One decode step over a cache with a precomputed key index: query
    projection, token selection, sparse attention on retrieval heads and SWA
    on streaming heads."""

    def __init__(self, B, L, Hq, Hkv, ret_heads, window, ret_window, topk, device, sink=1,
                 scale=None):
        """``L`` is the longest cache the step will see (its workspace is sized
        for it); each call may pass a shorter current length."""
        self.B, self.L, self.Hq, self.Hkv = B, L, Hq, Hkv
        self.ret = list(ret_heads)
        self.swa_heads = [h for h in range(Hq) if h not in set(self.ret)]
        self.window, self.ret_window, self.topk, self.sink = window, ret_window, topk, sink
        self.scale = 1.0 / math.sqrt(D_HEAD) if scale is None else scale
        self.kv_ret = [kv_of(h, Hq, Hkv) for h in self.ret]
        self.idx = torch.empty(B, len(self.ret), topk, dtype=torch.int32, device=device) if self.ret else None
        wmax = max(ret_window if self.ret else 0, window if self.swa_heads else 0)
        self.ws = torch.empty(lib().rtp_workspace_size_decode_step(B, L, Hq, len(self.ret), topk, wmax),
                              dtype=torch.uint8, device=device)

    def __call__(self, q, kc, vc, kindex, P, o, stream=None, L: Optional[int] = None, kindex8=None, kscale=None):
        """q/o [B,Hq,D]; kc/vc [B,cap,Hkv,D]; kindex [B,Hkv,cap,r]; the cache
        holds L <= self.L tokens (default: kc's length). With ``kindex8`` /
        ``kscale`` (``index_quantize``) the selection scans the 8-bit index.
        One rtp_decode_step call."""
        L = kc.shape[1] if L is None else L
        assert L <= self.L, "the workspace is sized for at most L tokens"
        decode_step(q, P, kindex, kc, vc, o, self.ret, self.idx, self.ret_window, self.swa_heads, self.window,
                    self.topk, self.sink, self.scale, self.ws, stream=stream, L=L, kindex8=kindex8, kscale=kscale)
        return o

    def graph(self, q, kc, vc, kindex, P, o, kindex8=None, kscale=None) -> "torch.cuda.CUDAGraph":
        """Captures one step on these buffers into a CUDA graph.

        ``graph.replay()`` then runs the whole step (projection, selection,
        attention: every kernel, one launch from the host) reading the query
        currently in ``q`` and writing ``o``; write each new query into ``q``
        (and append to the cache in place) before replaying. Run the step once
        eagerly before capturing, so that every kernel attribute is set."""
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            self(q, kc, vc, kindex, P, o, kindex8=kindex8, kscale=kscale)
        return g


__all__ = ["lib", "RtpError", "index_project", "index_append", "index_quantize", "select_prefill", "select_decode",
           "select_decode_q8", "KeyClusters", "kcluster_build", "select_decode_clustered",
           "sparse_attn_prefill", "triangle_prefill", "sparse_attn_decode", "swa", "decode_attn_hybrid",
           "decode_step", "decode_step_clustered",
           "PrefillLayer", "DecodeStep", "OrthrosStep",
           "kv_of", "LIB_PATH"]
