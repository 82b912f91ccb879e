"""Seeded synthetic inputs for head-wise hybrid attention workloads.

This module only draws random tensors: it holds none of the attention,
indexer or selection arithmetic. Both the CPU oracle and the CUDA path read
the tensors it returns (one generation serves both sides: the tensors are
made once, on one device, and copied where the other side needs them).

Recipe (the clustered Gaussian generator of the workload descriptions):
  * ``C`` cluster centres, each ``3 * unit(N(0, I_D))``;
  * every Q row (per query head) and every K row (per KV head) is a uniformly
    drawn centre plus ``N(0, I_D)`` noise;
  * ``V ~ N(0, 1)``;
  * the projector ``P`` is one ``D x r`` matrix per KV head, entries
    ``N(0, 1/D)``;
  * every tensor is rounded to bf16 (round-to-nearest-even, torch's cast).

Planted structure:
  * decode needles: per (sequence, KV group) ``n_needles`` distinct cache
    positions whose key is ``bf16(4 * unit(q_h*))``, where ``h*`` is the
    lowest-numbered retrieval head of that group (the group's lowest head when
    every head retrieves);
  * prefill needle blocks: ``n_needle_blocks`` distinct key blocks drawn from
    ``[1, N/64)``; every key of such a block, on every KV head, is
    ``bf16(4 * unit(c))`` for one uniformly drawn centre ``c``.

Every draw comes from its own ``torch.Generator`` seeded from
``(seed, stream id)``, so the order in which tensors are made does not change
their values. CPU and CUDA generators give different streams; a tensor is
always made on one device and copied, never regenerated on the other.
"""
from __future__ import annotations

import dataclasses
from typing import Optional, Sequence

import torch

D_HEAD = 128
R_INDEX = 16
BLOCK = 64

# Stream ids: one independent generator per drawn tensor.
_S_CENTRES, _S_QASSIGN, _S_QNOISE, _S_KASSIGN, _S_KNOISE, _S_V, _S_P = range(7)
_S_NEEDLE_POS, _S_NEEDLE_BLK, _S_NEEDLE_CENTRE = 7, 8, 9


@dataclasses.dataclass(frozen=True)
class PrefillConfig:
    """One prefill layer workload."""
    name: str
    B: int
    N: int
    Hq: int
    Hkv: int
    ret_heads: tuple
    window: int            # SWA window of streaming heads (tokens)
    ret_window: int        # local window of retrieval heads (tokens, multiple of 64)
    topk: int              # selected key blocks per query block
    centres: int
    needle_blocks: int = 0
    seed: int = 0
    D: int = D_HEAD
    r: int = R_INDEX
    sink_blocks: int = 1


@dataclasses.dataclass(frozen=True)
class DecodeConfig:
    """One decode step over a pre-filled cache."""
    name: str
    B: int
    L: int
    Hq: int
    Hkv: int
    ret_heads: tuple
    window: int            # SWA window of streaming heads (tokens)
    ret_window: int        # local window of retrieval heads (tokens)
    topk: int              # selected tokens per retrieval head
    centres: int
    needles: int = 0
    seed: int = 0
    D: int = D_HEAD
    r: int = R_INDEX
    sink: int = 1


# The five seeded workloads (seed = 1000 + workload number).
TINY_PREFILL = PrefillConfig("prefill_2k_tiny", B=1, N=2048, Hq=8, Hkv=2, ret_heads=(0, 4),
                             window=256, ret_window=256, topk=8, centres=64, seed=1001)
PREFILL_32K = PrefillConfig("prefill_32k", B=1, N=32768, Hq=32, Hkv=4,
                            ret_heads=(0, 7, 13, 19, 26), window=8192, ret_window=8192,
                            topk=64, centres=512, seed=1002)
DECODE_128K = DecodeConfig("decode_128k_b8", B=8, L=131072, Hq=32, Hkv=4,
                           ret_heads=(0, 7, 13, 19, 26), window=8192, ret_window=8192,
                           topk=2048, centres=512, needles=32, seed=1003)
PREFILL_1M = PrefillConfig("prefill_1m", B=1, N=1048576, Hq=32, Hkv=4,
                           ret_heads=(0, 7, 13, 19, 26), window=8192, ret_window=8192,
                           topk=256, centres=4096, needle_blocks=64, seed=1004)
PREFILL_128K_ALL = PrefillConfig("prefill_128k_all_sparse", B=1, N=131072, Hq=32, Hkv=4,
                                 ret_heads=tuple(range(32)), window=2048, ret_window=2048,
                                 topk=128, centres=1024, seed=1005)
DECODE_64K_ALL = DecodeConfig("decode_64k_b32_all_sparse", B=32, L=65536, Hq=32, Hkv=4,
                              ret_heads=tuple(range(32)), window=2048, ret_window=2048,
                              topk=2048, centres=1024, seed=1005)

ALL_CONFIGS = {c.name: c for c in (TINY_PREFILL, PREFILL_32K, DECODE_128K, PREFILL_1M,
                                   PREFILL_128K_ALL, DECODE_64K_ALL)}


def _gen(seed: int, stream: int, device) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed((int(seed) * 1_000_003 + 7919 * int(stream)) & ((1 << 62) - 1))
    return g


def _unit_rows(x: torch.Tensor) -> torch.Tensor:
    return x / x.norm(dim=-1, keepdim=True)


def make_centres(seed: int, n: int, D: int, device) -> torch.Tensor:
    """``n`` cluster centres, ``3 * unit(N(0, I_D))``, fp32 (not rounded)."""
    g = _gen(seed, _S_CENTRES, device)
    c = torch.randn(n, D, generator=g, device=device, dtype=torch.float32)
    return 3.0 * _unit_rows(c)


def clustered_rows(seed: int, stream_assign: int, stream_noise: int, n_rows: int,
                   centres: torch.Tensor, out: torch.Tensor, chunk: int = 1 << 22) -> None:
    """Fill ``out`` (bf16, ``[n_rows, D]`` view) with centre + N(0, I) rows.

    Drawn in chunks of ``chunk`` rows so the fp32 temporaries stay small;
    every chunk uses the same two generators, continuing their streams.
    """
    device = out.device
    ga = _gen(seed, stream_assign, device)
    gn = _gen(seed, stream_noise, device)
    D = centres.shape[1]
    for r0 in range(0, n_rows, chunk):
        r1 = min(n_rows, r0 + chunk)
        a = torch.randint(0, centres.shape[0], (r1 - r0,), generator=ga, device=device)
        x = torch.randn(r1 - r0, D, generator=gn, device=device, dtype=torch.float32)
        x += centres[a]
        out[r0:r1].copy_(x)


def normal_bf16(seed: int, stream: int, shape: Sequence[int], std: float, device,
                chunk: int = 1 << 28) -> torch.Tensor:
    g = _gen(seed, stream, device)
    out = torch.empty(*shape, dtype=torch.bfloat16, device=device)
    flat = out.view(-1)
    for e0 in range(0, flat.numel(), chunk):
        e1 = min(flat.numel(), e0 + chunk)
        x = torch.randn(e1 - e0, generator=g, device=device, dtype=torch.float32)
        if std != 1.0:
            x *= std
        flat[e0:e1].copy_(x)
    return out


def kv_of_head(h: int, Hq: int, Hkv: int) -> int:
    """Contiguous GQA grouping: query head h reads KV head floor(h / (Hq/Hkv))."""
    return h // (Hq // Hkv)


def make_prefill(cfg: PrefillConfig, device="cpu", seed: Optional[int] = None,
                 N: Optional[int] = None) -> dict:
    """Q [B,N,Hq,D], K/V [B,N,Hkv,D], P [Hkv,D,r] (all bf16) for a prefill workload.

    ``N`` overrides the sequence length (same recipe at another size).
    """
    seed = cfg.seed if seed is None else seed
    N = cfg.N if N is None else N
    B, Hq, Hkv, D, r = cfg.B, cfg.Hq, cfg.Hkv, cfg.D, cfg.r
    centres = make_centres(seed, cfg.centres, D, device)
    q = torch.empty(B, N, Hq, D, dtype=torch.bfloat16, device=device)
    k = torch.empty(B, N, Hkv, D, dtype=torch.bfloat16, device=device)
    clustered_rows(seed, _S_QASSIGN, _S_QNOISE, B * N * Hq, centres, q.view(-1, D))
    clustered_rows(seed, _S_KASSIGN, _S_KNOISE, B * N * Hkv, centres, k.view(-1, D))
    v = normal_bf16(seed, _S_V, (B, N, Hkv, D), 1.0, device)
    P = normal_bf16(seed, _S_P, (Hkv, D, r), 1.0 / D ** 0.5, device)
    needle_blocks = None
    nb_total = N // BLOCK
    if cfg.needle_blocks and nb_total > 1:
        n_nb = min(cfg.needle_blocks, nb_total - 1)
        g = _gen(seed, _S_NEEDLE_BLK, "cpu")
        needle_blocks = (torch.randperm(nb_total - 1, generator=g)[:n_nb] + 1).sort().values
        gc = _gen(seed, _S_NEEDLE_CENTRE, "cpu")
        which = torch.randint(0, cfg.centres, (n_nb,), generator=gc)
        dirs = 4.0 * _unit_rows(centres[which.to(device)].float())
        for b in range(B):
            for i, blk in enumerate(needle_blocks.tolist()):
                k[b, blk * BLOCK:(blk + 1) * BLOCK, :, :] = dirs[i].to(torch.bfloat16)
    return dict(q=q, k=k, v=v, P=P, needle_blocks=needle_blocks, N=N, seed=seed)


def make_decode(cfg: DecodeConfig, device="cpu", seed: Optional[int] = None,
                L: Optional[int] = None, B: Optional[int] = None) -> dict:
    """q [B,Hq,D], K/V cache [B,L,Hkv,D], P [Hkv,D,r] (bf16) for a decode step.

    The cache holds ``L`` tokens; the new token's own K/V row is the last one
    (position ``L-1``). ``L`` and ``B`` override the workload's sizes.
    """
    seed = cfg.seed if seed is None else seed
    L = cfg.L if L is None else L
    B = cfg.B if B is None else B
    Hq, Hkv, D, r = cfg.Hq, cfg.Hkv, cfg.D, cfg.r
    centres = make_centres(seed, cfg.centres, D, device)
    q = torch.empty(B, Hq, D, dtype=torch.bfloat16, device=device)
    kc = torch.empty(B, L, Hkv, D, dtype=torch.bfloat16, device=device)
    clustered_rows(seed, _S_QASSIGN, _S_QNOISE, B * Hq, centres, q.view(-1, D))
    clustered_rows(seed, _S_KASSIGN, _S_KNOISE, B * L * Hkv, centres, kc.view(-1, D))
    vc = normal_bf16(seed, _S_V, (B, L, Hkv, D), 1.0, device)
    P = normal_bf16(seed, _S_P, (Hkv, D, r), 1.0 / D ** 0.5, device)
    needle_pos = None
    if cfg.needles:
        G = Hq // Hkv
        n = min(cfg.needles, L)
        g = _gen(seed, _S_NEEDLE_POS, "cpu")
        needle_pos = torch.empty(B, Hkv, n, dtype=torch.int64)
        for b in range(B):
            for grp in range(Hkv):
                in_group = [h for h in cfg.ret_heads if kv_of_head(h, Hq, Hkv) == grp]
                h_star = min(in_group) if in_group else grp * G
                pos = torch.randperm(L, generator=g)[:n].sort().values
                needle_pos[b, grp] = pos
                d = 4.0 * _unit_rows(q[b, h_star].float().unsqueeze(0))[0]
                kc[b, pos.to(device), grp, :] = d.to(torch.bfloat16)
    return dict(q=q, kc=kc, vc=vc, P=P, needle_pos=needle_pos, L=L, B=B, seed=seed)


def flush_buffer(device, nbytes: int = 256 << 20) -> torch.Tensor:
    """A buffer larger than the 126 MB L2, written between timed steps."""
    return torch.empty(nbytes // 4, dtype=torch.float32, device=device)
