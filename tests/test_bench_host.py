"""Host-side logic of bench.py: the algorithmic work counts (checked against
the oracle's own attended sets) and the multi-rank timing reduction (gloo,
world size 2, on CPU)."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

import bench
import oracle as O


def test_swa_pairs_brute():
    for N, W in [(10, 3), (10, 10), (10, 50), (1000, 64), (4096, 4096)]:
        want = sum(min(t + 1, W) for t in range(N))
        assert bench.swa_pairs(N, W) == want


def test_causal_pairs_brute():
    for N in (64, 128, 640):
        assert bench.causal_pairs(N) == N * (N + 1) // 2


def test_sparse_pairs_matches_oracle_sets():
    rs = np.random.default_rng(0)
    nb, k, wb, sink = 40, 6, 5, 1
    blocks = -np.ones((1, 2, nb, k), np.int32)
    counts = np.zeros((1, 2, nb), np.int32)
    want = 0
    for j in range(2):
        for i in range(nb):
            n = min(k, i + 1)
            sel = np.sort(rs.choice(i + 1, n, replace=False))
            blocks[0, j, i, :n] = sel
            counts[0, j, i] = n
            att = O.attended_blocks(sel, i, wb, sink)
            want += sum(64 * 64 if jb < i else 64 * 65 // 2 for jb in att)
    got = bench.sparse_pairs(torch.from_numpy(blocks), torch.from_numpy(counts), wb, sink)
    assert got == want


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    import torch.distributed as dist
    dist.init_process_group("gloo", rank=rank, world_size=world)
    v = bench.max_over_ranks(float(10 + rank * 5), world)
    bench.barrier(world)
    out[rank] = v
    dist.destroy_process_group()


def test_max_over_ranks_gloo_world2():
    ctx = mp.get_context("spawn")
    mgr = ctx.Manager()
    out = mgr.dict()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, out)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    assert out[0] == 15.0 and out[1] == 15.0


def test_traffic_is_reported_only_for_the_captured_sources(monkeypatch):
    files = ["select.cu", "rtp_common.cuh"]
    digest = bench._sources_digest(files)
    monkeypatch.setattr(bench, "NCU_TRAFFIC", {
        "k_current": {"bytes_per_unit": 2.5, "sources": files, "digest": digest},
        "k_stale": {"bytes_per_unit": 2.5, "sources": files, "digest": "0" * 16},
    })
    assert bench.traffic_for("k_current", 1000) == 2500
    assert bench.traffic_for("k_stale", 1000) is None
    assert bench.traffic_for("k_missing", 1000) is None


def test_triangle_pairs_match_oracle_key_sets():
    for N, sink, wb, last in [(1024, 1, 2, 256), (640, 0, 3, 0), (512, 2, 1, 512), (1536, 1, 4, 320), (960, 3, 2, 64)]:
        want = sum(len(O.triangle_keys(t, N, sink, wb, last)) for t in range(N))
        assert bench.triangle_pairs(N, sink, wb, last) == want, (N, sink, wb, last)


def test_decode_bytes_counts_every_row_the_step_needs_once():
    """The decode roofline's bytes: per (sequence, KV group) every row the
    attention needs (the window of every KV group, and for the groups of
    retrieval heads the sink and the selected rows outside the window, each
    row once however many heads select it), plus the key index of the
    retrieval groups and q / o; checked against explicit sets built from the
    oracle's attended sets."""
    from types import SimpleNamespace
    cfg = SimpleNamespace(Hq=8, Hkv=4, ret_heads=[0, 1, 5], window=40, ret_window=40, sink=1)
    B, L, k = 3, 300, 25
    rs = np.random.default_rng(3)
    idx = torch.full((B, len(cfg.ret_heads), k), -1, dtype=torch.int32)
    for b in range(B):
        for j in range(len(cfg.ret_heads)):
            sel = np.sort(rs.choice(L, size=k - 3, replace=False))
            idx[b, j, :len(sel)] = torch.from_numpy(sel.astype(np.int32))
    got = bench.decode_bytes(cfg, idx, L, B)
    G = cfg.Hq // cfg.Hkv
    rows = 0
    for b in range(B):
        for g in range(cfg.Hkv):
            need = set(range(L - cfg.window, L))
            for j, h in enumerate(cfg.ret_heads):
                if h // G == g:
                    sel = idx[b, j].numpy()
                    need |= set(O.decode_attended(sel[sel >= 0], L, cfg.ret_window, cfg.sink).tolist())
            rows += len(need)
    kv_ret = {h // G for h in cfg.ret_heads}
    want_scan = B * len(kv_ret) * L * 16 * 2
    assert got["scan"] == want_scan
    assert got["window"] + got["gathered"] == rows * 128 * 2 * 2
    assert got["qo"] == B * cfg.Hq * 128 * 2 * 2
    assert got["total"] == want_scan + rows * 128 * 2 * 2 + got["qo"]
