"""Benchmark: head-wise hybrid attention, one layer, on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

A step is one pass of the whole hot path: one prefill layer over the 1M-token
workload (index projection, block selection, sparse attention on the
retrieval heads, SWA on the streaming heads) followed by one decode step over
the 128K-token, batch-8 cache (query projection, token selection, sparse
attention on the retrieval heads, SWA on the streaming heads). Prints one
JSON line on rank 0: ``value`` is prefill tokens/s per layer (whole job),
``decode`` carries the decode tokens/s per layer.

Inputs are synthetic (the seeded clustered Gaussian recipe of ``synth``),
resident in HBM before timing; they exceed the 126 MB L2 (Q/K/V 10 GiB for
prefill, 2.1 GiB of cache for decode) and L2 is flushed between decode steps.
Times are CUDA events on the launching stream, max over ranks.

With ``--gpus N`` every rank runs its own independent layer (weak scaling, no
data-path collective); torch.distributed only carries the barrier and the
max-over-ranks of the times.
"""
from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import torch  # noqa: E402

import synth  # noqa: E402

PEAK_FALLBACK = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
BLOCK, D, R = 64, 128, 16


# ---------------------------------------------------------------------------
# Peaks, clocks, ranks
# ---------------------------------------------------------------------------
def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            p = json.load(f)
        return {"hbm_gbs": float(p["hbm_gbs"]), "bf16_tflops": float(p["bf16_tflops"]),
                "bf16_tflops_sustained": float(p.get("bf16_tflops_sustained", p["bf16_tflops"])),
                "source": "measured"}
    except (OSError, KeyError, ValueError):
        return dict(PEAK_FALLBACK, source="fallback")


class ClockSampler:
    """nvidia-smi sampling of SM clocks and throttle reasons while timing."""
    QUERY = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index: int):
        self.idx = device_index
        self.proc = None
        self.path = None

    def start(self):
        fd, self.path = tempfile.mkstemp(suffix=".csv")
        os.close(fd)
        try:
            self.proc = subprocess.Popen(["nvidia-smi", f"--id={self.idx}", f"--query-gpu={self.QUERY}",
                                          "--format=csv,noheader,nounits", "-lms", "200"],
                                         stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except OSError:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        sm, smax, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        with open(self.path) as f:
            for line in f:
                parts = [x.strip() for x in line.split(",")]
                if len(parts) < 9:
                    continue
                try:
                    sm.append(float(parts[1]))
                    smax.append(float(parts[2]))
                except ValueError:
                    continue
                for n, val in zip(names, parts[5:9]):
                    if val.lower() == "active":
                        reasons.add(n)
        os.unlink(self.path)
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": max(smax) if smax else None,
                "reasons": sorted(reasons), "samples": len(sm)}


def dist_setup(n_gpus):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        import torch.distributed as dist
        backend = "nccl" if torch.cuda.is_available() else "gloo"
        if torch.cuda.is_available():
            torch.cuda.set_device(local)
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=600))
    elif torch.cuda.is_available():
        torch.cuda.set_device(0)
    return rank, world, local


def max_over_ranks(x: float, world: int) -> float:
    if world == 1:
        return x
    import torch.distributed as dist
    dev = torch.device("cuda", torch.cuda.current_device()) if torch.cuda.is_available() else "cpu"
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


# ---------------------------------------------------------------------------
# Algorithmic work (what the path must do, independent of how it is done)
# ---------------------------------------------------------------------------
def swa_pairs(N: int, W: int) -> int:
    """Causal (query, key) pairs of one streaming head: sum_t min(t+1, W)."""
    if N <= W:
        return N * (N + 1) // 2
    return W * (W + 1) // 2 + (N - W) * W


def sparse_pairs(blocks: torch.Tensor, counts: torch.Tensor, window_blocks: int, sink_blocks: int) -> int:
    """Attended causal pairs of the retrieval heads, counted from the actual
    selected lists: |selected U sink U window| blocks per query block, the
    diagonal block holding 64*65/2 causal pairs and every other one 64*64."""
    B, Hr, nb, k = blocks.shape
    i = torch.arange(nb, device=blocks.device).view(1, 1, nb, 1)
    lo = (i - window_blocks + 1).clamp(min=0)
    valid = (torch.arange(k, device=blocks.device).view(1, 1, 1, k) < counts.unsqueeze(-1))
    sel_out = valid & (blocks >= sink_blocks) & (blocks < lo) & (blocks >= 0)
    n_sel = sel_out.sum(-1)                                         # [B,Hr,nb]
    iv = torch.arange(nb, device=blocks.device).view(1, 1, nb)
    n_win = torch.minimum(iv + 1, torch.tensor(window_blocks, device=blocks.device))
    n_sink = (iv - window_blocks + 1).clamp(min=0).clamp(max=sink_blocks)
    n_att = n_sel + n_win + n_sink
    pairs = (n_att - 1) * BLOCK * BLOCK + BLOCK * (BLOCK + 1) // 2
    return int(pairs.sum().item())


def causal_pairs(N: int) -> int:
    """All causal (query, key) pairs of one head (the indexer scores each once)."""
    nb = N // BLOCK
    return BLOCK * BLOCK * nb * (nb - 1) // 2 + BLOCK * (BLOCK + 1) // 2 * nb


def triangle_pairs(N: int, sink_blocks: int, window_blocks: int, last: int) -> int:
    """Attended causal pairs of one head under the triangle-shaped mask:
    streaming-region query block i attends its band blocks (min(i+1, wb)) and
    the sink blocks outside the band, the diagonal block holding 64*65/2
    causal pairs; a row t of the last region attends every key u <= t."""
    n_stream = N - last
    nb = n_stream // BLOCK
    blocks = sum(min(i + 1, window_blocks) + max(0, min(sink_blocks, i + 1 - window_blocks)) for i in range(nb))
    pairs = (blocks - nb) * BLOCK * BLOCK + nb * BLOCK * (BLOCK + 1) // 2
    return pairs + sum(n_stream + t + 1 for t in range(last))


def decode_bytes(cfg, idx: torch.Tensor, L: int, B: int) -> dict:
    """HBM bytes a decode step must move: the key index of every KV head that
    serves a retrieval head (32 B/token), the window K/V of every KV group once
    (512 B/token), the out-of-window selected K/V rows deduplicated per KV
    group (512 B/token), q and o."""
    G = cfg.Hq // cfg.Hkv
    ret = list(cfg.ret_heads)
    kv_ret = sorted(set(h // G for h in ret))
    W = max(cfg.window, cfg.ret_window)
    scan = B * len(kv_ret) * L * R * 2
    window = B * cfg.Hkv * min(W, L) * D * 2 * 2
    gathered_tokens = 0
    lo = max(0, L - cfg.ret_window)
    for b in range(B):
        for g in kv_ret:
            rows = [j for j, h in enumerate(ret) if h // G == g]
            x = idx[b, rows].reshape(-1)
            x = x[(x >= cfg.sink) & (x < lo)]
            n = torch.unique(x).numel() + min(cfg.sink, lo)
            gathered_tokens += n
    gathered = gathered_tokens * D * 2 * 2
    qo = B * cfg.Hq * D * 2 * 2
    return {"scan": scan, "window": window, "gathered": gathered, "qo": qo,
            "total": scan + window + gathered + qo}


# ---------------------------------------------------------------------------
# GPU arm
# ---------------------------------------------------------------------------
# Nominal dense peaks of one B200 (context beside the measured ones)
NOMINAL_BF16_TFLOPS = 2250.0
NOMINAL_HBM_GBS = 7700.0

# DRAM traffic (dram__bytes_read.sum + dram__bytes_write.sum) per unit of
# work, from one ncu capture of each kernel on a small case of the same
# kernel (profiles/ names the command), scaled here by the units one launch of
# the benchmark processes. Each entry records a digest of the sources the
# kernel is built from: when they have changed since the capture, the entry
# is stale and the line reports null.
NCU_TRAFFIC = {
    # one decode step of the 128K x 8 workload at full size (zero + projection,
    # scan, filter, attention, merge): profiles/decode_128k_b8.md
    "decode_step": {"bytes_per_unit": 338815232 / (8 * 131072), "unit": "cached token",
                    "sources": ["select.cu", "decode_attn.cu", "rtp_common.cuh", "rtp_internal.h", "api.cu"],
                    "digest": "9501a8709f25eabd"},
}


def _sources_digest(files):
    import hashlib
    h = hashlib.sha256()
    for f in files:
        with open(os.path.join(ROOT, "long_context_hybrid_b200", "csrc", f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:16]


def traffic_for(name, units):
    """DRAM bytes of one launch of kernel ``name`` processing ``units`` units
    of work, or None when no capture of the current sources exists."""
    e = NCU_TRAFFIC.get(name)
    if e is None:
        return None
    try:
        if _sources_digest(e["sources"]) != e["digest"]:
            return None
    except OSError:
        return None
    return int(e["bytes_per_unit"] * units)


def run_ours(args, rank, world):
    import long_context_hybrid_b200 as rtp
    from long_context_hybrid_b200 import build as _build
    if rank == 0:
        _build.build()
    barrier(world)
    rtp.lib()
    dev = torch.device("cuda", torch.cuda.current_device())
    stream = torch.cuda.current_stream()
    peaks = load_peaks()
    pcfg = synth.ALL_CONFIGS[args.prefill]
    dcfg = synth.ALL_CONFIGS[args.decode]

    # ---- prefill data and layer
    pd = synth.make_prefill(pcfg, device=dev, seed=pcfg.seed + 7919 * rank)
    q, k, v, P = pd["q"], pd["k"], pd["v"], pd["P"]
    N = pcfg.N
    layer = rtp.PrefillLayer(pcfg.B, N, pcfg.Hq, pcfg.Hkv, pcfg.ret_heads, pcfg.window,
                             pcfg.ret_window, pcfg.topk, dev)
    o = torch.empty(pcfg.B, N, pcfg.Hq, D, dtype=torch.bfloat16, device=dev)

    # ---- decode data and step
    dd = synth.make_decode(dcfg, device=dev, seed=dcfg.seed + 7919 * rank)
    qd, kc, vc, Pd = dd["q"], dd["kc"], dd["vc"], dd["P"]
    Bd, L = dcfg.B, dcfg.L
    kindex = rtp.index_project(kc, Pd, list(range(dcfg.Hkv)), list(range(dcfg.Hkv)))
    step = rtp.DecodeStep(Bd, L, dcfg.Hq, dcfg.Hkv, dcfg.ret_heads, dcfg.window, dcfg.ret_window,
                          dcfg.topk, dev, sink=dcfg.sink)
    od = torch.empty(Bd, dcfg.Hq, D, dtype=torch.bfloat16, device=dev)
    flush = synth.flush_buffer(dev)

    names_p = ["project_k", "project_q", "select_prefill", "sparse_attn_prefill", "swa_prefill"]
    names_d = ["project_q", "select_decode", "decode_attn_hybrid"]

    def prefill_step(ev):
        ev[0].record(stream)
        rtp.index_project(k, P, layer.kv_used, layer.kv_used, out=layer.kt)
        ev[1].record(stream)
        rtp.index_project(q, P, layer.ret, layer.kv_ret, out=layer.qt)
        ev[2].record(stream)
        rtp.select_prefill(layer.qt, layer.kt, layer.kv_slot, layer.topk, layer.blocks, layer.counts,
                           ws=layer.ws_sel)
        ev[3].record(stream)
        rtp.sparse_attn_prefill(q, k, v, o, layer.ret, layer.blocks, layer.counts, layer.window_blocks,
                                layer.sink_blocks, layer.scale, ws=layer.ws_sparse)
        ev[4].record(stream)
        if layer.swa_heads:
            rtp.swa(q, k, v, o, layer.swa_heads, layer.window, 0, layer.scale, ws=layer.ws_swa)
        ev[5].record(stream)

    # the decode step's three calls on their own (per-kernel breakdown only;
    # the step itself is one rtp_decode_step call, DecodeStep)
    b_qt = torch.empty(Bd, len(step.ret), R, dtype=torch.float32, device=dev)
    b_idx = torch.empty_like(step.idx)
    b_ws_sel = torch.empty(rtp.lib().rtp_workspace_size_select_decode(Bd, L, len(step.ret), step.topk),
                           dtype=torch.uint8, device=dev)
    b_ws_att = torch.empty(rtp.lib().rtp_workspace_size_decode_attn_hybrid(
        Bd, L, dcfg.Hq, step.topk, max(step.window, step.ret_window)), dtype=torch.uint8, device=dev)
    b_od = torch.empty_like(od)

    def decode_step(ev):
        ev[0].record(stream)
        step(qd, kc, vc, kindex, Pd, od)
        ev[1].record(stream)

    def new_events(n):
        return [torch.cuda.Event(enable_timing=True) for _ in range(n)]

    # ---- warm-up
    for _ in range(args.warmup):
        prefill_step(new_events(6))
        flush.zero_()
        decode_step(new_events(2))
    torch.cuda.synchronize()
    # The decode step runs as one CUDA graph (the way a serving loop replays
    # it): one host launch per step, every kernel of the step inside. Each
    # call is also captured on its own for the per-kernel breakdown.
    g_step = step.graph(qd, kc, vc, kindex, Pd, od)
    d_calls = [
        lambda: rtp.index_project(qd.unsqueeze(1), Pd, step.ret, step.kv_ret, out=b_qt.view(Bd, len(step.ret), 1, R)),
        lambda: rtp.select_decode(b_qt, kindex, step.kv_ret, step.topk, b_idx, b_ws_sel),
        lambda: rtp.decode_attn_hybrid(qd, kc, vc, b_od, step.ret, b_idx, step.ret_window, step.swa_heads,
                                       step.window, step.sink, step.scale, b_ws_att),
    ]
    for fn in d_calls:                      # once eagerly before capture
        fn()
    torch.cuda.synchronize()
    g_calls = []
    for fn in d_calls:
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            fn()
        g_calls.append(g)
    for _ in range(args.warmup):
        flush.zero_()
        g_step.replay()
        for g in g_calls:
            flush.zero_()
            g.replay()
    torch.cuda.synchronize()

    # ---- timed region
    clocks = ClockSampler(torch.cuda.current_device())
    if rank == 0:
        clocks.start()
    barrier(world)
    torch.cuda.synchronize()
    pev, dev_ev = [], []
    for _ in range(args.steps):
        e = new_events(6)
        prefill_step(e)
        pev.append(e)
        flush.zero_()                       # L2 flush between timed decode steps (not timed)
        e = new_events(2)
        e[0].record(stream)
        g_step.replay()
        e[1].record(stream)
        dev_ev.append(e)
        flush.zero_()
    torch.cuda.synchronize()
    barrier(world)
    clk = clocks.stop() if rank == 0 else None
    if layer.device_status() != 0:
        raise RuntimeError("a prefill kernel reported a timed-out wait")
    if rtp.workspace_status(step.ws) != 0:
        raise RuntimeError("the decode attention reported an error status")
    # per-call breakdown of the decode step (after the timed region)
    call_ev = []
    for _ in range(max(args.steps, 3)):
        row = []
        for g in g_calls:
            flush.zero_()
            e = new_events(2)
            e[0].record(stream)
            g.replay()
            e[1].record(stream)
            row.append(e)
        call_ev.append(row)
    torch.cuda.synchronize()

    def per_call(evs, names):
        tot = {n: 0.0 for n in names}
        for e in evs:
            for i, n in enumerate(names):
                tot[n] += e[i].elapsed_time(e[i + 1])
        return {n: t / len(evs) for n, t in tot.items()}

    p_ms = per_call(pev, names_p)
    d_ms = {n: sum(r[i][0].elapsed_time(r[i][1]) for r in call_ev) / len(call_ev) for i, n in enumerate(names_d)}
    p_step_ms = sum(p_ms.values())
    d_step_ms = sum(e[0].elapsed_time(e[1]) for e in dev_ev) / len(dev_ev)
    p_steps = [e[0].elapsed_time(e[5]) for e in pev]
    d_steps = [e[0].elapsed_time(e[1]) for e in dev_ev]
    step_stats = {"prefill_ms_median": round(statistics.median(p_steps), 3), "prefill_ms_min": round(min(p_steps), 3),
                  "decode_ms_median": round(statistics.median(d_steps), 4), "decode_ms_min": round(min(d_steps), 4)}
    p_step_ms = max_over_ranks(p_step_ms, world)
    d_step_ms = max_over_ranks(d_step_ms, world)

    # ---- algorithmic work
    G = pcfg.Hq // pcfg.Hkv
    n_swa = len(layer.swa_heads)
    sw_pairs = n_swa * pcfg.B * swa_pairs(N, pcfg.window)
    sp_pairs = sparse_pairs(layer.blocks, layer.counts, layer.window_blocks, layer.sink_blocks)
    sel_pairs = len(layer.ret) * pcfg.B * causal_pairs(N)
    # units: what the traffic of a launch scales with (attended pairs; rows)
    work = {
        "swa_prefill": {"flops": 4 * D * sw_pairs, "bound": "tensor", "units": sw_pairs},
        "sparse_attn_prefill": {"flops": 4 * D * sp_pairs, "bound": "tensor", "units": sp_pairs},
        "select_prefill": {"flops": 2 * R * sel_pairs, "bound": "tensor", "units": sel_pairs},
        "project_k": {"bytes": pcfg.B * N * len(layer.kv_used) * (D + R) * 2, "bound": "hbm",
                      "units": pcfg.B * N * len(layer.kv_used)},
        "project_q": {"bytes": pcfg.B * N * len(layer.ret) * (D + R) * 2, "bound": "hbm",
                      "units": pcfg.B * N * len(layer.ret)},
    }
    tflops_peak = peaks["bf16_tflops_sustained"]
    kernels = {}
    for n in names_p:
        w = work[n]
        t = max(p_ms[n] / 1e3, 1e-12)
        if "flops" in w:
            ach = w["flops"] / t / 1e12
            kernels[n] = {"ms": round(p_ms[n], 4), "achieved": round(ach, 2), "unit": "TFLOP/s",
                          "frac": round(ach / tflops_peak, 4)}
        else:
            ach = w["bytes"] / t / 1e9
            kernels[n] = {"ms": round(p_ms[n], 4), "achieved": round(ach, 1), "unit": "GB/s",
                          "frac": round(ach / peaks["hbm_gbs"], 4)}
    dom = max(names_p, key=lambda n: p_ms[n])
    dw = work[dom]
    if "flops" in dw:
        roofline = {"bound": "tensor", "kernel": dom, "achieved": kernels[dom]["achieved"],
                    "peak": tflops_peak, "unit": "TFLOP/s", "frac": kernels[dom]["frac"],
                    "traffic": traffic_for(dom, dw["units"]),
                    "peak_source": f"{peaks['source']} bf16 sustained",
                    "work_per_launch": dw["flops"]}
    else:
        roofline = {"bound": "hbm", "kernel": dom, "achieved": kernels[dom]["achieved"],
                    "peak": peaks["hbm_gbs"], "unit": "GB/s", "frac": kernels[dom]["frac"],
                    "traffic": traffic_for(dom, dw["units"]), "peak_source": f"{peaks['source']} copy",
                    "work_per_launch": dw["bytes"]}
    selected_flops = sum(work[n]["flops"] for n in ("swa_prefill", "sparse_attn_prefill", "select_prefill"))
    layer_frac = selected_flops / (p_step_ms / 1e3) / 1e12 / tflops_peak
    att_ms = p_ms["swa_prefill"] + p_ms["sparse_attn_prefill"]
    att_frac = (work["swa_prefill"]["flops"] + work["sparse_attn_prefill"]["flops"]) / max(att_ms / 1e3, 1e-12) \
        / 1e12 / tflops_peak

    db = decode_bytes(dcfg, step.idx, L, Bd)
    d_kern = {}
    for n in names_d:
        d_kern[n] = {"ms": round(d_ms[n], 4)}
    d_ach = db["total"] / (d_step_ms / 1e3) / 1e9
    d_kern["select_decode"].update({"achieved_gbs": round(db["scan"] / (d_ms["select_decode"] / 1e3) / 1e9, 1),
                                    "bytes": db["scan"]})
    att_bytes = db["window"] + db["gathered"] + db["qo"]
    d_kern["decode_attn_hybrid"].update({"achieved_gbs": round(att_bytes / (d_ms["decode_attn_hybrid"] / 1e3) / 1e9, 1),
                                         "bytes": att_bytes})

    total_tokens = pcfg.B * N * world
    value = total_tokens / (p_step_ms / 1e3)
    d_value = Bd * world / (d_step_ms / 1e3)
    launches_p = 5 if (layer.ret and layer.swa_heads) else 3
    launches = launches_p + 5   # decode: projection, scan, filter, attention, merge

    # ---- end to end through the API with host buffers (rank-local, fewer steps)
    e2e = None
    if args.e2e:
        e2e = run_e2e(args, pcfg, layer, q, k, v, P, o, qd, od, g_step, world, stream)

    # ---- the other workloads (one GPU only: they are reported, not scaled)
    others = run_other_configs(args, dev, peaks, stream) if (args.configs and world == 1) else None

    line = {
        "metric": "hybrid-attn prefill tok/s @1M & decode tok/s @128K per layer; % of roofline",
        "value": round(value, 1), "unit": "tok/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": round(p_step_ms, 3), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": {"workload": pcfg.name, "B": pcfg.B, "N": N, "Hq": pcfg.Hq, "Hkv": pcfg.Hkv,
                   "retrieval_heads": list(pcfg.ret_heads), "swa_window": pcfg.window,
                   "topk_blocks": pcfg.topk, "block": BLOCK, "D": D, "r": R,
                   "decode_workload": dcfg.name, "decode_B": Bd, "decode_L": L,
                   "decode_topk": dcfg.topk, "parallelism": f"independent layer per GPU x{world}",
                   "l2": "inputs larger than L2 (prefill Q/K/V 10 GiB); L2 flushed between decode steps"},
        "roofline": roofline,
        "roofline_nominal": {"peak_tflops": NOMINAL_BF16_TFLOPS, "peak_gbs": NOMINAL_HBM_GBS,
                             "frac": round(roofline["achieved"] / (NOMINAL_BF16_TFLOPS if roofline["unit"] == "TFLOP/s"
                                                                   else NOMINAL_HBM_GBS), 4)},
        "step_stats": step_stats,
        "layer_frac_of_tensor_peak": round(layer_frac, 4),
        "attention_frac_of_tensor_peak": round(att_frac, 4),
        "kernels_prefill": kernels,
        "decode": {"value": round(d_value, 1), "unit": "tok/s", "ms_per_step": round(d_step_ms, 4),
                   "roofline": {"bound": "hbm", "achieved": round(d_ach, 1), "peak": peaks["hbm_gbs"],
                                "unit": "GB/s", "frac": round(d_ach / peaks["hbm_gbs"], 4),
                                "frac_nominal": round(d_ach / NOMINAL_HBM_GBS, 4),
                                "traffic": traffic_for("decode_step", Bd * L), "bytes_per_step": db},
                   "kernels": d_kern},
        "other_configs": others,
        "gpu_launches": launches * args.steps,
        "clocks": clk,
        "e2e": e2e,
    }
    return line


def run_other_configs(args, dev, peaks, stream):
    """The other seeded workloads, each timed on its own (device-resident
    inputs, the layer or step replayed as one CUDA graph, L2 flushed before
    every timed step, CUDA events on the launching stream, median of the
    timed steps),
    with the roofline fraction of its own algorithmic work: prefill layers
    against the sustained bf16 peak (selected work: attended pairs x 4 D plus
    the indexer's 2 r per causal pair), decode steps against the HBM peak
    (bytes: key index scan, window K/V once per KV group, gathered rows once
    per KV group, q and o). The 128K decode also runs over the 8-bit key index
    (16 bytes per token in the scan instead of 32)."""
    import long_context_hybrid_b200 as rtp
    out = {}
    tflops = peaks["bf16_tflops_sustained"]
    flush = synth.flush_buffer(dev)
    for name in ("prefill_2k_tiny", "prefill_32k", "prefill_128k_all_sparse"):
        cfg = synth.ALL_CONFIGS[name]
        d = synth.make_prefill(cfg, device=dev)
        q, k, v, P = d["q"], d["k"], d["v"], d["P"]
        layer = rtp.PrefillLayer(cfg.B, cfg.N, cfg.Hq, cfg.Hkv, cfg.ret_heads, cfg.window, cfg.ret_window,
                                 cfg.topk, dev)
        o = torch.empty(cfg.B, cfg.N, cfg.Hq, D, dtype=torch.bfloat16, device=dev)
        layer(q, k, v, P, o)
        torch.cuda.synchronize()
        g = layer.graph(q, k, v, P, o)
        for _ in range(3):
            g.replay()
        times = []
        for _ in range(5):
            flush.zero_()                   # L2 flush between timed steps (not timed)
            s0, s1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            s0.record(stream)
            g.replay()
            s1.record(stream)
            torch.cuda.synchronize()
            times.append(s0.elapsed_time(s1))
        if layer.device_status() != 0:
            raise RuntimeError(f"{name}: a prefill kernel reported a timed-out wait")
        ms = statistics.median(times)
        flops = 4 * D * len(layer.swa_heads) * cfg.B * swa_pairs(cfg.N, cfg.window)
        if layer.ret:
            flops += 4 * D * sparse_pairs(layer.blocks, layer.counts, layer.window_blocks, layer.sink_blocks)
            flops += 2 * R * len(layer.ret) * cfg.B * causal_pairs(cfg.N)
        ach = flops / (ms / 1e3) / 1e12
        out[name] = {"value": round(cfg.B * cfg.N / (ms / 1e3), 1), "unit": "tok/s", "ms_per_step": round(ms, 4),
                     "roofline": {"bound": "tensor", "achieved": round(ach, 2), "peak": tflops, "unit": "TFLOP/s",
                                  "frac": round(ach / tflops, 4), "work": "selected work of the layer"}}
        del d, q, k, v, P, layer, o, g
    for name, bits in (("decode_64k_b32_all_sparse", 16), ("decode_128k_b8", 8)):
        cfg = synth.ALL_CONFIGS[name]
        d = synth.make_decode(cfg, device=dev)
        qd, kc, vc, P = d["q"], d["kc"], d["vc"], d["P"]
        kindex = rtp.index_project(kc, P, list(range(cfg.Hkv)), list(range(cfg.Hkv)))
        k8, ks = rtp.index_quantize(kindex, 0, cfg.L // 64) if bits == 8 else (None, None)
        step = rtp.DecodeStep(cfg.B, cfg.L, cfg.Hq, cfg.Hkv, cfg.ret_heads, cfg.window, cfg.ret_window, cfg.topk,
                              dev, sink=cfg.sink)
        od = torch.empty(cfg.B, cfg.Hq, D, dtype=torch.bfloat16, device=dev)
        step(qd, kc, vc, kindex, P, od, kindex8=k8, kscale=ks)
        torch.cuda.synchronize()
        g = step.graph(qd, kc, vc, kindex, P, od, kindex8=k8, kscale=ks)
        for _ in range(3):
            flush.zero_()
            g.replay()
        times = []
        for _ in range(10):
            flush.zero_()
            s0, s1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            s0.record(stream)
            g.replay()
            s1.record(stream)
            torch.cuda.synchronize()
            times.append(s0.elapsed_time(s1))
        ms = statistics.median(times)
        db = decode_bytes(cfg, step.idx, cfg.L, cfg.B)
        if bits == 8:       # codes of the full groups + their scales + the bf16 rows of a partial group
            n_full = cfg.L // 64 * 64
            n_kv = db["scan"] // (cfg.B * cfg.L * R * 2)
            scan8 = cfg.B * n_kv * (n_full * R + (n_full // 64) * 4 + (cfg.L - n_full) * R * 2)
            db["total"] += scan8 - db["scan"]
            db["scan"] = scan8
        ach = db["total"] / (ms / 1e3) / 1e9
        key = name if bits == 16 else name + "_8bit_index"
        out[key] = {"value": round(cfg.B / (ms / 1e3), 1), "unit": "tok/s", "ms_per_step": round(ms, 4),
                    "roofline": {"bound": "hbm", "achieved": round(ach, 1), "peak": peaks["hbm_gbs"], "unit": "GB/s",
                                 "frac": round(ach / peaks["hbm_gbs"], 4), "bytes_per_step": db}}
        del g, d, qd, kc, vc, P, kindex, k8, ks, step, od
    out.update(run_preset_configs(dev, peaks, stream, flush))
    torch.cuda.synchronize()
    return out


def _time_graph(fn, stream, flush, reps=10):
    """Median CUDA-event time (ms) of ``fn`` captured as one graph, L2 flushed
    before every replay."""
    fn()
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        fn()
    for _ in range(3):
        flush.zero_()
        g.replay()
    times = []
    for _ in range(reps):
        flush.zero_()
        s0, s1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        s0.record(stream)
        g.replay()
        s1.record(stream)
        torch.cuda.synchronize()
        times.append(s0.elapsed_time(s1))
    del g
    return statistics.median(times)


def run_preset_configs(dev, peaks, stream, flush):
    """The rows beyond the hot path, each on the workload shape it belongs to:
    the 128K decode over a clustered key index (one rtp_decode_step_clustered
    call: projection, two-level selection, attention), Orthros' decode (SWA plus a full cross-attention over the
    128K cache, every head), and the triangle-mask prefill on the 128K
    all-sparse shape (sink block, 2048-token band, last 2048 queries dense)."""
    import long_context_hybrid_b200 as rtp
    out = {}
    hbm = peaks["hbm_gbs"]
    tflops = peaks["bf16_tflops_sustained"]
    cfg = synth.DECODE_128K
    d = synth.make_decode(cfg, device=dev)
    qd, kc, vc, P = d["q"], d["kc"], d["vc"], d["P"]
    B, L, Hq, Hkv = cfg.B, cfg.L, cfg.Hq, cfg.Hkv
    kindex = rtp.index_project(kc, P, list(range(Hkv)), list(range(Hkv)))
    ret = list(cfg.ret_heads)
    kv_ret = [rtp.kv_of(h, Hq, Hkv) for h in ret]
    swa_heads = [h for h in range(Hq) if h not in ret]
    # clustered selection: clusters of 64 tokens, 64 probed per head
    cl = rtp.kcluster_build(kindex, L, 64, 2)
    n_probe = 64
    qt = torch.empty(B, len(ret), R, dtype=torch.float32, device=dev)
    idx = torch.empty(B, len(ret), cfg.topk, dtype=torch.int32, device=dev)
    od = torch.empty(B, Hq, D, dtype=torch.bfloat16, device=dev)
    ws_step = torch.empty(rtp.lib().rtp_workspace_size_decode_step_clustered(B, L, Hq, len(ret), cl.C, n_probe,
                                                                             cfg.topk, cfg.window),
                          dtype=torch.uint8, device=dev)
    rtp.index_project(qd.unsqueeze(1), P, ret, kv_ret, out=qt.view(B, len(ret), 1, R))   # for the byte count

    def clustered_step():
        rtp.decode_step_clustered(qd, P, kindex, cl, kc, vc, od, ret, idx, cfg.ret_window, swa_heads, cfg.window,
                                  cfg.topk, n_probe, sink=cfg.sink, ws=ws_step)
    ms = _time_graph(clustered_step, stream, flush)
    counts = torch.diff(cl.offsets.long(), dim=-1)                         # [B, Hkv, C]
    probed = 0
    for j, g in enumerate(kv_ret):
        top = torch.topk((cl.centroids[:, g] @ qt[:, j].unsqueeze(-1)).squeeze(-1), n_probe, dim=1).indices
        probed += int(torch.gather(counts[:, g], 1, top).sum())
    db = decode_bytes(cfg, idx, L, B)
    sel_bytes = B * len(kv_ret) * cl.C * R * 4 + probed * R * 2       # centroids + the probed rows of the index
    total = db["total"] - db["scan"] + sel_bytes
    ach = total / (ms / 1e3) / 1e9
    out["decode_128k_b8_clustered"] = {
        "value": round(B / (ms / 1e3), 1), "unit": "tok/s", "ms_per_step": round(ms, 4),
        "n_probe": n_probe, "cluster_size": 64,
        "roofline": {"bound": "hbm", "achieved": round(ach, 1), "peak": hbm, "unit": "GB/s", "frac": round(ach / hbm, 4),
                     "bytes_per_step": total}}
    # Orthros decode: SWA (window 8192) and a full cross-attention, every head
    orth = rtp.OrthrosStep(B, L, Hq, Hkv, cfg.window, dev)
    o_ca = torch.empty_like(od)
    ms = _time_graph(lambda: orth.decode(qd, kc, vc, od, o_ca, L=L), stream, flush)
    total = B * Hkv * (min(cfg.window, L) + L) * D * 2 * 2 + 3 * B * Hq * D * 2
    ach = total / (ms / 1e3) / 1e9
    out["decode_128k_b8_orthros"] = {
        "value": round(B / (ms / 1e3), 1), "unit": "tok/s", "ms_per_step": round(ms, 4),
        "roofline": {"bound": "hbm", "achieved": round(ach, 1), "peak": hbm, "unit": "GB/s", "frac": round(ach / hbm, 4),
                     "bytes_per_step": total}}
    del d, qd, kc, vc, P, kindex, cl, qt, idx, od, ws_step, orth, o_ca
    # triangle mask on the 128K all-sparse shape
    pc = synth.PREFILL_128K_ALL
    dp = synth.make_prefill(pc, device=dev)
    q, k, v = dp["q"], dp["k"], dp["v"]
    o = torch.empty(pc.B, pc.N, pc.Hq, D, dtype=torch.bfloat16, device=dev)
    heads = list(range(pc.Hq))
    sink, wb, last = 1, pc.ret_window // BLOCK, 2048
    ws = torch.zeros(256, dtype=torch.uint8, device=dev)
    rtp.triangle_prefill(q, k, v, o, heads, sink, wb, last, ws=ws)
    torch.cuda.synchronize()
    times = []
    for _ in range(5):
        s0, s1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        s0.record(stream)
        rtp.triangle_prefill(q, k, v, o, heads, sink, wb, last, ws=ws)
        s1.record(stream)
        torch.cuda.synchronize()
        times.append(s0.elapsed_time(s1))
    if rtp.workspace_status(ws) != 0:
        raise RuntimeError("triangle prefill reported a timed-out wait")
    ms = statistics.median(times)
    flops = 4 * D * triangle_pairs(pc.N, sink, wb, last) * len(heads) * pc.B
    ach = flops / (ms / 1e3) / 1e12
    out["prefill_128k_triangle"] = {
        "value": round(pc.B * pc.N / (ms / 1e3), 1), "unit": "tok/s", "ms_per_step": round(ms, 4),
        "sink_blocks": sink, "window_blocks": wb, "last_tokens": last,
        "roofline": {"bound": "tensor", "achieved": round(ach, 2), "peak": tflops, "unit": "TFLOP/s",
                     "frac": round(ach / tflops, 4), "work": "attended causal pairs x 4 D"}}
    del dp, q, k, v, o
    return out


def run_e2e(args, pcfg, layer, q, k, v, P, o, qd, od, g_step, world, stream):
    """Same metric through the public API with host buffers: every step copies
    its inputs from pinned host memory and reads the result back (prefill:
    pipelined over steps, double-buffered on the device)."""
    import long_context_hybrid_b200 as rtp
    hq = torch.empty(q.shape, dtype=q.dtype, pin_memory=True)
    hk = torch.empty(k.shape, dtype=k.dtype, pin_memory=True)
    hv = torch.empty(v.shape, dtype=v.dtype, pin_memory=True)
    hP = torch.empty(P.shape, dtype=P.dtype, pin_memory=True)
    ho = torch.empty(o.shape, dtype=o.dtype, pin_memory=True)
    hq.copy_(q); hk.copy_(k); hv.copy_(v); hP.copy_(P)
    hqd = torch.empty(qd.shape, dtype=qd.dtype, pin_memory=True)
    hod = torch.empty(od.shape, dtype=od.dtype, pin_memory=True)
    hqd.copy_(qd)
    torch.cuda.synchronize()

    def dstep():
        qd.copy_(hqd, non_blocking=True)
        g_step.replay()                     # DecodeStep.graph: the step captured on qd / od
        hod.copy_(od, non_blocking=True)

    # Prefill steps as a serving loop would run them: inputs and outputs
    # double-buffered on the device, each step's host-to-device copies on one
    # copy stream (issued two steps ahead, once the step that last used the
    # buffers is done with them), its kernels on the compute stream, and the
    # read-back of its output on a second copy stream, so that the copies of
    # neighbouring steps overlap the kernels (PCIe carries both directions at
    # once). Every step still copies all of its inputs in and its output out
    # inside the timed region.
    h2d_s, d2h_s = torch.cuda.Stream(), torch.cuda.Stream()
    ins = [(q, k, v, P), tuple(torch.empty_like(t) for t in (q, k, v, P))]
    outs = [o, torch.empty_like(o)]
    ev = lambda: torch.cuda.Event()
    in_ready, comp_done, out_free = [ev(), ev()], [ev(), ev()], [ev(), ev()]

    def h2d(i):
        h2d_s.wait_event(comp_done[i % 2])          # the step two back is done reading these inputs
        with torch.cuda.stream(h2d_s):
            for dst, src in zip(ins[i % 2], (hq, hk, hv, hP)):
                dst.copy_(src, non_blocking=True)
        in_ready[i % 2].record(h2d_s)

    def compute(i):
        stream.wait_event(in_ready[i % 2])
        stream.wait_event(out_free[i % 2])          # the step two back has read its output out
        layer(*ins[i % 2], outs[i % 2], stream=stream)
        comp_done[i % 2].record(stream)

    def d2h(i):
        d2h_s.wait_event(comp_done[i % 2])
        with torch.cuda.stream(d2h_s):
            ho.copy_(outs[i % 2], non_blocking=True)
        out_free[i % 2].record(d2h_s)

    def prefill_steps(n):
        h2d(0)
        if n > 1:
            h2d(1)
        for i in range(n):
            compute(i)
            d2h(i)
            if i + 2 < n:
                h2d(i + 2)
        stream.wait_stream(h2d_s)
        stream.wait_stream(d2h_s)

    # the first step's input copy and the last step's read-back overlap no
    # kernel: eight or more steps, so that the loop's steady state dominates
    steps = max(8, min(args.steps, 12))
    prefill_steps(2); dstep()
    torch.cuda.synchronize()
    barrier(world)
    s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    s.record(stream)
    h2d_s.wait_stream(stream)
    d2h_s.wait_stream(stream)
    prefill_steps(steps)
    e.record(stream)
    torch.cuda.synchronize()
    p_ms = max_over_ranks(s.elapsed_time(e) / steps, world)
    dsteps = 20
    s.record(stream)
    for _ in range(dsteps):
        dstep()
    e.record(stream)
    torch.cuda.synchronize()
    d_ms = max_over_ranks(s.elapsed_time(e) / dsteps, world)
    h2d = sum(t.numel() * t.element_size() for t in (hq, hk, hv, hP))
    d2h = ho.numel() * ho.element_size()
    return {"value": round(pcfg.B * pcfg.N * world / (p_ms / 1e3), 1), "unit": "tok/s",
            "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "ms_per_step": round(p_ms, 3),
            "steps": steps,
            "note": "steps pipelined: each step's copies in and out overlap the neighbouring steps' kernels",
            "decode": {"value": round(qd.shape[0] * world / (d_ms / 1e3), 1), "unit": "tok/s",
                       "h2d_bytes_per_step": hqd.numel() * 2, "d2h_bytes_per_step": hod.numel() * 2,
                       "ms_per_step": round(d_ms, 4),
                       "note": "KV cache and key index stay resident; each step copies the new query in and the output out"}}


# ---------------------------------------------------------------------------
# CPU oracle (baseline and reference arm)
# ---------------------------------------------------------------------------
def oracle_prefill_rate(pcfg, q, k, v, P, budget_s: float = 20.0, seed: int = 0):
    """Oracle prefill throughput, extrapolated from a bounded sample.

    Times the index projection of the whole sequence (the keys of every KV
    head serving a retrieval head, the queries of every retrieval head) once,
    then a full layer (all heads) on the first, last and window-boundary query
    blocks and on seeded uniformly drawn blocks until ``budget_s`` seconds of
    block work have run (at least four drawn blocks). The rate is
    tokens / (t_projection + (N/64) * mean time of a drawn block): the drawn
    blocks are a uniform sample of the per-block cost, which grows with the
    block's position; the fixed blocks are reported beside it."""
    import numpy as np
    import oracle as O
    N = q.shape[0]
    nb = N // BLOCK
    G = pcfg.Hq // pcfg.Hkv
    t0 = time.perf_counter()
    kt = {g: O.project(k[:, g, :], P[g]) for g in sorted(set(h // G for h in pcfg.ret_heads))}
    qt = {h: O.project(q[:, h, :], P[h // G]) for h in pcfg.ret_heads}
    t_proj = time.perf_counter() - t0
    index = {"kt": kt, "qt": qt}

    def block_time(i):
        t = time.perf_counter()
        O.prefill_layer(q, k, v, P, pcfg.ret_heads, pcfg.window, pcfg.ret_window, pcfg.topk,
                        1 / math.sqrt(D), qblocks=[i], index=index)
        return time.perf_counter() - t

    wb = pcfg.ret_window // BLOCK
    fixed = sorted({0, min(nb - 1, wb - 1), min(nb - 1, wb), nb - 1})
    fixed_t = {i: round(block_time(i), 3) for i in fixed}
    rs = np.random.default_rng(seed)
    drawn, spent = [], 0.0
    while len(drawn) < 4 or spent < budget_s:
        i = int(rs.integers(0, nb))
        dt = block_time(i)
        drawn.append((i, round(dt, 3)))
        spent += dt
        if len(drawn) >= 64:
            break
    per_block = sum(t for _, t in drawn) / len(drawn)
    rate = N / (t_proj + nb * per_block)
    return rate, {"t_projection_s": round(t_proj, 3), "t_per_block_s": round(per_block, 3),
                  "drawn_blocks": drawn, "fixed_blocks": fixed_t}


def cpu_cores():
    try:
        import threadpoolctl
        info = threadpoolctl.threadpool_info()
        n = max((i.get("num_threads", 1) for i in info), default=1)
        return int(n)
    except Exception:
        return os.cpu_count() or 1


def host_copies(pcfg, dev_tensors):
    q, k, v, P = dev_tensors
    return q[0].cpu(), k[0].cpu(), v[0].cpu(), P.cpu()


def run_cpu_baseline(pcfg, q, k, v, P, budget_s):
    qc, kc_, vc_, Pc = host_copies(pcfg, (q, k, v, P))
    t0 = time.perf_counter()
    rate, info = oracle_prefill_rate(pcfg, qc, kc_, vc_, Pc, budget_s)
    wall = time.perf_counter() - t0
    return {"value": round(rate, 2), "unit": "tok/s", "cores": cpu_cores(), "kind": "oracle",
            "sample": (f"{pcfg.name}: index projection of the whole sequence, then all {pcfg.Hq} heads on "
                       f"{len(info['drawn_blocks'])} uniformly drawn query blocks of 64 (plus the first, last and "
                       f"window-boundary blocks, reported apart), extrapolated to N={pcfg.N}"),
            "wall_s": round(wall, 1), "detail": info}


def run_reference(args, rank, world):
    """The oracle, as it stands, timed on the host cores over bounded samples of
    the same prefill workload (rank 0 only)."""
    if rank != 0:
        return None
    pcfg = synth.ALL_CONFIGS[args.prefill]
    dev = torch.device("cuda", 0) if torch.cuda.is_available() else torch.device("cpu")
    pd = synth.make_prefill(pcfg, device=dev)
    qc, kc_, vc_, Pc = host_copies(pcfg, (pd["q"], pd["k"], pd["v"], pd["P"]))
    del pd
    import numpy as np
    import oracle as O
    N, nb, G = pcfg.N, pcfg.N // BLOCK, pcfg.Hq // pcfg.Hkv
    t0 = time.perf_counter()
    kt = {g: O.project(kc_[:, g, :], Pc[g]) for g in sorted(set(h // G for h in pcfg.ret_heads))}
    qt = {h: O.project(qc[:, h, :], Pc[h // G]) for h in pcfg.ret_heads}
    t_proj = time.perf_counter() - t0
    rs = np.random.default_rng(1)
    times = []
    for s in range(args.warmup + args.steps):
        blk = [int(rs.integers(0, nb))]
        t0 = time.perf_counter()
        O.prefill_layer(qc, kc_, vc_, Pc, pcfg.ret_heads, pcfg.window, pcfg.ret_window, pcfg.topk,
                        1 / math.sqrt(D), qblocks=blk, index={"kt": kt, "qt": qt})
        if s >= args.warmup:
            times.append(time.perf_counter() - t0)
    per_block = sum(times) / len(times)
    step_s = t_proj / nb + per_block           # one query block with its share of the projection
    value = BLOCK / step_s
    cores = cpu_cores()
    return {"impl": "reference",
            "metric": "hybrid-attn prefill tok/s @1M & decode tok/s @128K per layer; % of roofline",
            "value": round(value, 2), "unit": "tok/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": round(step_s * 1e3, 1), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": pcfg.name, "B": pcfg.B, "N": N, "Hq": pcfg.Hq, "Hkv": pcfg.Hkv,
                       "retrieval_heads": list(pcfg.ret_heads), "swa_window": pcfg.window,
                       "topk_blocks": pcfg.topk},
            "cpu_baseline": {"value": round(value, 2), "unit": "tok/s", "cores": cores, "kind": "oracle",
                             "sample": ("each step: all heads on one random query block of 64 tokens, "
                                        "plus 1/(N/64) of the whole-sequence index projection")},
            "e2e": {"value": round(value, 2), "unit": "tok/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=3)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--prefill", default="prefill_1m")
    ap.add_argument("--decode", default="decode_128k_b8")
    ap.add_argument("--no-e2e", dest="e2e", action="store_false")
    ap.add_argument("--no-cpu-baseline", dest="cpu_baseline", action="store_false")
    ap.add_argument("--no-configs", dest="configs", action="store_false",
                    help="skip the other workloads' timings")
    ap.add_argument("--cpu-budget", type=float, default=20.0,
                    help="seconds of oracle block work in the CPU baseline sample")
    args = ap.parse_args()
    args.warmup = max(3, args.warmup)
    rank, world, local = dist_setup(args.gpus)
    if args.impl == "reference":
        line = run_reference(args, rank, world)
    else:
        line = run_ours(args, rank, world)
        if rank == 0 and world == 1 and args.cpu_baseline and line is not None:
            pcfg = synth.ALL_CONFIGS[args.prefill]
            pd = synth.make_prefill(pcfg, device=torch.device("cuda", 0))
            line["cpu_baseline"] = run_cpu_baseline(pcfg, pd["q"], pd["k"], pd["v"], pd["P"],
                                                    args.cpu_budget)
        elif line is not None:
            line["cpu_baseline"] = None
    if rank == 0 and line is not None:
        print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
