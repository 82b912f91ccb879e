"""Comparison rules shared by the parity tests.

Index sets: identical, except inside the band of the k-th score. An oracle
element is ambiguous when its score s satisfies |s - s_k| <= 1e-3 * |s_k|
(s_k the oracle's k-th best score); such elements may be in or out. The GPU
set must hold every non-ambiguous selected element, no non-ambiguous
unselected element, and have the same size.

Attention outputs: max-abs <= 2e-2 and relative L2 <= 5e-3 against the fp64
oracle, with bf16 inputs.
"""
import numpy as np

BAND_REL = 1e-3
ATOL_MAX = 2e-2
REL_L2 = 5e-3


def band_check(gpu_sel, oracle_sel, scores, k):
    """Returns (ok, n_ambiguous, message) for one list.

    ``gpu_sel`` may carry -1 padding. ``scores`` are the oracle's scores over
    all candidates (index = candidate id).
    """
    g = np.asarray(gpu_sel)
    g = np.sort(g[g >= 0])
    o = np.sort(np.asarray(oracle_sel))
    if len(g) != len(o):
        return False, 0, f"size {len(g)} != {len(o)}"
    if np.array_equal(g, o):
        return True, 0, ""
    scores = np.asarray(scores, dtype=np.float64)
    n = len(scores)
    if n <= k:
        return False, 0, "all candidates must be selected"
    sk = np.sort(scores)[::-1][k - 1]
    amb = np.abs(scores - sk) <= BAND_REL * abs(sk)
    gs, os_ = set(g.tolist()), set(o.tolist())
    for x in os_ - gs:
        if not amb[x]:
            return False, int(amb.sum()), f"missing non-ambiguous {x} (score {scores[x]}, s_k {sk})"
    for x in gs - os_:
        if x < 0 or x >= n or not amb[x]:
            return False, int(amb.sum()), f"extra non-ambiguous {x}"
    return True, int(amb.sum()), ""


def attn_errors(gpu, ref):
    gpu = np.asarray(gpu, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    max_abs = float(np.abs(gpu - ref).max()) if gpu.size else 0.0
    rel = float(np.linalg.norm(gpu - ref) / max(np.linalg.norm(ref), 1e-30))
    return max_abs, rel


def assert_attn_close(gpu, ref, what=""):
    max_abs, rel = attn_errors(gpu, ref)
    assert max_abs <= ATOL_MAX and rel <= REL_L2, f"{what}: max_abs {max_abs:.3e}, rel_l2 {rel:.3e}"
    return max_abs, rel


def bf16_ulp_diff(a, b):
    """Distance in bf16 units in the last place between two bf16-valued arrays."""
    import torch
    ta = torch.as_tensor(np.asarray(a, dtype=np.float32)).to(torch.bfloat16).view(torch.int16).to(torch.int32)
    tb = torch.as_tensor(np.asarray(b, dtype=np.float32)).to(torch.bfloat16).view(torch.int16).to(torch.int32)
    # map sign-magnitude to a monotone integer line
    ta = torch.where(ta < 0, -(ta & 0x7FFF), ta)
    tb = torch.where(tb < 0, -(tb & 0x7FFF), tb)
    return (ta - tb).abs().numpy()


def assert_index_close(gpu_bf16, x, P, min_identical=0.999):
    """A bf16 key/query index computed with fp32 accumulation: every element
    lies within the fp32 summation bound (n * 2**-24 * sum|x||P|) plus half a
    bf16 ulp (2**-8 relative) of the exact product, and nearly all elements
    equal the oracle's correctly rounded value bit for bit."""
    import oracle as O
    x64 = O.to_f64(x)
    P64 = O.to_f64(P)
    exact = O.project(x64, P64, round_to_bf16=False)
    g = np.asarray(gpu_bf16, dtype=np.float64)
    accum = (np.abs(x64) @ np.abs(P64)) * x64.shape[-1] * 2.0 ** -24
    bound = np.abs(exact) * 2.0 ** -8 + accum * (1 + 2.0 ** -7) + 1e-30
    err = np.abs(g - exact)
    assert np.all(err <= bound), f"projection error {float((err / bound).max()):.3f} x bound"
    n_diff = int(np.sum(g != O.bf16_round(exact)))
    allowed = max(4, int((1 - min_identical) * g.size))
    assert n_diff <= allowed, f"{n_diff} of {g.size} elements differ from the rounded exact value"
    return n_diff
