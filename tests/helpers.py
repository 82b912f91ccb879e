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


def index_bounds(x, P):
    """Where an fp32-accumulated, bf16-rounded index element may lie.

    The GPU sums the n = D exact bf16 x bf16 products in fp32 (tensor cores);
    the computed sum s is within ``accum = 2 * n * 2**-24 * sum|x||P|`` of the
    exact value y (recursive fp32 summation moves each partial sum by at most
    half an fp32 ulp; the factor 2 covers an accumulator that truncates).
    Rounding to bf16 is monotone, so bf16(s) lies in
    [bf16(y - accum), bf16(y + accum)]: where those two agree, the stored
    element is fixed exactly (it must equal the oracle's correctly rounded
    value); where they differ, y sits within the accumulation error of a bf16
    rounding boundary and either neighbour is correct.

    Returns (exact, accum, lo, hi) as fp64 arrays.
    """
    import oracle as O
    x64 = O.to_f64(x)
    P64 = O.to_f64(P)
    exact = O.project(x64, P64, round_to_bf16=False)
    accum = 2.0 * (np.abs(x64) @ np.abs(P64)) * x64.shape[-1] * 2.0 ** -24
    return exact, accum, O.bf16_round(exact - accum), O.bf16_round(exact + accum)


def assert_index_close(gpu_bf16, x, P):
    """A bf16 key/query index computed with fp32 accumulation: every element
    is the bf16 rounding of some value within the fp32 summation bound of the
    exact product (``index_bounds``). Elements whose rounding the bound
    decides must equal the correctly rounded exact value bit for bit; no
    count of mismatches is tolerated. Returns how many elements sat on a
    rounding boundary (either neighbour allowed)."""
    exact, accum, lo, hi = index_bounds(x, P)
    g = np.asarray(gpu_bf16, dtype=np.float64)
    bad = (g < lo) | (g > hi)
    if bad.any():
        k = np.flatnonzero(bad.reshape(-1))[0]
        raise AssertionError(f"{int(bad.sum())} of {g.size} index elements outside their rounding interval; "
                             f"first: got {g.reshape(-1)[k]!r}, exact {exact.reshape(-1)[k]!r}, "
                             f"allowed [{lo.reshape(-1)[k]!r}, {hi.reshape(-1)[k]!r}]")
    return int(np.sum(lo != hi))


def assert_f32_index_close(gpu_f32, x, P):
    """An fp32 (unrounded) query index: within the fp32 summation bound of the
    exact product."""
    exact, accum, _, _ = index_bounds(x, P)
    err = np.abs(np.asarray(gpu_f32, dtype=np.float64) - exact)
    assert np.all(err <= accum + 1e-30), f"fp32 index error {float((err / (accum + 1e-30)).max()):.3f} x bound"
