"""The comparison helpers themselves, on the CPU: the index rounding-interval
check must accept an fp32-accumulated, bf16-rounded projection and reject one
with a plausible mistake (a dropped product, truncation instead of
round-to-nearest-even, a transposed projector)."""
import numpy as np
import pytest
import torch

from helpers import assert_index_close, band_check, index_bounds


def _data(n_rows=4000, seed=0):
    g = torch.Generator().manual_seed(seed)
    c = torch.randn(64, 128, generator=g)
    c = 3 * c / c.norm(dim=1, keepdim=True)
    x = (c[torch.randint(0, 64, (n_rows,), generator=g)] + torch.randn(n_rows, 128, generator=g)).to(torch.bfloat16)
    P = (torch.randn(128, 16, generator=g) / np.sqrt(128)).to(torch.bfloat16)
    return x, P


def _fp32_sum(x, P, order=None, drop=None):
    """fp32 sequential accumulation of the exact bf16 x bf16 products."""
    xf = x.float().numpy().astype(np.float32)
    Pf = P.float().numpy().astype(np.float32)
    acc = np.zeros((xf.shape[0], Pf.shape[1]), np.float32)
    for d in (order if order is not None else range(xf.shape[1])):
        if d == drop:
            continue
        acc = (acc + xf[:, d:d + 1] * Pf[d:d + 1, :]).astype(np.float32)
    return acc


def test_index_check_accepts_fp32_accumulation_in_any_order():
    x, P = _data()
    for order in (None, list(range(127, -1, -1)), list(np.random.default_rng(1).permutation(128))):
        g = torch.from_numpy(_fp32_sum(x, P, order)).to(torch.bfloat16).double().numpy()
        n_boundary = assert_index_close(g, x, P)
        assert n_boundary < g.size // 4      # the worst-case bound leaves most elements decided


def test_index_check_rejects_a_dropped_product():
    x, P = _data()
    g = torch.from_numpy(_fp32_sum(x, P, drop=37)).to(torch.bfloat16).double().numpy()
    with pytest.raises(AssertionError):
        assert_index_close(g, x, P)


def test_index_check_rejects_truncation():
    x, P = _data()
    f = torch.from_numpy(_fp32_sum(x, P))
    trunc = (f.view(torch.int32) & ~0xFFFF).view(torch.float32).double().numpy()   # round toward zero
    with pytest.raises(AssertionError):
        assert_index_close(trunc, x, P)


def test_index_check_rejects_a_transposed_projector_row_order():
    x, P = _data()
    Pw = P.flip(0)
    g = torch.from_numpy(_fp32_sum(x, Pw)).to(torch.bfloat16).double().numpy()
    with pytest.raises(AssertionError):
        assert_index_close(g, x, P)


def test_index_bounds_interval_holds_the_rounded_exact_value():
    x, P = _data(500)
    exact, accum, lo, hi = index_bounds(x, P)
    import oracle as O
    r = O.bf16_round(exact)
    assert np.all((lo <= r) & (r <= hi))
    assert np.all(accum > 0)


def test_band_check_rules():
    scores = np.array([5.0, 4.0, 3.0, 3.0005, 1.0])
    # k = 3: s_k = 3.0005 is within 1e-3 of 3.0, so {0, 1, 2} is also correct
    ok, amb, _ = band_check([0, 1, 2], [0, 1, 3], scores, 3)
    assert ok and amb == 2
    ok, _, msg = band_check([0, 2, 3], [0, 1, 3], scores, 3)
    assert not ok and "missing" in msg
    ok, _, msg = band_check([0, 1, 4], [0, 1, 3], scores, 3)
    assert not ok
    ok, _, msg = band_check([0, 1], [0, 1, 3], scores, 3)
    assert not ok and "size" in msg
