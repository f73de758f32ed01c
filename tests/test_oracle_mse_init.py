"""Pins of the oracle's MSE grid-search initialisation (oracle.autoround.mse_init).

The reading of "_init_scale_zp: Min-Max or MSE": per group, the clip ratio p on
the grid 1.00, 0.99, ..., 0.50 whose round-to-nearest weights have the smallest
squared error.  None of these tests re-types the oracle's arithmetic:
  * a group whose values sit exactly on the p = 1 grid has error 0 there;
  * an exact rational brute force (fractions.Fraction, round half to even) of
    the same definition picks the same ratio wherever its minimum is clear;
  * the chosen error never exceeds plain RTN's (the separate oracle.rtn path);
  * scaling W by a power of two leaves every choice unchanged.
"""
from fractions import Fraction

import numpy as np
import pytest

import oracle
from oracle import autoround as oar

F32 = np.float32


def _exact_round_half_even(x: Fraction) -> int:
    f = x.numerator // x.denominator
    rem = x - f
    if rem > Fraction(1, 2) or (rem == Fraction(1, 2) and f % 2 == 1):
        return f + 1
    return f


def _exact_group_errors(w, bits, sym):
    """Squared RTN error of one group for every grid ratio, in exact arithmetic."""
    Q = 2 ** bits - 1
    ws = [Fraction(float(x)) for x in w]
    wmin = min(min(ws), Fraction(0))
    wmax = max(max(ws), Fraction(0))
    errs = []
    for i in range(oar.MSE_GRID):
        p = Fraction(float(F32(100 - i) / F32(100)))   # the grid value as stored
        if sym:
            s = 2 * p * max(-wmin, wmax) / Q
            zp = 2 ** (bits - 1)
        else:
            s = (p * wmax - p * wmin) / Q
            zp = None
        if s == 0:
            s = Fraction(1)
        if zp is None:
            zp = min(max(_exact_round_half_even(-p * wmin / s), 0), Q)
        e = Fraction(0)
        for x in ws:
            q = min(max(_exact_round_half_even(x / s) + zp, 0), Q)
            e += (s * (q - zp) - x) ** 2
        errs.append(e)
    return errs


def test_grid_aligned_group_keeps_full_range():
    # k / 16, k = 0 .. 15 on 4 bits: s = 1/16 exactly at p = 1, every value a level
    W = (np.arange(16, dtype=np.float32) / 16)[None, :]
    p, e = oar.mse_init(W, 16, 4, False)
    assert p[0, 0] == F32(1.0) and e[0, 0] == 0.0


@pytest.mark.parametrize("bits,sym", [(2, False), (3, False), (4, False), (3, True), (4, True)])
def test_exact_brute_force_agrees(bits, sym):
    rng = np.random.default_rng(10 + bits + 7 * sym)
    g = 8
    W = rng.normal(0, 0.02, (60, g)).astype(np.float32)
    W[::3, rng.integers(0, g)] *= 6                      # outliers in every third group
    p, _ = oar.mse_init(W, g, bits, sym)
    checked = 0
    for row in range(W.shape[0]):
        errs = _exact_group_errors(W[row], bits, sym)
        order = sorted(range(len(errs)), key=lambda i: (errs[i], i))
        best, second = errs[order[0]], errs[order[1]]
        if best > 0 and (second - best) / best < Fraction(1, 10 ** 5):
            continue                                     # a near tie: fp32 may pick either
        assert p[row, 0] == F32(100 - order[0]) / F32(100), (row, order[:3])
        checked += 1
    assert checked >= 40


@pytest.mark.parametrize("bits,sym", [(2, False), (4, False), (3, True)])
def test_never_worse_than_rtn(bits, sym):
    W = np.random.default_rng(3).normal(0, 0.02, (32, 256)).astype(np.float32)
    p, e = oar.mse_init(W, 64, bits, sym)
    _, _, _, Wq = oracle.rtn(W, bits, 64, sym)
    rtn_err = ((Wq.astype(np.float64) - W.astype(np.float64)) ** 2).reshape(32, 4, 64).sum(axis=2)
    assert np.all(e <= rtn_err * (1 + 1e-12))
    assert np.any(p < 1)


def test_power_of_two_scale_invariance():
    W = np.random.default_rng(4).normal(0, 0.02, (16, 128)).astype(np.float32)
    p1, e1 = oar.mse_init(W, 32, 3, False)
    p2, e2 = oar.mse_init(W * F32(4), 32, 3, False)
    assert np.array_equal(p1, p2)
    assert np.array_equal(e2, e1 * 16)


def test_tune_layer_uses_mse_ratios_at_step_zero():
    """iters = 0 applies the initial state: the scales are those of the chosen ratios."""
    rng = np.random.default_rng(5)
    W = rng.normal(0, 0.02, (8, 128)).astype(np.float32)
    X = oracle.autoround._to_f32(rng.standard_normal((64, 128)).astype(np.float32))
    res = oar.tune_layer(W, X, 2, 64, False, 0, 0.005, -1.0, 64, 0, init="mse")
    p, _ = oar.mse_init(W, 64, 2, False)
    wmin, wmax = oar.group_minmax(W, 64)
    s, _ = oar.scale_zero_point(wmin, wmax, p, p, 2, False)
    assert np.array_equal(res.scale, s)
    assert np.array_equal(res.alpha, p) and np.array_equal(res.beta, p)


def test_all_zero_group_keeps_full_range():
    """Every ratio gives an all-zero group zero error: the first minimum (p = 1) is kept."""
    W = np.zeros((2, 64), dtype=np.float32)
    W[1, :32] = np.random.default_rng(6).normal(0, 0.02, 32).astype(np.float32)   # one live group
    p, e = oar.mse_init(W, 32, 4, False)
    assert p[0, 0] == F32(1.0) and p[0, 1] == F32(1.0) and e[0, 0] == 0.0
