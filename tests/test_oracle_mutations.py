"""Planted mistakes: each plausible slip in the oracle must make one of its pins fail.

The mistakes are planted in the oracle, on the CPU, by monkeypatching one of its
functions with a wrong variant; the pins are the functions of test_oracle_pins.
"""
import numpy as np
import pytest

import oracle
from oracle import autoround as oar
from tests import test_oracle_pins as pins

F32 = np.float32


def _szp_zp_sign(wmin, wmax, alpha, beta, bits, sym):
    s, zp = _orig_szp(wmin, wmax, alpha, beta, bits, sym)
    if not sym:
        Q = oar.qmax(bits)
        zp = np.clip(np.rint((beta * wmin) / s), F32(0), Q).astype(F32)   # lost the minus sign
    return s, zp


def _szp_q_plus_one(wmin, wmax, alpha, beta, bits, sym):
    s, zp = _orig_szp(wmin, wmax, alpha, beta, bits, sym)
    s = (s * oar.qmax(bits) / F32(2 ** bits)).astype(F32)                # divided by 2^b, not 2^b - 1
    return s, zp


_orig_szp = oar.scale_zero_point
_orig_grads = oar.step_gradients
_orig_fq = oar.fake_quant


def _grads_no_mask(W, V, alpha, beta, wmin, wmax, G, group_size, bits, sym):
    sgn, da, db = _orig_grads(W, V, alpha, beta, wmin, wmax, G, group_size, bits, sym)
    return np.sign(G).astype(F32), da, db                                # forgot the clamp mask


def _grads_alpha_flipped(W, V, alpha, beta, wmin, wmax, G, group_size, bits, sym):
    sgn, da, db = _orig_grads(W, V, alpha, beta, wmin, wmax, G, group_size, bits, sym)
    return sgn, -da, db                                                  # wrong sign of ds/dalpha


def _grads_no_zp_term(W, V, alpha, beta, wmin, wmax, G, group_size, bits, sym):
    # recompute dbeta with the zero-point's derivative dropped in the clamped branch
    sgn, da, db = _orig_grads(W, V, alpha, beta, wmin, wmax, G, group_size, bits, sym)
    s, zp = oar.scale_zero_point(wmin, wmax, alpha, beta, bits, sym)
    fq = oar.fake_quant(W, V, s, zp, group_size, bits)
    g = group_size
    ds_b = -np.asarray(wmin, np.float64) / float(oar.qmax(bits))
    qz = fq.q.astype(np.float64) - np.repeat(zp.astype(np.float64), g, 1)
    ratio = W.astype(np.float64) / np.repeat(s.astype(np.float64), g, 1)
    dWb = np.where(fq.m, np.repeat(ds_b, g, 1) * (fq.r - ratio), np.repeat(ds_b, g, 1) * qz)
    db2 = (np.asarray(G) * dWb).reshape(W.shape[0], -1, g).sum(-1)
    return sgn, da, (np.zeros_like(db2) if sym else db2)


def _fq_round_half_up(W, V, s, zp, group_size, bits):
    fq = _orig_fq(W, V, s, zp, group_size, bits)
    r = np.floor(fq.t + F32(0.5)).astype(F32)                           # not torch.round's half-to-even
    Q = oar.qmax(bits)
    ze = np.repeat(np.asarray(zp, F32), W.shape[1] // np.asarray(s).shape[1], 1)
    se = np.repeat(np.asarray(s, F32), W.shape[1] // np.asarray(s).shape[1], 1)
    p = r + ze
    q = np.clip(p, F32(0), Q)
    return oar.FakeQuant(fq.u, fq.t, r, p, q, (p >= 0) & (p <= Q), se * (q - ze))


def _plant(monkeypatch, name, fn):
    """Replace an oracle function everywhere it can be reached from."""
    monkeypatch.setattr(oar, name, fn)
    if hasattr(oracle, name):
        monkeypatch.setattr(oracle, name, fn)


def _caught(*checks) -> bool:
    """True if at least one pin fails under the planted mistake."""
    for check in checks:
        try:
            check()
        except AssertionError:
            return True
    return False


RTN_PINS = (lambda: pins.test_rtn_worked_grid_example(), lambda: pins.test_rtn_is_nearest_level(4, False),
            lambda: pins.test_rtn_minmax_span(4))


def test_zero_point_sign_is_caught(monkeypatch):
    _plant(monkeypatch, "scale_zero_point", _szp_zp_sign)
    assert _caught(*RTN_PINS)


def test_wrong_level_count_is_caught(monkeypatch):
    _plant(monkeypatch, "scale_zero_point", _szp_q_plus_one)
    assert _caught(*RTN_PINS)


@pytest.mark.parametrize("mutant", [_grads_no_mask, _grads_alpha_flipped, _grads_no_zp_term])
def test_gradient_mistakes_are_caught(monkeypatch, mutant):
    _plant(monkeypatch, "step_gradients", mutant)
    with pytest.raises(AssertionError):
        pins.test_gradients_match_autograd(False, 2)


def test_update_direction_is_caught(monkeypatch):
    def ascend(W, V, alpha, beta, wmin, wmax, G, group_size, bits, sym):
        sgn, da, db = _orig_grads(W, V, alpha, beta, wmin, wmax, G, group_size, bits, sym)
        return -sgn, -da, -db                                            # V += lr*sign(grad)
    _plant(monkeypatch, "step_gradients", ascend)
    with pytest.raises(AssertionError):
        pins.test_one_step_from_zero()


def test_rounding_mode_is_caught(monkeypatch):
    _plant(monkeypatch, "fake_quant", _fq_round_half_up)
    with pytest.raises(AssertionError):
        pins.test_rounding_is_torch_round()


# ---------------------------------------------------------------- MSE init and full-precision target

from tests import test_oracle_mse_init as mse_pins  # noqa: E402

_orig_mse_init = oar.mse_init


def _mse_init_variant(W, group_size, bits, sym, score="l2", beta_one=False, last_min=False):
    """mse_init with one slip: an L1 score, beta left at 1, or the last minimum kept."""
    W = oar._to_f32(W)
    out, inn = W.shape
    g = oar._group(inn, group_size)
    wmin, wmax = oar.group_minmax(W, g)
    best_p = np.ones(wmin.shape, dtype=F32)
    best_e = np.full(wmin.shape, np.inf)
    for i in range(oar.MSE_GRID):
        p = F32(100 - i) / F32(100)
        a = np.full(wmin.shape, p, dtype=F32)
        b = np.ones_like(a) if beta_one else a
        sc, zp = oar.scale_zero_point(wmin, wmax, a, b, bits, sym)
        d = oar.fake_quant(W, np.zeros_like(W), sc, zp, g, bits).Wq - W
        d = d.astype(np.float64).reshape(out, inn // g, g)
        e = np.cumsum(np.abs(d) if score == "l1" else d * d, axis=2)[:, :, -1]
        better = (e <= best_e) if last_min else (e < best_e)
        best_e = np.where(better, e, best_e)
        best_p = np.where(better, p, best_p).astype(F32)
    return best_p, best_e


MSE_PINS = (lambda: mse_pins.test_grid_aligned_group_keeps_full_range(),
            lambda: mse_pins.test_exact_brute_force_agrees(2, False),
            lambda: mse_pins.test_exact_brute_force_agrees(4, False),
            lambda: mse_pins.test_never_worse_than_rtn(2, False),
            lambda: mse_pins.test_all_zero_group_keeps_full_range())


@pytest.mark.parametrize("slip", [dict(score="l1"), dict(beta_one=True), dict(last_min=True)],
                         ids=["l1-score", "beta-left-at-1", "last-minimum"])
def test_mse_init_mistakes_are_caught(monkeypatch, slip):
    _plant(monkeypatch, "mse_init", lambda W, gs, bits, sym: _mse_init_variant(W, gs, bits, sym, **slip))
    assert _caught(*MSE_PINS)


def test_dropped_target_input_is_caught(monkeypatch):
    """The full-precision-target mode silently running the usual loop."""
    orig = oar.tune_layer

    def dropped(*args, X_target=None, **kw):
        return orig(*args, **kw)
    _plant(monkeypatch, "tune_layer", dropped)
    assert _caught(lambda: pins.test_fp_target_gradients_match_autograd(False),
                   lambda: pins.test_fp_target_final_mse_and_same_input())


_orig_tune = oar.tune_layer


def _tune_shrink_ignored(*args, **kw):
    kw["minmax_shrink"] = 1.0                                            # the start ignores minmax_shrink
    return _orig_tune(*args, **kw)


def _tune_shrink_alpha_only(W, X, bits, group_size, sym, iters, lr, minmax_lr, batch_rows, seed,
                            minmax_shrink=1.0, **kw):
    wmin, _ = oar.group_minmax(W, group_size)
    kw["beta0"] = np.ones(wmin.shape, F32)                               # beta left at 1
    return _orig_tune(W, X, bits, group_size, sym, iters, lr, minmax_lr, batch_rows, seed,
                      minmax_shrink=minmax_shrink, **kw)


@pytest.mark.parametrize("slip", [_tune_shrink_ignored, _tune_shrink_alpha_only])
def test_minmax_shrink_mistakes_are_caught(monkeypatch, slip):
    _plant(monkeypatch, "tune_layer", slip)
    assert _caught(lambda: pins.test_minmax_shrink_worked_example(0), lambda: pins.test_minmax_shrink_worked_example(1))


def _tune_layer_wide_as_per_row(*args, **kw):
    if kw.get("keep_best") == 2:
        kw["keep_best"] = True                                           # the layer choice made per row
    return _orig_tune(*args, **kw)


def _tune_layer_wide_as_last(*args, **kw):
    if kw.get("keep_best") == 2:
        kw["keep_best"] = False                                          # the last state applied
    return _orig_tune(*args, **kw)


@pytest.mark.parametrize("slip", [_tune_layer_wide_as_per_row, _tune_layer_wide_as_last])
def test_layer_wide_keep_best_mistakes_are_caught(monkeypatch, slip):
    _plant(monkeypatch, "tune_layer", slip)
    assert _caught(lambda: pins.test_layer_wide_keep_best_applies_one_step())
