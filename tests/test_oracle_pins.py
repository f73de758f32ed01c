"""Pins of the CPU oracle to facts fixed by the pages and by mathematics.

None of these re-types an oracle formula: each checks the oracle against a
closed form, a worked example, brute force on a tiny input, an invariant, or an
independent computation (torch autograd for the straight-through gradients,
two separate matmuls for the layer MSE).
"""
import json
import os

import numpy as np
import pytest
import torch

import oracle
from oracle import autoround as ar
from workloads import bf16_round, channel_scale, make_weight

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")
F32 = np.float32


def _tiny_x(n, inn, seed=0, outliers=(1, 5)):
    rng = np.random.default_rng(seed)
    x = rng.standard_normal((n, inn)).astype(np.float32)
    x[:, list(outliers)] *= 20
    return bf16_round(x)


# ---------------------------------------------------------------- RTN / forward

def test_rtn_worked_grid_example():
    d = json.load(open(os.path.join(GOLDEN, "rtn_grid_example.json")))
    W = np.array([d["w"]], dtype=np.float32)
    codes, s, zp, Wq = oracle.rtn(W, d["bits"], d["group_size"], d["sym"])
    assert s[0, 0] == F32(d["scale"])
    assert zp[0, 0] == d["zero_point"]
    assert codes[0].tolist() == d["codes"]
    assert np.array_equal(Wq, W)


@pytest.mark.parametrize("case", [0, 1])
def test_minmax_shrink_worked_example(case):
    """minmax_shrink ("AutoRoundModifier 생성자 파라미터": the initial min/max range is
    scaled by this factor) on hand-worked grid groups: at iters = 0 the applied
    state is alpha = beta = shrink with V = 0, so the tuned layer's scale, zero-point
    and codes are the hand-worked ones; with shrink 1 they are the RTN ones."""
    d = json.load(open(os.path.join(GOLDEN, "shrink_grid_example.json")))["cases"][case]
    W = np.array([d["w"]], dtype=np.float32)
    X = _tiny_x(8, W.shape[1], seed=case)
    res = oracle.tune_layer(W, X, d["bits"], d["group_size"], d["sym"], 0, 0.005, -1.0, 8, 0,
                            minmax_shrink=d["minmax_shrink"])
    assert res.scale[0, 0] == F32(d["scale"])
    assert res.zero_point[0, 0] == d["zero_point"]
    assert res.codes[0].tolist() == d["codes"]
    one = oracle.tune_layer(W, X, d["bits"], d["group_size"], d["sym"], 0, 0.005, -1.0, 8, 0, minmax_shrink=1.0)
    assert one.scale[0, 0] == F32(d["rtn_scale"])
    assert one.codes[0].tolist() == d["rtn_codes"]
    # the shrunk start is where tuning begins: one step moves alpha (and beta) off it
    # by at most minmax_lr, inside [0.5, 1]
    r1 = oracle.tune_layer(W, X, d["bits"], d["group_size"], d["sym"], 1, 0.005, 0.005, 8, 0,
                           minmax_shrink=d["minmax_shrink"], keep_best=False)
    assert abs(float(r1.alpha[0, 0]) - d["minmax_shrink"]) <= 0.005 + 1e-9
    assert 0.5 <= float(r1.alpha[0, 0]) <= 1.0


@pytest.mark.parametrize("bits", [2, 3, 4, 8])
@pytest.mark.parametrize("sym", [False, True])
def test_rtn_is_nearest_level(bits, sym):
    """RTN picks, per element, the nearest of the Q+1 levels s*(c - zp) (brute force)."""
    W = make_weight(6, 64, 0.02, "f32", seed=3)
    W[0, :16] = 0.0                        # an all-zero group
    W[1, 16:32] = np.abs(W[1, 16:32])      # a one-signed group
    g = 16
    codes, s, zp, Wq = oracle.rtn(W, bits, g, sym)
    Q = 2 ** bits - 1
    se = np.repeat(s.astype(np.float64), g, 1)
    ze = np.repeat(zp.astype(np.float64), g, 1)
    levels = se[..., None] * (np.arange(Q + 1)[None, None, :] - ze[..., None])
    dist = np.abs(levels - W.astype(np.float64)[..., None])
    best = dist.min(axis=-1)
    mine = np.take_along_axis(dist, codes[..., None].astype(np.int64), -1)[..., 0]
    # the decision is taken on the fp32 quotient W/s: nearest up to its rounding
    ulp_u = np.abs(W.astype(np.float64) / se) * 2.0 ** -23
    assert np.all(mine <= best + se * (2 * ulp_u + 1e-9))
    np.testing.assert_allclose(Wq, np.take_along_axis(levels, codes[..., None].astype(np.int64), -1)[..., 0],
                               rtol=1e-7, atol=0)
    # the levels cover the group: every element within half a step of its level
    assert np.all(np.abs(Wq.astype(np.float64) - W) <= se * (0.5 + 2 * ulp_u + 1e-9))
    clear = np.sort(dist, axis=-1)[..., 1] - best > se * (4 * ulp_u + 1e-9)
    assert np.array_equal(codes[clear], dist.argmin(axis=-1)[clear])
    assert codes.max() <= Q


@pytest.mark.parametrize("bits", [2, 4, 8])
def test_rtn_minmax_span(bits):
    """Asymmetric min-max: level 0 sits on the group minimum and level Q on the maximum
    (within half a step), so every element is reconstructed to within s/2."""
    W = make_weight(8, 128, 0.02, "f32", seed=4)
    g = 32
    codes, s, zp, Wq = oracle.rtn(W, bits, g, False)
    Wg = W.reshape(8, -1, g).astype(np.float64)
    s64 = s.astype(np.float64)
    lo = s64 * (0 - zp)
    hi = s64 * (2 ** bits - 1 - zp)
    assert np.all(np.abs(lo - np.minimum(Wg.min(-1), 0)) <= 0.5 * s64 * (1 + 1e-5))
    assert np.all(np.abs(hi - np.maximum(Wg.max(-1), 0)) <= 0.5 * s64 * (1 + 1e-5))
    err = np.abs(Wq.astype(np.float64) - W).reshape(8, -1, g).max(-1)
    assert np.all(err <= 0.5 * s64 * (1 + 1e-5))


@pytest.mark.parametrize("sym", [False, True])
def test_rtn_scale_invariance(sym):
    """W -> 2W: identical codes and zero-points, scale exactly doubled."""
    W = make_weight(16, 256, 0.02, "bf16", seed=5)
    c1, s1, z1, _ = oracle.rtn(W, 4, 64, sym)
    c2, s2, z2, _ = oracle.rtn(2 * W, 4, 64, sym)
    assert np.array_equal(c1, c2) and np.array_equal(z1, z2)
    assert np.array_equal(s2, 2 * s1)


def test_group_size_minus_one_is_whole_row():
    W = make_weight(4, 96, 0.02, "f32", seed=6)
    a = oracle.rtn(W, 4, -1, False)
    b = oracle.rtn(W, 4, 96, False)
    for x, y in zip(a, b):
        assert np.array_equal(x, y)
    assert a[1].shape == (4, 1)


def test_fixed_offset_rounding_reachable_and_monotone():
    """With V in [-0.5, 0.5] the code moves at most one level from W/s, and a larger
    offset never gives a smaller code ("V controls the rounding direction")."""
    W = make_weight(8, 128, 0.02, "f32", seed=7)
    g, bits = 32, 4
    wmin, wmax = oracle.group_minmax(W, g)
    one = np.ones_like(wmin)
    s, zp = oracle.scale_zero_point(wmin, wmax, one, one, bits, False)
    rng = np.random.default_rng(0)
    V = rng.uniform(-0.5, 0.5, W.shape).astype(np.float32)
    V[0, :8] = 0.5
    V[0, 8:16] = -0.5
    fq = oracle.fake_quant(W, V, s, zp, g, bits)
    u = W.astype(np.float64) / np.repeat(s, g, 1)
    assert np.all(np.abs(fq.r - u) <= 1.0 + 1e-6)
    fq_hi = oracle.fake_quant(W, np.clip(V + F32(0.1), -0.5, 0.5), s, zp, g, bits)
    assert np.all(fq_hi.q >= fq.q)
    fq0 = oracle.fake_quant(W, np.zeros_like(W), s, zp, g, bits)
    assert np.all(fq.q[V > 0] >= fq0.q[V > 0]) and np.all(fq.q[V < 0] <= fq0.q[V < 0])


def test_rounding_is_torch_round():
    """The page's code rounds with torch.round (half to even).  On offsets built to
    put W/s + V exactly on half-integers, the codes equal torch's evaluation of
    clamp(round(W/s + V) + zp, 0, Q) in fp32."""
    W = make_weight(4, 64, 0.02, "f32", seed=8)
    g, bits = 16, 4
    wmin, wmax = oracle.group_minmax(W, g)
    one = np.ones_like(wmin)
    s, zp = oracle.scale_zero_point(wmin, wmax, one, one, bits, False)
    se = np.repeat(s, g, 1)
    ze = np.repeat(zp, g, 1)
    u = W / se
    V = ((np.floor(u) + F32(0.5)) - u).astype(np.float32)
    t = u + V
    assert np.sum(t == np.floor(t) + F32(0.5)) > 100          # many exact ties
    fq = oracle.fake_quant(W, V, s, zp, g, bits)
    tq = torch.clamp(torch.round(torch.from_numpy(W) / torch.from_numpy(se) + torch.from_numpy(V))
                     + torch.from_numpy(ze), 0, 2 ** bits - 1)
    assert np.array_equal(fq.q, tq.numpy())


# ---------------------------------------------------------------- gradients

def _ste(x):
    return x + (torch.round(x) - x).detach()


def _autograd_grads(W, V, alpha, beta, wmin, wmax, X, g, bits, sym, X_target=None):
    """dL/dV, dL/dalpha, dL/dbeta by torch autograd in fp64, rounding made straight-through.
    With X_target the target output is X_target W^T instead of X W^T."""
    Q = float(2 ** bits - 1)
    Wt = torch.from_numpy(W.astype(np.float64))
    Vt = torch.from_numpy(V.astype(np.float64)).requires_grad_()
    at = torch.from_numpy(alpha.astype(np.float64)).requires_grad_()
    bt = torch.from_numpy(beta.astype(np.float64)).requires_grad_()
    wmn = torch.from_numpy(wmin.astype(np.float64))
    wmx = torch.from_numpy(wmax.astype(np.float64))
    # the forward value of s is the fp32 one (the pages quantise W.float()); its
    # gradient is that of the exact formula
    s32, _ = oracle.scale_zero_point(wmin, wmax, alpha, beta, bits, sym)
    if sym:
        s = 2 * at * torch.maximum(-wmn, wmx) / Q
    else:
        s = (at * wmx - bt * wmn) / Q
    s = s + (torch.from_numpy(s32.astype(np.float64)) - s).detach()
    if sym:
        zp = torch.full_like(s, float(2 ** (bits - 1)))
    else:
        zp = torch.clamp(_ste(-bt * wmn / s), 0, Q)
    se = s.repeat_interleave(g, 1)
    ze = zp.repeat_interleave(g, 1)
    q = torch.clamp(_ste(Wt / se + Vt) + ze, 0, Q)
    Wq = se * (q - ze)
    Xt = torch.from_numpy(X.astype(np.float64))
    if X_target is None:
        R = Xt @ (Wq - Wt).T
    else:
        R = Xt @ Wq.T - torch.from_numpy(X_target.astype(np.float64)) @ Wt.T
    loss = (R ** 2).sum() / R.numel()
    loss.backward()
    db = np.zeros_like(beta, dtype=np.float64) if bt.grad is None else bt.grad.numpy()
    return Vt.grad.numpy(), at.grad.numpy(), db, R.detach().numpy()


@pytest.mark.parametrize("sym", [False, True])
@pytest.mark.parametrize("bits", [2, 4])
def test_gradients_match_autograd(sym, bits):
    _check_gradients(sym, bits, 16)


@pytest.mark.parametrize("sym", [False, True])
@pytest.mark.parametrize("bits", [2, 4])
def test_whole_row_gradients_match_autograd(sym, bits):
    """group_size = -1: d alpha and d beta summed over the whole row."""
    _check_gradients(sym, bits, -1)


def _check_gradients(sym, bits, group_size):
    out, inn, n = 8, 64, 48
    g = inn if group_size == -1 else group_size
    W = make_weight(out, inn, 0.02, "f32", seed=11)
    X = _tiny_x(n, inn, seed=12)
    rng = np.random.default_rng(13)
    V = rng.uniform(-0.5, 0.5, W.shape).astype(np.float32)
    wmin, wmax = oracle.group_minmax(W, group_size)
    alpha = rng.uniform(0.5, 1.0, wmin.shape).astype(np.float32)
    beta = rng.uniform(0.5, 1.0, wmin.shape).astype(np.float32)
    dV, da, db, R = _autograd_grads(W, V, alpha, beta, wmin, wmax, X, g, bits, sym)
    G = R.T @ X.astype(np.float64)
    sgn, dalpha, dbeta = oracle.step_gradients(W, V, alpha, beta, wmin, wmax, G, group_size, bits, sym)
    c = 2.0 / (n * out)                    # the factor the oracle leaves out of G
    assert np.array_equal(sgn[np.abs(dV) > 1e-12], np.sign(dV)[np.abs(dV) > 1e-12])
    assert np.all(sgn[dV == 0] == 0)
    np.testing.assert_allclose(c * dalpha, da, rtol=1e-9, atol=1e-15)
    np.testing.assert_allclose(c * dbeta, db, rtol=1e-9, atol=1e-15)
    # the clamp must have been active somewhere, so the clamped branch is exercised
    fq = oracle.fake_quant(W, V, *oracle.scale_zero_point(wmin, wmax, alpha, beta, bits, sym), group_size, bits)
    assert (~fq.m).any() and fq.m.any()


def test_one_step_from_zero():
    """From V = 0 one step moves every offset by exactly -lr*sign(dL/dV) (autograd)."""
    out, inn, g, n = 8, 64, 16, 64
    W = make_weight(out, inn, 0.02, "f32", seed=21)
    X = _tiny_x(n, inn, seed=22)
    lr = 0.005
    res = oracle.tune_layer(W, X, 4, g, False, 1, lr, 0.0, n, 0, keep_best=False,
                            want_final_mse=False)
    wmin, wmax = oracle.group_minmax(W, g)
    one = np.ones_like(wmin)
    dV, *_ = _autograd_grads(W, np.zeros_like(W), one, one, wmin, wmax, X, g, 4, False)
    expect = (-F32(lr) * np.sign(dV)).astype(np.float32)
    assert np.array_equal(res.V, expect)
    assert set(np.unique(res.V).tolist()) <= {-F32(lr), 0.0, F32(lr)}


def _quant_input(X, seed):
    """Stand-in for the output of already-quantised layers: X plus small noise, in bf16."""
    rng = np.random.default_rng(seed)
    return bf16_round(X + F32(0.05) * rng.standard_normal(X.shape).astype(np.float32) * np.abs(X).mean())


@pytest.mark.parametrize("sym", [False, True])
def test_fp_target_gradients_match_autograd(sym):
    """quant-aware input with a full-precision target: one step's moves of V, alpha
    and beta against autograd of mean((X W'^T - X_fp W^T)^2), from a random state
    (an exact-tie-free start: V = 0 puts the symmetric group maximum on W/s = 3.5
    exactly in fp32, which fp64 autograd rounds from the other side)."""
    out, inn, g, n = 8, 64, 16, 48
    W = make_weight(out, inn, 0.02, "f32", seed=41)
    Xf = _tiny_x(n, inn, seed=42)
    Xq = _quant_input(Xf, 43)
    lr = 0.005
    rng = np.random.default_rng(47)
    V0 = rng.uniform(-0.5, 0.5, W.shape).astype(np.float32)
    wmin, wmax = oracle.group_minmax(W, g)
    a0 = rng.uniform(0.6, 0.9, wmin.shape).astype(np.float32)
    b0 = rng.uniform(0.6, 0.9, wmin.shape).astype(np.float32)
    res = oracle.tune_layer(W, Xq, 3, g, sym, 1, lr, lr, n, 0, keep_best=False, want_final_mse=False,
                            V0=V0, alpha0=a0, beta0=b0, X_target=Xf)
    dV, da, db, R = _autograd_grads(W, V0, a0, b0, wmin, wmax, Xq, g, 3, sym, X_target=Xf)
    moved = np.abs(dV) > 1e-12
    expect_V = np.clip(V0 - F32(lr) * np.sign(dV).astype(np.float32), F32(-0.5), F32(0.5))
    assert np.array_equal(res.V[moved], expect_V[moved])
    assert np.array_equal(res.V[dV == 0], V0[dV == 0])
    assert np.array_equal(res.alpha, np.clip(a0 - F32(lr) * np.sign(da).astype(np.float32), F32(0.5), F32(1)))
    if not sym:
        assert np.array_equal(res.beta, np.clip(b0 - F32(lr) * np.sign(db).astype(np.float32), F32(0.5), F32(1)))
    # the step's loss is the batch MSE against the full-precision target (the oracle's W'
    # is the fp32 one, autograd's the fp64 product of the same factors)
    assert res.loss_trace[0] == pytest.approx(float(np.mean(R ** 2)), rel=1e-6)


def test_fp_target_final_mse_and_same_input():
    W = make_weight(16, 64, 0.02, "f32", seed=44)
    Xf = _tiny_x(128, 64, seed=45)
    Xq = _quant_input(Xf, 46)
    res = oracle.tune_layer(W, Xq, 4, 32, False, 6, 0.005, 0.005, 64, 0, X_target=Xf)
    Y = torch.from_numpy(Xf.astype(np.float64)) @ torch.from_numpy(W.astype(np.float64)).T
    Yq = torch.from_numpy(Xq.astype(np.float64)) @ torch.from_numpy(res.Wq.astype(np.float64)).T
    assert res.final_mse == pytest.approx(float(((Yq - Y) ** 2).mean()), rel=1e-10)
    # the target's own input gives the layer's usual loop
    a = oracle.tune_layer(W, Xf, 4, 32, False, 6, 0.005, 0.005, 64, 0, X_target=Xf)
    b = oracle.tune_layer(W, Xf, 4, 32, False, 6, 0.005, 0.005, 64, 0)
    assert np.array_equal(a.codes, b.codes)
    np.testing.assert_allclose(a.loss_trace, b.loss_trace, rtol=1e-9)


# ---------------------------------------------------------------- loop

def test_loss_trace_is_layer_mse():
    """The first step's batch loss equals mean((X W'^T - X W^T)^2) of RTN, from two matmuls."""
    W = make_weight(32, 64, 0.02, "f32", seed=31)
    X = _tiny_x(128, 64, seed=32)
    res = oracle.tune_layer(W, X, 4, 32, False, 3, 0.005, 0.005, 128, 0)
    _, _, _, Wq = oracle.rtn(W, 4, 32, False)
    assert res.loss_trace[0] == pytest.approx(ar.layer_mse(W, Wq, X), rel=1e-10)
    assert res.final_mse == pytest.approx(ar.layer_mse(W, res.Wq, X), rel=1e-10)


@pytest.mark.parametrize("sym", [False, True])
def test_iters_zero_is_rtn(sym):
    W = make_weight(16, 128, 0.02, "bf16", seed=41)
    X = _tiny_x(64, 128, seed=42)
    res = oracle.tune_layer(W, X, 3, 64, sym, 0, 0.005, -1.0, 64, 0)
    c, s, z, _ = oracle.rtn(W, 3, 64, sym)
    assert np.array_equal(res.codes, c) and np.array_equal(res.scale, s)
    assert np.array_equal(res.zero_point, z)


def _reachable_optimum(W, X, s, zp, g, bits):
    """Per output row, the lowest loss over every code vector the offsets can reach."""
    Q = 2 ** bits - 1
    u = W / np.repeat(s, g, 1)
    lo = np.rint(u - F32(0.5)).astype(np.int64)
    hi = np.rint(u + F32(0.5)).astype(np.int64)
    ze = np.repeat(zp, g, 1).astype(np.float64)
    se = np.repeat(s, g, 1).astype(np.float64)
    X64 = X.astype(np.float64)
    total = 0.0
    for j in range(W.shape[0]):
        choices = [np.arange(lo[j, k], hi[j, k] + 1) for k in range(W.shape[1])]
        grids = np.meshgrid(*choices, indexing="ij")
        r = np.stack([gr.ravel() for gr in grids], axis=1).astype(np.float64)
        q = np.clip(r + ze[j], 0, Q)
        Wq = se[j] * (q - ze[j])
        R = X64 @ (Wq - W[j].astype(np.float64)).T
        total += (R ** 2).sum(axis=0).min()
    return total / (X.shape[0] * W.shape[0])


@pytest.mark.parametrize("bits", [2, 4])
def test_tuned_loss_between_optimum_and_rtn(bits):
    """Tiny layer, one full batch, clip factors frozen.  The tuned codes are
    reachable by the offsets, so their loss is at least the brute-force optimum
    over every reachable rounding (hard, for the best and for the last iterate).
    The best-loss iterate includes step 0 = RTN, so it is never worse than RTN,
    and here it is strictly better."""
    out, inn, g, n = 4, 16, 8, 64
    W = make_weight(out, inn, 0.02, "f32", seed=51)
    X = _tiny_x(n, inn, seed=52, outliers=(3, 11))
    best = oracle.tune_layer(W, X, bits, g, False, 200, 0.005, 0.0, n, 0)
    last = oracle.tune_layer(W, X, bits, g, False, 200, 0.005, 0.0, n, 0, keep_best=False)
    wmin, wmax = oracle.group_minmax(W, g)
    one = np.ones_like(wmin)
    s, zp = oracle.scale_zero_point(wmin, wmax, one, one, bits, False)
    opt = _reachable_optimum(W, X, s, zp, g, bits)
    _, _, _, Wrtn = oracle.rtn(W, bits, g, False)
    rtn_loss = ar.layer_mse(W, Wrtn, X)
    assert best.final_mse >= opt * (1 - 1e-12)
    assert last.final_mse >= opt * (1 - 1e-12)
    assert best.final_mse < rtn_loss
    assert best.final_mse == pytest.approx(best.best_loss.mean(), rel=1e-12)
    assert best.final_mse <= best.loss_trace.min()
    assert opt < rtn_loss


def test_tuned_beats_rtn_tiny_config():
    """The tiny workload (256x256, W4 g64, 50 steps): tuned loss below RTN, states in range."""
    from workloads import TINY, make_activations
    W = make_weight(TINY.out, TINY.inn, TINY.w_std, TINY.w_dtype, seed=0)
    X = make_activations(TINY.n_rows, TINY.inn, TINY.x_kind, seed=0)
    res = oracle.tune_layer(W, X, TINY.bits, TINY.group_size, TINY.sym, TINY.iters, TINY.lr,
                            TINY.minmax_lr, TINY.batch_rows, 0)
    _, _, _, Wrtn = oracle.rtn(W, TINY.bits, TINY.group_size, TINY.sym)
    assert res.final_mse < ar.layer_mse(W, Wrtn, X)
    assert res.loss_trace[-1] < res.loss_trace[0]
    assert res.V.min() >= -0.5 and res.V.max() <= 0.5
    for a in (res.alpha, res.beta):
        assert a.min() >= 0.5 and a.max() <= 1.0
    assert res.codes.max() <= 15
    assert (res.alpha < 1).any()           # the clip factors actually moved
    last = oracle.tune_layer(W, X, TINY.bits, TINY.group_size, TINY.sym, TINY.iters, TINY.lr,
                             TINY.minmax_lr, TINY.batch_rows, 0, keep_best=False)
    assert last.final_mse < ar.layer_mse(W, Wrtn, X)   # the page's last iterate, 50 steps


def test_activation_scale_invariance():
    """X -> 2X scales every gradient by 4 exactly: same trajectory, loss x4."""
    W = make_weight(16, 64, 0.02, "f32", seed=61)
    X = _tiny_x(64, 64, seed=62)
    a = oracle.tune_layer(W, X, 4, 32, False, 30, 0.005, 0.005, 32, 7)
    b = oracle.tune_layer(W, 2 * X, 4, 32, False, 30, 0.005, 0.005, 32, 7)
    assert np.array_equal(a.codes, b.codes) and np.array_equal(a.V, b.V)
    assert np.array_equal(a.alpha, b.alpha) and np.array_equal(a.beta, b.beta)
    np.testing.assert_allclose(b.loss_trace, 4 * a.loss_trace, rtol=1e-12)


def test_row_independence():
    """Each output row tunes on its own: a row subset, or permuted rows, give the same rows."""
    W = make_weight(12, 64, 0.02, "f32", seed=71)
    X = _tiny_x(96, 64, seed=72)
    full = oracle.tune_layer(W, X, 2, 32, False, 25, 0.005, 0.005, 32, 3)
    perm = np.random.default_rng(0).permutation(12)
    sub = oracle.tune_layer(W[perm[:5]], X, 2, 32, False, 25, 0.005, 0.005, 32, 3)
    assert np.array_equal(sub.codes, full.codes[perm[:5]])
    assert np.array_equal(sub.V, full.V[perm[:5]])
    assert np.array_equal(sub.alpha, full.alpha[perm[:5]])
    assert np.array_equal(sub.V_best, full.V_best[perm[:5]])
    last = oracle.tune_layer(W[perm[:5]], X, 2, 32, False, 25, 0.005, 0.005, 32, 3, keep_best=False)
    assert np.array_equal(last.V, full.V[perm[:5]])


def test_resume_equals_uninterrupted():
    W = make_weight(8, 64, 0.02, "f32", seed=81)
    X = _tiny_x(128, 64, seed=82)
    full = oracle.tune_layer(W, X, 4, 32, False, 20, 0.005, 0.005, 32, 9)
    a = oracle.tune_layer(W, X, 4, 32, False, 7, 0.005, 0.005, 32, 9)
    b = oracle.tune_layer(W, X, 4, 32, False, 13, 0.005, 0.005, 32, 9,
                          V0=a.V, alpha0=a.alpha, beta0=a.beta, start_step=7,
                          best0=(a.best_loss, a.V_best, a.alpha_best, a.beta_best))
    assert np.array_equal(b.codes, full.codes) and np.array_equal(b.V, full.V)
    assert np.array_equal(b.V_best, full.V_best)
    assert np.array_equal(b.best_loss, full.best_loss)
    np.testing.assert_array_equal(np.concatenate([a.loss_trace, b.loss_trace]), full.loss_trace)


def test_best_step_is_the_applied_state():
    """The per-row loss trace and best step the oracle reports describe the state it
    applies: the trace's row mean is the batch loss, the best loss is the trace's first
    minimum per row, and re-running the loop for exactly best_step steps yields, on each
    row, the live state that keep-best applied (a run of k steps ends in the state that
    step k is evaluated at)."""
    W = make_weight(12, 64, 0.02, "f32", seed=83)
    X = _tiny_x(128, 64, seed=84)
    r = oracle.tune_layer(W, X, 3, 32, False, 16, 0.01, 0.01, 32, 5)
    np.testing.assert_allclose(r.row_loss_trace.mean(axis=1), r.loss_trace, rtol=1e-12)
    first_min = np.argmin(r.row_loss_trace, axis=0)
    assert np.array_equal(r.best_step, first_min)
    assert np.array_equal(r.best_loss, r.row_loss_trace[first_min, np.arange(12)])
    for j in range(12):
        k = int(r.best_step[j])
        part = oracle.tune_layer(W, X, 3, 32, False, k, 0.01, 0.01, 32, 5, want_final_mse=False)
        assert np.array_equal(part.V[j], r.V_best[j]), j
        assert np.array_equal(part.alpha[j], r.alpha_best[j]) and np.array_equal(part.beta[j], r.beta_best[j])


def test_layer_wide_keep_best_applies_one_step():
    """keep_best=2: one step for every row, the first minimum of the layer's batch loss
    (the trace), and its state is the live state after exactly that many steps, so a
    keep_best=False run of best_step steps gives the same codes, scales and zero-points.
    The per-row choice on the same case picks different steps for different rows (so the
    case separates the two modes), and with one row the two modes coincide."""
    W = make_weight(12, 64, 0.02, "f32", seed=83)
    X = _tiny_x(128, 64, seed=84)
    args = (W, X, 3, 32, False, 16, 0.01, 0.01, 32, 5)
    lw = oracle.tune_layer(*args, keep_best=2)
    per_row = oracle.tune_layer(*args)
    assert len(set(per_row.best_step.tolist())) > 1
    k = int(np.argmin(lw.loss_trace))
    assert np.all(lw.best_step == k)
    np.testing.assert_allclose(lw.best_loss, lw.row_loss_trace[k].sum(), rtol=1e-12)
    part = oracle.tune_layer(*args[:5], k, *args[6:], keep_best=False)
    assert np.array_equal(lw.codes, part.codes)
    assert np.array_equal(lw.scale, part.scale) and np.array_equal(lw.zero_point, part.zero_point)
    one = (W[:1], X, 3, 32, False, 16, 0.01, 0.01, 32, 5)
    a, b = oracle.tune_layer(*one, keep_best=2), oracle.tune_layer(*one)
    assert np.array_equal(a.codes, b.codes) and np.array_equal(a.best_step, b.best_step)


def test_layer_wide_keep_best_resumes():
    """A layer-wide run split at step k (live and best state handed over) equals one run."""
    W = make_weight(8, 64, 0.02, "f32", seed=85)
    X = _tiny_x(128, 64, seed=86)
    full = oracle.tune_layer(W, X, 2, 32, False, 20, 0.01, 0.01, 32, 7, keep_best=2, want_final_mse=False)
    first = oracle.tune_layer(W, X, 2, 32, False, 9, 0.01, 0.01, 32, 7, keep_best=2, want_final_mse=False)
    rest = oracle.tune_layer(W, X, 2, 32, False, 11, 0.01, 0.01, 32, 7, keep_best=2, want_final_mse=False,
                             V0=first.V, alpha0=first.alpha, beta0=first.beta, start_step=9,
                             best0=(first.best_loss, first.V_best, first.alpha_best, first.beta_best))
    assert np.array_equal(rest.codes, full.codes) and np.array_equal(rest.best_loss, full.best_loss)


# ---------------------------------------------------------------- schedule, pack

def test_splitmix64_reference_vectors():
    d = json.load(open(os.path.join(GOLDEN, "splitmix64.json")))
    for case in d["cases"]:
        gen = oracle.splitmix64_stream(case["seed"])
        got = [next(gen) for _ in case["outputs"]]
        assert got == [int(x) for x in case["outputs"]]


def test_block_schedule_is_per_epoch_permutation():
    nb, iters = 16, 200
    sched = oracle.block_schedule(nb, iters, 0)
    assert len(sched) == iters
    for e in range(iters // nb):
        assert sorted(sched[e * nb:(e + 1) * nb]) == list(range(nb))
    assert sched[:nb] != sched[nb:2 * nb]
    assert sched[:nb] != list(range(nb))
    assert oracle.block_schedule(1, 5, 0) == [0] * 5
    assert oracle.block_schedule(nb, 40, 1) != oracle.block_schedule(nb, 40, 0)


def test_pack_golden_cases():
    d = json.load(open(os.path.join(GOLDEN, "pack_cases.json")))
    for case in d["cases"]:
        codes = np.array([case["codes"]], dtype=np.uint8)
        words = oracle.pack_codes(codes, case["bits"]).view(np.uint32)[0]
        assert [format(int(w), "08X") for w in words] == case["words_hex"]


@pytest.mark.parametrize("bits", [2, 3, 4, 8])
def test_pack_matches_bitstream_and_round_trips(bits):
    rng = np.random.default_rng(bits)
    codes = rng.integers(0, 2 ** bits, size=(5, 96), dtype=np.uint8)
    packed = oracle.pack_codes(codes, bits)
    assert packed.shape == (5, 96 * bits // 32)
    # independent reading: numpy's little-endian bit unpacking of the words
    stream = np.unpackbits(packed.view(np.uint32).astype("<u4").view(np.uint8), axis=1,
                           bitorder="little")
    weights = 1 << np.arange(bits)
    decoded = (stream.reshape(5, 96, bits) * weights).sum(-1)
    assert np.array_equal(decoded, codes)
    assert np.array_equal(oracle.unpack_codes(packed, bits, 96), codes)


# ---------------------------------------------------------------- layer chain

def _bf16_neighbours(x64):
    x32 = x64.astype(np.float32)
    b = x32.view(np.uint32).astype(np.uint64)
    lo = ((b >> 16) << 16).astype(np.uint32).view(np.float32).astype(np.float64)
    hi = (((b >> 16) + 1) << 16).astype(np.uint32).view(np.float32).astype(np.float64)
    return lo, hi


def test_chain_bf16_rounding_is_nearest():
    rng = np.random.default_rng(5)
    x = rng.standard_normal(20000) * 10.0 ** rng.uniform(-3, 3, 20000)
    r = oracle.chain._bf16_round(x).astype(np.float64)
    lo, hi = _bf16_neighbours(x)
    best = np.minimum(np.abs(x - lo), np.abs(hi - x))
    assert np.all(np.abs(r - x) <= best)
    x32 = rng.standard_normal(20000).astype(np.float32)          # fp32 inputs: plain RNE
    assert np.array_equal(oracle.chain._bf16_round(x32.astype(np.float64)), bf16_round(x32))


def test_chain_dequant_reconstructs_grid_example():
    d = json.load(open(os.path.join(GOLDEN, "rtn_grid_example.json")))
    codes = np.array([d["codes"]], dtype=np.uint8)
    W = oracle.chain.dequant(codes, np.array([[d["scale"]]], np.float32), np.array([[d["zero_point"]]]), 16)
    assert np.array_equal(W[0], np.array(d["w"], np.float32))


def test_chain_linear_and_silu_match_torch():
    rng = np.random.default_rng(6)
    X = bf16_round(rng.standard_normal((64, 96)).astype(np.float32))
    Wq = (rng.standard_normal((40, 96)) * 0.02).astype(np.float32)
    add = bf16_round(rng.standard_normal((64, 40)).astype(np.float32))
    Y = oracle.chain.linear(X, Wq, add).astype(np.float64)
    ref = (torch.nn.functional.linear(torch.from_numpy(X.astype(np.float64)),
                                      torch.from_numpy(Wq.astype(np.float64))) + torch.from_numpy(add.astype(np.float64))).numpy()
    lo, hi = _bf16_neighbours(ref)
    assert np.all(np.abs(Y - ref) <= np.minimum(np.abs(ref - lo), np.abs(hi - ref)))
    a = bf16_round(rng.standard_normal(5000).astype(np.float32) * 4)
    b = bf16_round(rng.standard_normal(5000).astype(np.float32))
    y = oracle.chain.silu_mul(a, b).astype(np.float64)
    ref = (torch.nn.functional.silu(torch.from_numpy(a.astype(np.float64))) * torch.from_numpy(b.astype(np.float64))).numpy()
    lo, hi = _bf16_neighbours(ref)
    assert np.all(np.abs(y - ref) <= np.minimum(np.abs(ref - lo), np.abs(hi - ref)))
