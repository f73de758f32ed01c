"""Tuning with group sizes other than the usual 32 .. 256, against the oracle.

The pages' group size is -1 (a whole row) or any divisor of the row width.  Groups
that divide 256 (16 included) are updated inside the step kernel's epilogue.  Any
other group (a whole row of a wide layer, 384 or 512 columns, or sizes such as 48,
96 and 160 whose groups straddle the epilogue's 128-column segments) takes the wide path: the
epilogue writes per-segment partials of d alpha and d beta, and a per-group kernel
finishes the clip-factor update and the next D.  Both evaluation orders, both
quantiser modes, keep-best and the last iterate, the MSE init and the
full-precision-target mode are checked against the oracle with the usual bars.
"""
import numpy as np
import pytest
import torch

import oracle
from workloads import make_activations, make_quantised_path_input, make_weight

pytestmark = pytest.mark.gpu

CODE_TOL = 0.005
MSE_RTOL = 0.02


@pytest.fixture(scope="module")
def ar():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    import signed_gradient_rounding_b200 as ar
    return ar


def _dev_w(W, wdt):
    t = torch.from_numpy(W)
    return (t.to(torch.bfloat16) if wdt == "bf16" else t).cuda()


def _dev_x(X):
    return torch.from_numpy(X).to(torch.bfloat16).cuda()


def _close(res, ref, what):
    codes = res.codes.cpu().numpy()
    frac = float(np.mean(codes != ref.codes))
    mse = float(res.final_mse.item())
    assert frac <= CODE_TOL, f"{what}: {frac:.4%} of codes differ"
    assert mse == pytest.approx(ref.final_mse, rel=MSE_RTOL), f"{what}: mse {mse} vs {ref.final_mse}"


# (in, group_size): whole rows wider than 256, groups spanning several segments,
# and groups that straddle segment boundaries (96, 160).
SHAPES = [(384, -1), (512, -1), (768, 384), (1024, 512), (288, 96), (320, 160), (256, 16), (288, 48)]


@pytest.mark.parametrize("algo", ["gram", "direct"])
@pytest.mark.parametrize("inn,g", SHAPES, ids=[f"in{i}-g{g}" for i, g in SHAPES])
def test_wide_groups_match_oracle(ar, inn, g, algo):
    out, n, B, iters, bits = 200, 1536, 512, 24, 3
    W = make_weight(out, inn, 0.02, "bf16", seed=inn + g)
    X = make_activations(n, inn, "llm", seed=inn)
    p = ar.make_params(bits=bits, group_size=g, iters=iters, batch_rows=B, seed=2, algo=algo)
    res = ar.tune_layer(_dev_w(W, "bf16"), _dev_x(X), p)
    assert ar.tune_status(res.workspace) == ar.AR_OK
    ref = oracle.tune_layer(W, X, bits, g, False, iters, 0.005, -1.0, B, 2)
    _close(res, ref, f"in {inn} g {g} {algo}")
    np.testing.assert_allclose(res.loss_trace.cpu().numpy().astype(np.float64), ref.loss_trace, rtol=0.05)


@pytest.mark.parametrize("algo", ["gram", "direct"])
@pytest.mark.parametrize("keep_best", [True, False])
def test_whole_row_symmetric(ar, algo, keep_best):
    """W4 per-channel (group_size = -1) symmetric on a 512-wide fp32 layer."""
    out, inn, n, B, iters = 128, 512, 2048, 512, 30
    W = make_weight(out, inn, 0.02, "f32", seed=11)
    X = make_activations(n, inn, "llm", seed=11)
    p = ar.make_params(bits=4, group_size=-1, sym=True, iters=iters, batch_rows=B, seed=1, keep_best=keep_best,
                       algo=algo)
    res = ar.tune_layer(_dev_w(W, "f32"), _dev_x(X), p)
    assert ar.tune_status(res.workspace) == ar.AR_OK
    ref = oracle.tune_layer(W, X, 4, -1, True, iters, 0.005, -1.0, B, 1, keep_best=keep_best)
    _close(res, ref, f"per-channel sym {algo} keep_best={keep_best}")


def test_wide_groups_mse_init(ar):
    out, inn, n, B = 128, 768, 1024, 512
    W = make_weight(out, inn, 0.02, "bf16", seed=12)
    X = make_activations(n, inn, "llm", seed=12)
    p = ar.make_params(bits=2, group_size=384, iters=20, batch_rows=B, init="mse")
    res = ar.tune_layer(_dev_w(W, "bf16"), _dev_x(X), p)
    assert ar.tune_status(res.workspace) == ar.AR_OK
    ref = oracle.tune_layer(W, X, 2, 384, False, 20, 0.005, -1.0, B, 0, init="mse")
    _close(res, ref, "mse init g384")


def test_wide_groups_full_precision_target(ar):
    out, inn, n, B, iters = 200, 384, 1536, 512, 20
    W = make_weight(out, inn, 0.02, "bf16", seed=13)
    Xf = make_activations(n, inn, "llm", seed=13)
    Xq = make_quantised_path_input(Xf, 0.05, seed=13)
    p = ar.make_params(bits=3, group_size=-1, iters=iters, batch_rows=B, algo="gram")
    res = ar.tune_layer_fp_target(_dev_w(W, "bf16"), _dev_x(Xq), _dev_x(Xf), p)
    assert ar.tune_status(res.workspace) == ar.AR_OK
    ref = oracle.tune_layer(W, Xq, 3, -1, False, iters, 0.005, -1.0, B, 0, X_target=Xf)
    _close(res, ref, "fp target per-channel")


def test_wide_groups_single_bf16_operands(ar):
    """split = 0 runs the wide epilogue on unfused stages; the state stays in range."""
    out, inn, n, B = 128, 512, 1024, 512
    W = make_weight(out, inn, 0.02, "bf16", seed=14)
    X = make_activations(n, inn, "llm", seed=14)
    for algo in ("gram", "direct"):
        p = ar.make_params(bits=4, group_size=-1, iters=20, batch_rows=B, algo=algo, split=False)
        st = ar.TuneState.empty(out, inn, -1)
        res = ar.tune_layer(_dev_w(W, "bf16"), _dev_x(X), p, state=st)
        assert ar.tune_status(res.workspace) == ar.AR_OK
        ref = oracle.tune_layer(W, X, 4, -1, False, 20, 0.005, -1.0, B, 0)
        assert float(res.final_mse.item()) == pytest.approx(ref.final_mse, rel=MSE_RTOL)
        al, be = st.alpha.cpu().numpy(), st.beta.cpu().numpy()
        assert al.min() >= 0.5 and al.max() <= 1.0 and be.min() >= 0.5 and be.max() <= 1.0
