"""The chunked-accumulation mode of the Gram step (ar_tune_params.split = 2).

The tensor cores add each MMA's products into the fp32 accumulator with less than
round-to-nearest accuracy, so one accumulation over K = in (three pair products of
in / 16 steps each) drifts from the exact sum.  With split = 2 the step contraction
sums K in chunks of 512, each a fresh accumulation, and the epilogue adds the chunks
in fp32 round to nearest before the step.  Checked here:
- a layer whose K fits one chunk gives results bit-identical to split = 1 (the same
  accumulation, copied once through the running sum);
- small multi-chunk layers meet the usual bars against the oracle over every row;
- on the full-size q_proj layer the free-running code divergence against the oracle
  on sampled rows is printed beside split = 1's and held to the same bound.
"""
import numpy as np
import pytest
import torch

import oracle
from tests.free_running import code_bound, oracle_drift
from workloads import Q_PROJ_7B, make_activations, make_activations_cuda, make_weight

pytestmark = pytest.mark.gpu

CODE_TOL = 0.005
MSE_RTOL = 0.02


@pytest.fixture(scope="module")
def ar():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    import signed_gradient_rounding_b200 as ar
    return ar


def _run(ar, W, X, split, **kw):
    p = ar.make_params(split=split, algo="gram", **kw)
    Wd = torch.from_numpy(W).to(torch.bfloat16).cuda()
    Xd = torch.from_numpy(X).to(torch.bfloat16).cuda()
    st = ar.TuneState.empty(W.shape[0], W.shape[1], kw["group_size"])
    res = ar.tune_layer(Wd, Xd, p, state=st)
    assert ar.tune_status(res.workspace) == ar.AR_OK
    return res, st


def test_one_chunk_equals_one_accumulation(ar):
    W = make_weight(300, 512, 0.02, "bf16", seed=71)
    X = make_activations(2048, 512, "llm", seed=71)
    kw = dict(bits=3, group_size=128, iters=20, batch_rows=512, seed=3)
    a, sa = _run(ar, W, X, 2, **kw)
    b, sb = _run(ar, W, X, 1, **kw)
    torch.cuda.synchronize()
    assert torch.equal(a.codes, b.codes) and torch.equal(a.scale, b.scale)
    assert torch.equal(sa.V, sb.V) and torch.equal(sa.best_loss, sb.best_loss)
    assert torch.equal(a.loss_trace, b.loss_trace)


@pytest.mark.parametrize("shape", [(256, 1024, 2048, 512, 4, 64), (200, 1536, 1536, 512, 2, 128)],
                         ids=["W4-g64-2chunks", "W2-g128-3chunks-ragged"])
def test_multichunk_against_oracle(ar, shape):
    out, inn, n, B, bits, g = shape
    W = make_weight(out, inn, 0.02, "bf16", seed=73)
    X = make_activations(n, inn, "llm", seed=73)
    res, _ = _run(ar, W, X, 2, bits=bits, group_size=g, iters=24, batch_rows=B, seed=1)
    ref = oracle.tune_layer(W, X, bits, g, False, 24, 0.005, -1.0, B, 1)
    frac = float(np.mean(res.codes.cpu().numpy() != ref.codes))
    assert frac <= CODE_TOL, f"{frac:.4%} of codes differ"
    assert float(res.final_mse.item()) == pytest.approx(ref.final_mse, rel=MSE_RTOL)


def test_q_proj_free_running_divergence(ar):
    """64 sampled rows of the q_proj layer, 200 steps: split = 2 beside split = 1."""
    c = Q_PROJ_7B
    rows = np.sort(np.random.default_rng(11).choice(c.out, 64, replace=False))
    Wfull = make_weight(c.out, c.inn, c.w_std, c.w_dtype, seed=0)
    Xd = make_activations_cuda(c.n_rows, c.inn, c.x_kind, seed=0, device="cuda")
    Wd = torch.from_numpy(Wfull).to(torch.bfloat16).cuda()
    out = {}
    for split in (1, 2):
        p = ar.make_params(bits=c.bits, group_size=c.group_size, iters=c.iters, lr=c.lr, minmax_lr=c.minmax_lr,
                           batch_rows=c.batch_rows, seed=0, split=split, algo="gram")
        res = ar.tune_layer(Wd, Xd, p, want_final_mse=False)
        assert ar.tune_status(res.workspace) == ar.AR_OK
        out[split] = res.codes.cpu().numpy()[rows]
        del res
    X = Xd.view(torch.int16).cpu().numpy().view(np.uint16)
    ref = oracle.tune_layer(Wfull[rows], X, c.bits, c.group_size, False, c.iters, c.lr, c.minmax_lr, c.batch_rows, 0,
                            want_final_mse=False)
    d1 = float(np.mean(out[1] != ref.codes))
    d2 = float(np.mean(out[2] != ref.codes))
    print(f"\nq_proj sampled rows, codes differing from the oracle: split=1 {d1:.3%}, split=2 {d2:.3%}")
    bound = code_bound(oracle_drift(ref, Wfull[rows], X, c.bits, c.group_size, False, c.iters, c.lr, c.minmax_lr,
                                    c.batch_rows), len(rows))
    assert d2 <= bound and d1 <= bound
