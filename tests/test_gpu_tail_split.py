"""The step launches split the tiles of a last partial wave of at most half the
clusters into two column-half units (N = 128 tcgen05 MMAs into that half's columns of
the accumulator, epilogue by that half's warps).  Every output element is the same
accumulation over K either way, so with the split (the default) and without it
(AR_TAIL_SPLIT=0) a tuning run must give bit-identical results: codes, scales,
zero-points, the live and best state, and the loss trace.

Shapes: 80 pair tiles (10 x 8; on 74 clusters a last wave of 6 tiles), 8 tiles
(all of them split), a per-channel layer (the wide-group epilogue) and g = 64,
in both the plain and the full-precision-target step.
"""
import os

import numpy as np
import pytest
import torch

from workloads import make_activations, make_weight

pytestmark = pytest.mark.gpu

CASES = {
    "tiles80_g128": dict(out=2560, inn=2048, n=2048, B=1024, bits=4, g=128),
    "tiles8_g64": dict(out=512, inn=1024, n=2048, B=512, bits=2, g=64),
    "per_channel": dict(out=512, inn=2048, n=2048, B=512, bits=2, g=-1),
    "wide_g512": dict(out=768, inn=2048, n=1024, B=512, bits=3, g=512),
}


@pytest.fixture(scope="module")
def ar():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    import signed_gradient_rounding_b200 as ar
    return ar


def _run(ar, c, split: bool, fp_target: bool):
    W = torch.from_numpy(make_weight(c["out"], c["inn"], 0.02, "bf16", seed=61)).to(torch.bfloat16).cuda()
    X = torch.from_numpy(make_activations(c["n"], c["inn"], "llm", seed=61)).to(torch.bfloat16).cuda()
    p = ar.make_params(bits=c["bits"], group_size=c["g"], iters=12, batch_rows=c["B"], seed=5, algo="gram")
    st = ar.TuneState.empty(c["out"], c["inn"], c["g"])
    old = os.environ.get("AR_TAIL_SPLIT")
    os.environ["AR_TAIL_SPLIT"] = "1" if split else "0"
    try:
        if fp_target:
            Xt = (X.float() * 1.01).to(torch.bfloat16)
            res = ar.tune_layer_fp_target(W, X, Xt, p, state=st)
        else:
            res = ar.tune_layer(W, X, p, state=st)
        torch.cuda.synchronize()
    finally:
        if old is None:
            del os.environ["AR_TAIL_SPLIT"]
        else:
            os.environ["AR_TAIL_SPLIT"] = old
    assert ar.tune_status(res.workspace) == ar.AR_OK
    outs = [res.codes, res.scale, res.zero_point, res.loss_trace, res.final_mse,
            st.V, st.alpha, st.beta, st.V_best, st.alpha_best, st.beta_best, st.best_loss]
    return [t.cpu().numpy() for t in outs]


@pytest.mark.parametrize("fp_target", [False, True], ids=["plain", "fp-target"])
@pytest.mark.parametrize("name", sorted(CASES))
def test_split_is_bit_identical(ar, name, fp_target):
    c = CASES[name]
    a = _run(ar, c, True, fp_target)
    b = _run(ar, c, False, fp_target)
    names = ["codes", "scale", "zp", "loss_trace", "final_mse", "V", "alpha", "beta", "V_best", "alpha_best",
             "beta_best", "best_loss"]
    for n, x, y in zip(names, a, b):
        assert np.array_equal(x, y), f"{n}: {np.count_nonzero(x != y)} of {x.size} differ"
