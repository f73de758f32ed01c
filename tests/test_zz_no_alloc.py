"""ar_tune_layer_static: tuning for callers that cannot allocate device memory.

Some callers cannot call cudaMalloc when they tune -- their device memory is
owned by another allocator, or the call must not trigger the synchronisation an
allocation can cause.  ar_tune_layer_static takes only inputs and outputs and
keeps its scratch in one fixed device array inside the library.  This file is
collected last, so that a run stopping at the first failure has run every other
test first.

The check: through the C ABI, two calls in a row of the static entry point give
exactly the outputs of ar_tune_layer with a caller-allocated workspace (the same
kernels on the same inputs are deterministic, so the tolerance is zero), the
second call leaves the device's free memory and torch's allocated bytes as the
first left them, and a layer needing more scratch than the array holds is
refused before any work.
"""
import ctypes

import numpy as np
import pytest
import torch

from workloads import TINY, make_activations, make_weight

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def ar():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    import signed_gradient_rounding_b200 as ar
    return ar


def _outputs(out, inn, p):
    G = inn // p.group_size
    return (torch.full((out, inn), 255, dtype=torch.uint8, device="cuda"),
            torch.full((out, G), -1.0, dtype=torch.float32, device="cuda"),
            torch.full((out, G), -1, dtype=torch.int32, device="cuda"),
            torch.full((p.iters,), -1.0, dtype=torch.float32, device="cuda"),
            torch.full((1,), -1.0, dtype=torch.float64, device="cuda"))


def _static_call(ar, Wd, Xd, p, outs):
    """One call of the static entry point into preallocated outputs; returns the
    device's free memory (cudaMemGetInfo) and torch's allocated bytes afterwards."""
    out, inn = Wd.shape
    codes, scale, zp, trace, mse = outs
    st = ar.lib.ar_tune_layer_static(ar._ptr(Wd), ar.AR_F32 if Wd.dtype == torch.float32 else ar.AR_BF16,
                                     out, inn, ar._ptr(Xd), Xd.shape[0], ctypes.byref(p), ar._ptr(codes),
                                     ar._ptr(scale), ar._ptr(zp), ar._ptr(trace), ar._ptr(mse),
                                     ar._stream(None))
    assert st == ar.AR_OK, ar.lib.ar_status_string(st)
    torch.cuda.synchronize()
    return torch.cuda.mem_get_info()[0], torch.cuda.memory_allocated()


@pytest.mark.parametrize("algo", ["gram", "direct"])
def test_static_scratch_matches_workspace_entry_point(ar, algo):
    c = TINY
    W = make_weight(c.out, c.inn, c.w_std, c.w_dtype, seed=0)
    X = make_activations(c.n_rows, c.inn, c.x_kind, seed=0)
    Wd = torch.from_numpy(W).cuda()
    Xd = torch.from_numpy(X).to(torch.bfloat16).cuda()
    p = ar.make_params(bits=c.bits, group_size=c.group_size, iters=c.iters, lr=c.lr, minmax_lr=c.minmax_lr,
                       batch_rows=c.batch_rows, seed=0, algo=algo)
    assert ar.tune_workspace_bytes(c.out, c.inn, c.n_rows, p) <= ar.lib_static_scratch_bytes()
    ref = ar.tune_layer(Wd, Xd, p)
    torch.cuda.synchronize()
    outs = [_outputs(c.out, c.inn, p) for _ in range(2)]
    # two calls in a row: the array keeps the previous call's contents
    mem = [_static_call(ar, Wd, Xd, p, o) for o in outs]
    for o in outs:
        codes, scale, zp, trace, mse = o
        assert torch.equal(codes, ref.codes)
        assert torch.equal(scale, ref.scale)
        assert torch.equal(zp, ref.zero_point)
        assert torch.equal(trace, ref.loss_trace)
        assert torch.equal(mse, ref.final_mse)
    # The second call allocated nothing: the device's free memory and torch's
    # allocated bytes are what the first call left (its outputs were made before).
    assert mem[1] == mem[0]


def test_static_scratch_refuses_oversized_layer(ar):
    out, inn, n = 4096, 4096, 16384
    p = ar.make_params(bits=4, group_size=128, iters=2, batch_rows=16384)
    assert ar.tune_workspace_bytes(out, inn, n, p) > ar.lib_static_scratch_bytes()
    codes = torch.zeros(1, dtype=torch.uint8, device="cuda")
    dummy = ctypes.c_void_p(codes.data_ptr())
    st = ar.lib.ar_tune_layer_static(dummy, ar.AR_BF16, out, inn, dummy, n, ctypes.byref(p), dummy, dummy,
                                     dummy, None, None, ar._stream(None))
    assert st == ar.AR_ENOMEM
    assert int(codes.item()) == 0
