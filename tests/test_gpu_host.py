"""The host-buffer entry point ar_tune_layer_host against ar_tune_layer.

ar_tune_layer_host copies W and X to the device itself (X one calibration block
at a time, overlapped with the work) and runs the same kernels in the same
order as ar_tune_layer on device buffers.  Its results must therefore equal the
device entry point's bit for bit, whatever the host memory (pinned or pageable)
and whatever the evaluation order.  The device entry point is itself checked
against the oracle in test_gpu_parity.py.
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


def _device_run(ar, W, X, p):
    Wd, Xd = W.cuda(), X.cuda()
    res = ar.tune_layer(Wd, Xd, p, want_final_mse=True)
    torch.cuda.synchronize()
    assert ar.tune_status(res.workspace) == ar.AR_OK
    return dict(codes=res.codes.cpu(), scale=res.scale.cpu(), zero_point=res.zero_point.cpu(),
                loss_trace=res.loss_trace.cpu(), final_mse=float(res.final_mse.item()))


def _same(a, b):
    assert torch.equal(a["codes"], b["codes"])
    assert torch.equal(a["scale"], b["scale"])
    assert torch.equal(a["zero_point"], b["zero_point"])
    assert torch.equal(a["loss_trace"], b["loss_trace"])
    assert a["final_mse"] == b["final_mse"]


# (out, in, n_rows, batch_rows, iters, bits, group, algo): one full batch, and
# several blocks visited in shuffled order, with fewer steps than blocks too.
CASES = [
    (TINY.out, TINY.inn, TINY.n_rows, TINY.batch_rows, 12, 4, 64, "gram"),
    (256, 512, 4096, 512, 20, 2, 128, "gram"),
    (256, 512, 4096, 512, 20, 3, 128, "direct"),
    (384, 256, 4096, 1024, 3, 4, 64, "gram"),
]


@pytest.mark.parametrize("case", CASES, ids=lambda c: f"{c[0]}x{c[1]}-n{c[2]}-b{c[3]}-it{c[4]}-{c[7]}")
def test_host_entry_matches_device_entry(ar, case):
    out, inn, n, B, iters, bits, g, algo = case
    W = torch.from_numpy(make_weight(out, inn, 0.02, "bf16", seed=3)).to(torch.bfloat16)
    X = torch.from_numpy(make_activations(n, inn, "llm", seed=4)).to(torch.bfloat16)
    p = ar.make_params(bits=bits, group_size=g, iters=iters, batch_rows=B, algo=algo)
    dev = _device_run(ar, W, X, p)
    host = ar.tune_layer_host(W.pin_memory(), X.pin_memory(), p)
    _same(host, dev)
    # a second call on a reused workspace gives the same again
    ws = torch.empty(ar.tune_host_workspace_bytes(out, inn, n, p), dtype=torch.uint8, device="cuda")
    _same(ar.tune_layer_host(W, X, p, workspace=ws), dev)
    _same(ar.tune_layer_host(W, X, p, workspace=ws), dev)


def test_host_entry_pageable_buffers(ar):
    """Plain (pageable) numpy buffers through the C ABI: the copies are synchronous
    but the results are the same."""
    out, inn, n, B = 128, 256, 2048, 512
    W = torch.from_numpy(make_weight(out, inn, 0.02, "f32", seed=5))
    X = torch.from_numpy(make_activations(n, inn, "llm", seed=6)).to(torch.bfloat16)
    p = ar.make_params(bits=4, group_size=128, iters=10, batch_rows=B)
    dev = _device_run(ar, W, X, p)
    Wn = W.numpy().copy()
    Xn = X.view(torch.int16).numpy().copy()
    G = inn // 128
    codes = np.zeros((out, inn), np.uint8)
    scale = np.zeros((out, G), np.float32)
    zp = np.zeros((out, G), np.int32)
    trace = np.zeros(10, np.float32)
    mse = np.zeros(1, np.float64)
    need = ar.tune_host_workspace_bytes(out, inn, n, p, ar.AR_F32)
    ws = torch.empty(need, dtype=torch.uint8, device="cuda")
    ptr = lambda a: ctypes.c_void_p(a.ctypes.data)
    st = ar._lib.ar_tune_layer_host(ptr(Wn), ar.AR_F32, out, inn, ptr(Xn), n, ctypes.byref(p),
                                    ctypes.c_void_p(ws.data_ptr()), need, ptr(codes), ptr(scale), ptr(zp),
                                    ptr(trace), ptr(mse), ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert st == ar.AR_OK
    _same(dict(codes=torch.from_numpy(codes), scale=torch.from_numpy(scale), zero_point=torch.from_numpy(zp),
               loss_trace=torch.from_numpy(trace), final_mse=float(mse[0])), dev)
    # too small a workspace is refused before any copy
    st = ar._lib.ar_tune_layer_host(ptr(Wn), ar.AR_F32, out, inn, ptr(Xn), n, ctypes.byref(p),
                                    ctypes.c_void_p(ws.data_ptr()), need - 256, ptr(codes), ptr(scale), ptr(zp),
                                    None, None, None)
    assert st == ar.AR_ENOMEM
