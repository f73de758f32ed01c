"""Host-side failure injection (no GPU needed): the AR_FAULT test hook makes argument
validation or the workspace fail before any CUDA call; the call returns its status,
enqueues nothing, and the next call without the hook behaves as before."""
import ctypes

import pytest


@pytest.fixture(scope="module")
def ar():
    import signed_gradient_rounding_b200 as ar
    return ar


def _tune(ar, ws_bytes=1 << 40, **kw):
    dummy = ctypes.c_void_p(4096)
    p = ar.make_params(batch_rows=512, group_size=64, **kw)
    return ar.lib.ar_tune_layer(dummy, 1, 64, 256, dummy, 1024, ctypes.byref(p), None, dummy, ws_bytes,
                                dummy, dummy, dummy, None, None, None)


def test_param_fault(ar, monkeypatch):
    dummy = ctypes.c_void_p(256)
    monkeypatch.setenv("AR_FAULT", "param")
    assert _tune(ar) == ar.AR_EINVAL
    assert ar.lib.ar_pack(dummy, 4, 32, 4, dummy, None) == ar.AR_EINVAL
    assert ar.lib.ar_rtn(dummy, 0, 4, 64, 4, 32, 0, dummy, dummy, dummy, None) == ar.AR_EINVAL
    assert ar.tune_workspace_bytes(64, 256, 1024, ar.make_params(batch_rows=512, group_size=64)) == 0
    monkeypatch.delenv("AR_FAULT")
    # valid arguments get past validation again: a too-small workspace is what fails now
    assert _tune(ar, ws_bytes=1024) == ar.AR_ENOMEM
    assert ar.tune_workspace_bytes(64, 256, 1024, ar.make_params(batch_rows=512, group_size=64)) > 0


def test_alloc_fault(ar, monkeypatch):
    monkeypatch.setenv("AR_FAULT", "alloc")
    assert _tune(ar) == ar.AR_ENOMEM
    host_p = ar.make_params(batch_rows=512, group_size=64)
    dummy = ctypes.c_void_p(4096)
    assert ar.lib.ar_tune_layer_host(dummy, 1, 64, 256, dummy, 1024, ctypes.byref(host_p), dummy, 1 << 40,
                                     dummy, dummy, dummy, None, None, None) == ar.AR_ENOMEM
    monkeypatch.delenv("AR_FAULT")
    # without the hook the library answers as before (the calls with real buffers
    # that then run are in tests/test_gpu_faults.py; the dummy pointers here must
    # never reach a kernel)
    assert _tune(ar, bits=5) == ar.AR_EINVAL
    assert ar.tune_workspace_bytes(64, 256, 1024, ar.make_params(batch_rows=512, group_size=64)) > 0


def test_unknown_fault_name_is_ignored(ar, monkeypatch):
    monkeypatch.setenv("AR_FAULT", "nonsense")
    assert _tune(ar, ws_bytes=1024) == ar.AR_ENOMEM   # the ordinary workspace check


def test_status_strings_cover_the_check_status(ar):
    assert ar.lib.ar_status_string(ar.AR_ECHECK).decode().startswith("AR_ECHECK")


def test_fp_target_gram_limit_and_direct_form(ar):
    """The full-precision-target mode keeps every block's C_b = W M_b in the Gram form;
    for the 8192 x 29568 down_proj with 262144 calibration rows (16 blocks) that would
    need about 80 GB, above the form's 64 GiB limit.  The automatic choice then takes
    the direct form (about 14 GB); an explicit Gram form is refused before any GPU work."""
    fpt = ar.lib.ar_tune_fp_target_workspace_bytes
    auto = ar.make_params(bits=2, group_size=128, iters=200, batch_rows=16384)
    gram = ar.make_params(bits=2, group_size=128, iters=200, batch_rows=16384, algo="gram")
    direct = ar.make_params(bits=2, group_size=128, iters=200, batch_rows=16384, algo="direct")
    ws_auto = fpt(8192, 29568, 262144, ar.AR_BF16, ctypes.byref(auto))
    assert ws_auto == fpt(8192, 29568, 262144, ar.AR_BF16, ctypes.byref(direct))
    assert 0 < ws_auto < 20 * 2**30
    assert fpt(8192, 29568, 262144, ar.AR_BF16, ctypes.byref(gram)) == 0
    assert fpt(4096, 4096, 262144, ar.AR_BF16, ctypes.byref(auto)) > 0       # q_proj: Gram form
    dummy = ctypes.c_void_p(4096)
    st = ar.lib.ar_tune_layer_fp_target(dummy, ar.AR_BF16, 8192, 29568, dummy, dummy, 262144, ctypes.byref(gram),
                                        None, dummy, 1 << 40, dummy, dummy, dummy, None, None, None)
    assert st == ar.AR_EUNSUPPORTED
