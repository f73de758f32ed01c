"""The C-ABI library: loads without a GPU, exports every declared symbol, and its
host-only logic (argument validation, workspace sizing, block schedule) behaves."""
import ctypes
import os
import re

import pytest

import oracle

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def ar():
    import signed_gradient_rounding_b200 as ar
    return ar


def _declared_functions():
    src = open(os.path.join(ROOT, "include", "ar.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(ar_[a-z_]+)\s*\(", src)))


def test_exports_every_declared_symbol(ar):
    declared = _declared_functions()
    assert declared == sorted(ar.EXPORTS)
    lib = ctypes.CDLL(ar.LIB_PATH)
    for name in declared:
        assert hasattr(lib, name), name


def test_version_and_status_strings(ar):
    assert ar.version().startswith("ar ")
    for s in range(6):
        assert ar.lib.ar_status_string(s).decode().startswith("AR_")


def test_argument_validation_needs_no_gpu(ar):
    lib = ar.lib
    dummy = ctypes.c_void_p(256)
    # bad bit width, bad group size, bad pack width: rejected before any CUDA call
    assert lib.ar_rtn(dummy, 0, 4, 64, 5, 32, 0, dummy, dummy, dummy, None) == ar.AR_EINVAL
    assert lib.ar_rtn(dummy, 0, 4, 64, 4, 48, 0, dummy, dummy, dummy, None) == ar.AR_EINVAL
    assert lib.ar_rtn(dummy, 0, 4, 64, 4, 32, 0, None, dummy, dummy, None) == ar.AR_EINVAL
    assert lib.ar_pack(dummy, 4, 10, 3, dummy, None) == ar.AR_EINVAL
    # empty inputs are a no-op
    assert lib.ar_rtn(None, 0, 0, 64, 4, 32, 0, None, None, None, None) == ar.AR_OK
    assert lib.ar_pack(None, 0, 32, 3, None, None) == ar.AR_OK


def test_tune_validation(ar):
    lib = ar.lib
    dummy = ctypes.c_void_p(4096)

    def call(out, inn, n, **kw):
        p = ar.make_params(**kw)
        return lib.ar_tune_layer(dummy, 1, out, inn, dummy, n, ctypes.byref(p), None, dummy, 1 << 40,
                                 dummy, dummy, dummy, None, None, None)

    assert call(64, 256, 1024, batch_rows=512, group_size=64, bits=5) == ar.AR_EINVAL
    assert call(64, 256, 1000, batch_rows=512, group_size=64) == ar.AR_EINVAL         # n % B
    assert call(64, 256, 1024, batch_rows=512, group_size=64, iters=-1) == ar.AR_EINVAL
    assert call(64, 256, 1024, batch_rows=512, group_size=64, lr=-0.1) == ar.AR_EINVAL
    assert call(64, 256, 1024, batch_rows=512, group_size=8) == ar.AR_EUNSUPPORTED    # g < 16
    assert call(64, 288, 1024, batch_rows=512, group_size=24) == ar.AR_EUNSUPPORTED   # g % 16
    assert call(64, 1024, 1024, batch_rows=512, group_size=384) == ar.AR_EINVAL        # in % g
    # groups wider than an epilogue thread's columns (or not dividing 256) are supported
    for inn, g in ((1024, 512), (1024, -1), (288, 96), (768, 384), (4096, -1), (256, 16), (288, 48)):
        p = ar.make_params(batch_rows=512, group_size=g)
        assert ar.tune_workspace_bytes(64, inn, 1024, p) > 0, (inn, g)
    assert call(64, 250, 1024, batch_rows=512, group_size=-1) == ar.AR_EUNSUPPORTED   # in % 32
    assert call(0, 256, 1024, batch_rows=512, group_size=64) == ar.AR_OK              # empty layer
    assert call(64, 256, 1024, batch_rows=512, group_size=64, init=2) == ar.AR_EINVAL  # unknown init
    assert call(64, 256, 1024, batch_rows=512, group_size=64, keep_best=3) == ar.AR_EINVAL  # unknown keep-best
    assert call(64, 256, 1024, batch_rows=512, group_size=64, keep_best=-1) == ar.AR_EINVAL
    assert call(64, 256, 1024, batch_rows=512, group_size=64, split=3) == ar.AR_EINVAL
    # the chunked accumulation (split = 2): the plain Gram step with narrow groups only
    assert call(64, 256, 1024, batch_rows=512, group_size=64, split=2, algo="direct") == ar.AR_EUNSUPPORTED
    assert call(64, 1024, 1024, batch_rows=512, group_size=512, split=2, algo="gram") == ar.AR_EUNSUPPORTED
    assert ar.make_params(keep_best="layer").keep_best == ar.AR_KEEP_BEST_LAYER
    assert ar.make_params(keep_best=True).keep_best == ar.AR_KEEP_BEST_ROW
    assert ar.make_params(keep_best="last").keep_best == ar.AR_KEEP_LAST
    # too small a workspace
    p = ar.make_params(batch_rows=512, group_size=64)
    assert lib.ar_tune_layer(dummy, 1, 64, 256, dummy, 1024, ctypes.byref(p), None, dummy, 1024,
                             dummy, dummy, dummy, None, None, None) == ar.AR_ENOMEM


def test_workspace_bytes(ar):
    p = ar.make_params(batch_rows=16384, group_size=128, algo="direct")
    ws = ar.tune_workspace_bytes(4096, 4096, 262144, p)
    # R^T as a bf16 pair, D as a pair, V and V_best; X is read in place (no X^T copy)
    assert ws >= 2 * 4096 * 16384 * 2 + 4096 * 4096 * (4 + 4 + 4)
    assert ws < 262144 * 4096 * 2 / 2
    g = ar.make_params(batch_rows=16384, group_size=128, algo="gram")
    wg = ar.tune_workspace_bytes(4096, 4096, 262144, g)
    assert wg >= 16 * 4096 * 4096 * 4                           # 16 Gram matrices as pairs
    assert wg < 16 * 4096 * 4096 * 4 + 262144 * 4096 * 2 / 2
    # auto picks the Gram form for a 4096 x 4096 layer, the direct one for the 72B down_proj
    assert ar.tune_workspace_bytes(4096, 4096, 262144, ar.make_params(batch_rows=16384)) == wg
    wide = ar.make_params(batch_rows=16384, bits=2)
    assert ar.tune_workspace_bytes(8192, 29568, 262144, wide) == \
        ar.tune_workspace_bytes(8192, 29568, 262144, ar.make_params(batch_rows=16384, bits=2, algo="direct"))
    assert ar.tune_workspace_bytes(4096, 4096, 262143, p) == 0
    bad = ar.make_params(batch_rows=16384, group_size=100)
    assert ar.tune_workspace_bytes(4096, 4096, 262144, bad) == 0


@pytest.mark.parametrize("n_blocks,seed", [(16, 0), (16, 123), (3, 7), (1, 0), (97, 2 ** 63 + 5)])
def test_block_schedule_matches_oracle(ar, n_blocks, seed):
    total = 5 * n_blocks + 3
    assert ar.block_schedule(n_blocks, 0, total, seed) == oracle.block_schedule(n_blocks, total, seed)
    first = min(11, total // 2)
    assert ar.block_schedule(n_blocks, first, total - first, seed) == \
        oracle.block_schedule(n_blocks, total, seed)[first:]


def test_host_entry_validation(ar):
    """ar_tune_layer_host checks its arguments before it creates a stream or copies."""
    lib = ar.lib
    dummy = ctypes.c_void_p(4096)
    p = ar.make_params(batch_rows=512, group_size=64)
    need = lib.ar_tune_host_workspace_bytes(64, 256, 1024, 1, ctypes.byref(p))
    assert need > lib.ar_tune_workspace_bytes(64, 256, 1024, ctypes.byref(p)) + 64 * 256 * 2 + 1024 * 256 * 2
    assert lib.ar_tune_host_workspace_bytes(64, 256, 1024, 7, ctypes.byref(p)) == 0      # bad W dtype

    def call(out, inn, n, ws_bytes=1 << 40, W=dummy, codes=dummy, **kw):
        q = ar.make_params(**kw)
        return lib.ar_tune_layer_host(W, 1, out, inn, dummy, n, ctypes.byref(q), dummy, ws_bytes,
                                      codes, dummy, dummy, None, None, None)

    assert call(64, 256, 1024, batch_rows=512, group_size=64, bits=5) == ar.AR_EINVAL
    assert call(64, 256, 1000, batch_rows=512, group_size=64) == ar.AR_EINVAL
    assert call(64, 256, 1024, W=None, batch_rows=512, group_size=64) == ar.AR_EINVAL
    assert call(64, 256, 1024, codes=None, batch_rows=512, group_size=64) == ar.AR_EINVAL
    assert call(64, 256, 1024, batch_rows=512, group_size=8) == ar.AR_EUNSUPPORTED
    assert call(64, 256, 1024, ws_bytes=need - 1, batch_rows=512, group_size=64) == ar.AR_ENOMEM
    assert call(0, 256, 1024, batch_rows=512, group_size=64) == ar.AR_OK


def test_fp_target_validation(ar):
    lib = ar.lib
    dummy = ctypes.c_void_p(4096)
    p = ar.make_params(batch_rows=512, group_size=64)
    need = lib.ar_tune_fp_target_workspace_bytes(64, 256, 1024, 1, ctypes.byref(p))
    assert need > lib.ar_tune_workspace_bytes(64, 256, 1024, ctypes.byref(p))
    q = ar.make_params(batch_rows=512, group_size=64, algo="direct")
    # the direct form holds E_b^T = W dX_b^T of every block ([out, n] as a bf16 pair)
    assert lib.ar_tune_fp_target_workspace_bytes(64, 256, 1024, 1, ctypes.byref(q)) >= \
        lib.ar_tune_workspace_bytes(64, 256, 1024, ctypes.byref(q)) + 64 * 1024 * 4

    def call(Xt=dummy, params=p):
        return lib.ar_tune_layer_fp_target(dummy, 1, 64, 256, dummy, Xt, 1024, ctypes.byref(params), None, dummy,
                                           1 << 40, dummy, dummy, dummy, None, None, None)

    assert call(Xt=None) == ar.AR_EINVAL
    assert call(params=ar.make_params(batch_rows=512, group_size=64, bits=5)) == ar.AR_EINVAL
