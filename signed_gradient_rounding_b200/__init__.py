"""Python binding of libar: AutoRound per-layer SignSGD tuning on one B200.

Argument marshalling only: every step of the computation runs in libar's CUDA
kernels (``libar.so``, built in-tree by ``python signed_gradient_rounding_b200/build.py``).
PyTorch provides device memory and streams.  Importing this package fails
loudly when the library is missing; there is no CPU fallback.

Entry points (same names as the C ABI in include/ar.h):
  rtn, fake_quant, pack, tune_workspace_bytes, tune_layer, tune_status,
  and tune_layer_host (host arrays in and out, the copies included).
"""
from __future__ import annotations

import ctypes
import dataclasses
import os

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libar.so")

AR_OK, AR_EINVAL, AR_EUNSUPPORTED, AR_ENOMEM, AR_ECUDA, AR_ETIMEOUT, AR_ECHECK = range(7)
AR_F32, AR_BF16 = 0, 1
AR_ALGO_AUTO, AR_ALGO_DIRECT, AR_ALGO_GRAM = 0, 1, 2
ALGOS = {"auto": AR_ALGO_AUTO, "direct": AR_ALGO_DIRECT, "gram": AR_ALGO_GRAM}
AR_INIT_MINMAX, AR_INIT_MSE = 0, 1
INITS = {"minmax": AR_INIT_MINMAX, "mse": AR_INIT_MSE}
AR_KEEP_LAST, AR_KEEP_BEST_ROW, AR_KEEP_BEST_LAYER = 0, 1, 2
KEEPS = {"last": AR_KEEP_LAST, "row": AR_KEEP_BEST_ROW, "layer": AR_KEEP_BEST_LAYER}

# Every exported symbol of include/ar.h.
EXPORTS = ("ar_version", "ar_status_string", "ar_rtn", "ar_fake_quant", "ar_pack",
           "ar_tune_workspace_bytes", "ar_tune_layer", "ar_tune_layer_timed", "ar_block_schedule",
           "ar_tune_host_workspace_bytes", "ar_tune_layer_host", "ar_tune_fp_target_workspace_bytes",
           "ar_tune_layer_fp_target", "ar_selftest_division",
           "ar_tune_status", "ar_tune_row_losses", "ar_selftest_timeout", "ar_tune_layer_static", "ar_static_scratch_bytes", "ar_dequant", "ar_linear",
           "ar_silu_mul")


class ArError(RuntimeError):
    def __init__(self, status: int, what: str):
        self.status = status
        super().__init__(f"{what}: {_lib.ar_status_string(status).decode()}")


class TuneParams(ctypes.Structure):
    _fields_ = [("bits", ctypes.c_int32), ("group_size", ctypes.c_int32), ("sym", ctypes.c_int32),
                ("iters", ctypes.c_int32), ("lr", ctypes.c_float), ("minmax_lr", ctypes.c_float),
                ("minmax_shrink", ctypes.c_float), ("keep_best", ctypes.c_int32),
                ("batch_rows", ctypes.c_int64), ("seed", ctypes.c_uint64), ("start_step", ctypes.c_int64),
                ("algo", ctypes.c_int32), ("split", ctypes.c_int32), ("init", ctypes.c_int32)]


class _TuneStateC(ctypes.Structure):
    _fields_ = [("V", ctypes.c_void_p), ("alpha", ctypes.c_void_p), ("beta", ctypes.c_void_p),
                ("best_loss", ctypes.c_void_p), ("V_best", ctypes.c_void_p),
                ("alpha_best", ctypes.c_void_p), ("beta_best", ctypes.c_void_p),
                ("initialized", ctypes.c_int32)]


class TuneTiming(ctypes.Structure):
    _fields_ = [("residual_ms", ctypes.c_float), ("update_ms", ctypes.c_float), ("total_ms", ctypes.c_float),
                ("gemm_launches", ctypes.c_int32), ("kernel_launches", ctypes.c_int32), ("algo", ctypes.c_int32),
                ("setup_ms", ctypes.c_float)]


def _load() -> ctypes.CDLL:
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"{LIB_PATH} is missing; build it with "
                          "`python signed_gradient_rounding_b200/build.py`")
    lib = ctypes.CDLL(LIB_PATH)
    P, I32, I64, U64, SZ = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64, ctypes.c_uint64, ctypes.c_size_t
    lib.ar_version.restype = ctypes.c_char_p
    lib.ar_version.argtypes = []
    lib.ar_status_string.restype = ctypes.c_char_p
    lib.ar_status_string.argtypes = [ctypes.c_int]
    lib.ar_rtn.restype = ctypes.c_int
    lib.ar_rtn.argtypes = [P, ctypes.c_int, I64, I64, I32, I32, I32, P, P, P, P]
    lib.ar_fake_quant.restype = ctypes.c_int
    lib.ar_fake_quant.argtypes = [P, ctypes.c_int, I64, I64, P, P, P, I32, I32, I32, P, P, P, P, P]
    lib.ar_pack.restype = ctypes.c_int
    lib.ar_pack.argtypes = [P, I64, I64, I32, P, P]
    lib.ar_tune_workspace_bytes.restype = SZ
    lib.ar_tune_workspace_bytes.argtypes = [I64, I64, I64, ctypes.POINTER(TuneParams)]
    lib.ar_tune_layer.restype = ctypes.c_int
    lib.ar_tune_layer.argtypes = [P, ctypes.c_int, I64, I64, P, I64, ctypes.POINTER(TuneParams),
                                  ctypes.POINTER(_TuneStateC), P, SZ, P, P, P, P, P, P]
    lib.ar_tune_layer_timed.restype = ctypes.c_int
    lib.ar_tune_layer_timed.argtypes = lib.ar_tune_layer.argtypes + [ctypes.POINTER(TuneTiming)]
    lib.ar_tune_fp_target_workspace_bytes.restype = SZ
    lib.ar_tune_fp_target_workspace_bytes.argtypes = [I64, I64, I64, ctypes.c_int, ctypes.POINTER(TuneParams)]
    lib.ar_tune_layer_fp_target.restype = ctypes.c_int
    lib.ar_tune_layer_fp_target.argtypes = [P, ctypes.c_int, I64, I64, P, P, I64, ctypes.POINTER(TuneParams),
                                            ctypes.POINTER(_TuneStateC), P, SZ, P, P, P, P, P, P]
    lib.ar_tune_host_workspace_bytes.restype = SZ
    lib.ar_tune_host_workspace_bytes.argtypes = [I64, I64, I64, ctypes.c_int, ctypes.POINTER(TuneParams)]
    lib.ar_tune_layer_host.restype = ctypes.c_int
    lib.ar_tune_layer_host.argtypes = [P, ctypes.c_int, I64, I64, P, I64, ctypes.POINTER(TuneParams), P, SZ,
                                       P, P, P, P, P, P]
    lib.ar_block_schedule.restype = ctypes.c_int
    lib.ar_block_schedule.argtypes = [I64, I64, I64, U64, P]
    lib.ar_tune_layer_static.restype = ctypes.c_int
    lib.ar_tune_layer_static.argtypes = [P, ctypes.c_int, I64, I64, P, I64, ctypes.POINTER(TuneParams),
                                         P, P, P, P, P, P]
    lib.ar_static_scratch_bytes.restype = SZ
    lib.ar_static_scratch_bytes.argtypes = []
    lib.ar_dequant.restype = ctypes.c_int
    lib.ar_dequant.argtypes = [P, P, P, I64, I64, I32, P, P, P, P]
    lib.ar_linear.restype = ctypes.c_int
    lib.ar_linear.argtypes = [P, I64, I64, P, P, I64, P, P, P, P]
    lib.ar_silu_mul.restype = ctypes.c_int
    lib.ar_silu_mul.argtypes = [P, P, I64, P, P]
    lib.ar_tune_status.restype = ctypes.c_int
    lib.ar_tune_status.argtypes = [P, P]
    lib.ar_tune_row_losses.restype = ctypes.c_int
    lib.ar_tune_row_losses.argtypes = [P, SZ, I64, I64, I64, ctypes.POINTER(TuneParams), P, P]
    lib.ar_selftest_division.restype = ctypes.c_int
    lib.ar_selftest_division.argtypes = [P, I64, P, I64, P, P, P]
    lib.ar_selftest_timeout.restype = ctypes.c_int
    lib.ar_selftest_timeout.argtypes = [P, U64, P]
    return lib


_lib = _load()
lib = _lib


def version() -> str:
    return _lib.ar_version().decode()


def lib_static_scratch_bytes() -> int:
    """Size of the fixed device scratch of ar_tune_layer_static, as the library was built."""
    return int(_lib.ar_static_scratch_bytes())


def _check(status: int, what: str) -> None:
    if status != AR_OK:
        raise ArError(status, what)


def _ptr(t: torch.Tensor | None):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream) -> ctypes.c_void_p:
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def _dev(t: torch.Tensor, name: str, dtype=None) -> torch.Tensor:
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if dtype is not None and t.dtype != dtype:
        raise ValueError(f"{name} must be {dtype}")
    return t


def _wdtype(W: torch.Tensor) -> int:
    if W.dtype == torch.float32:
        return AR_F32
    if W.dtype == torch.bfloat16:
        return AR_BF16
    raise ValueError("W must be float32 or bfloat16")


def _groups(inn: int, group_size: int) -> int:
    g = inn if group_size == -1 else group_size
    return inn // g if g > 0 and inn % g == 0 else 0


def rtn(W: torch.Tensor, bits: int, group_size: int, sym: bool = False, stream=None):
    """Round-to-nearest codes (uint8 [out, in]), scales (fp32 [out, G]), zero-points (int32 [out, G])."""
    _dev(W, "W")
    out, inn = W.shape
    G = max(_groups(inn, group_size), 1)
    codes = torch.empty((out, inn), dtype=torch.uint8, device=W.device)
    scale = torch.empty((out, G), dtype=torch.float32, device=W.device)
    zp = torch.empty((out, G), dtype=torch.int32, device=W.device)
    _check(_lib.ar_rtn(_ptr(W), _wdtype(W), out, inn, bits, group_size, int(sym), _ptr(codes), _ptr(scale),
                       _ptr(zp), _stream(stream)), "ar_rtn")
    return codes, scale, zp


def fake_quant(W, V, alpha, beta, bits: int, group_size: int, sym: bool = False, want_wq=True, stream=None):
    """Offset fake-quantisation: (codes, scale, zp, Wq fp32 or None)."""
    _dev(W, "W")
    out, inn = W.shape
    for t, n in ((V, "V"), (alpha, "alpha"), (beta, "beta")):
        _dev(t, n, torch.float32)
    G = max(_groups(inn, group_size), 1)
    codes = torch.empty((out, inn), dtype=torch.uint8, device=W.device)
    scale = torch.empty((out, G), dtype=torch.float32, device=W.device)
    zp = torch.empty((out, G), dtype=torch.int32, device=W.device)
    Wq = torch.empty((out, inn), dtype=torch.float32, device=W.device) if want_wq else None
    _check(_lib.ar_fake_quant(_ptr(W), _wdtype(W), out, inn, _ptr(V), _ptr(alpha), _ptr(beta), bits,
                              group_size, int(sym), _ptr(codes), _ptr(scale), _ptr(zp), _ptr(Wq),
                              _stream(stream)), "ar_fake_quant")
    return codes, scale, zp, Wq


def pack(codes: torch.Tensor, bits: int, stream=None) -> torch.Tensor:
    """int32 [rows, cols*bits/32]: each row one little-endian bit stream of b-bit codes."""
    _dev(codes, "codes", torch.uint8)
    rows, cols = codes.shape
    packed = torch.empty((rows, cols * bits // 32), dtype=torch.int32, device=codes.device)
    _check(_lib.ar_pack(_ptr(codes), rows, cols, bits, _ptr(packed), _stream(stream)), "ar_pack")
    return packed


def dequant(codes: torch.Tensor, scale: torch.Tensor, zp: torch.Tensor, group_size: int, want_lo: bool = True,
            want_f32: bool = False, stream=None):
    """W' = s*(q - zp): (bf16 hi, bf16 lo or None, fp32 or None), each [out, in]."""
    _dev(codes, "codes", torch.uint8)
    out, inn = codes.shape
    hi = torch.empty((out, inn), dtype=torch.bfloat16, device=codes.device)
    lo = torch.empty_like(hi) if want_lo else None
    f32 = torch.empty((out, inn), dtype=torch.float32, device=codes.device) if want_f32 else None
    _check(_lib.ar_dequant(_ptr(codes), _ptr(scale), _ptr(zp), out, inn, group_size, _ptr(hi), _ptr(lo),
                           _ptr(f32), _stream(stream)), "ar_dequant")
    return hi, lo, f32


def linear(X: torch.Tensor, Wq_hi: torch.Tensor, Wq_lo: torch.Tensor | None = None,
           add: torch.Tensor | None = None, out: torch.Tensor | None = None, status: torch.Tensor | None = None,
           stream=None) -> torch.Tensor:
    """bf16(X (Wq_hi + Wq_lo)^T + add) on the tensor cores: X [n, in] bf16, Wq [out, in] bf16."""
    _dev(X, "X", torch.bfloat16)
    _dev(Wq_hi, "Wq_hi", torch.bfloat16)
    n, inn = X.shape
    o = Wq_hi.shape[0]
    Y = out if out is not None else torch.empty((n, o), dtype=torch.bfloat16, device=X.device)
    _check(_lib.ar_linear(_ptr(X), n, inn, _ptr(Wq_hi), _ptr(Wq_lo), o, _ptr(add), _ptr(Y), _ptr(status),
                          _stream(stream)), "ar_linear")
    return Y


def silu_mul(a: torch.Tensor, b: torch.Tensor, stream=None) -> torch.Tensor:
    """bf16(silu(a) * b) elementwise on bf16 tensors."""
    _dev(a, "a", torch.bfloat16)
    _dev(b, "b", torch.bfloat16)
    y = torch.empty_like(a)
    _check(_lib.ar_silu_mul(_ptr(a), _ptr(b), a.numel(), _ptr(y), _stream(stream)), "ar_silu_mul")
    return y


def make_params(bits=4, group_size=128, sym=False, iters=200, lr=0.005, minmax_lr=-1.0, minmax_shrink=1.0,
                keep_best=True, batch_rows=16384, seed=0, start_step=0, algo="auto", split=True,
                init="minmax") -> TuneParams:
    """ar_tune_params; algo is "auto", "direct" or "gram" (ar_algo in include/ar.h);
    init is "minmax" or "mse" (ar_init); keep_best is True / "row", False / "last" or
    "layer" (ar_keep_best)."""
    keep = KEEPS[keep_best] if isinstance(keep_best, str) else int(keep_best)
    return TuneParams(bits, group_size, int(sym), iters, lr, minmax_lr, minmax_shrink, keep,
                      batch_rows, seed, start_step, ALGOS[algo] if isinstance(algo, str) else int(algo),
                      int(split), INITS[init] if isinstance(init, str) else int(init))


def tune_workspace_bytes(out: int, inn: int, n_rows: int, params: TuneParams) -> int:
    return int(_lib.ar_tune_workspace_bytes(out, inn, n_rows, ctypes.byref(params)))


@dataclasses.dataclass
class TuneState:
    """Caller-owned tuning state on the device (see ar_tune_state)."""

    V: torch.Tensor
    alpha: torch.Tensor
    beta: torch.Tensor
    best_loss: torch.Tensor
    V_best: torch.Tensor
    alpha_best: torch.Tensor
    beta_best: torch.Tensor
    initialized: bool = False

    @classmethod
    def empty(cls, out: int, inn: int, group_size: int, device="cuda") -> "TuneState":
        G = max(_groups(inn, group_size), 1)
        f = dict(dtype=torch.float32, device=device)
        return cls(torch.empty((out, inn), **f), torch.empty((out, G), **f), torch.empty((out, G), **f),
                   torch.empty((out,), **f), torch.empty((out, inn), **f), torch.empty((out, G), **f),
                   torch.empty((out, G), **f))

    def _c(self) -> _TuneStateC:
        return _TuneStateC(self.V.data_ptr(), self.alpha.data_ptr(), self.beta.data_ptr(),
                           self.best_loss.data_ptr(), self.V_best.data_ptr(), self.alpha_best.data_ptr(),
                           self.beta_best.data_ptr(), int(self.initialized))


@dataclasses.dataclass
class TuneResult:
    codes: torch.Tensor
    scale: torch.Tensor
    zero_point: torch.Tensor
    loss_trace: torch.Tensor | None
    final_mse: torch.Tensor | None   # 1-element float64 tensor on the device
    workspace: torch.Tensor


def block_schedule(n_blocks: int, first: int, count: int, seed: int) -> list[int]:
    """The calibration-block index of steps first .. first+count-1 (host computation)."""
    buf = (ctypes.c_int64 * max(count, 1))()
    _check(_lib.ar_block_schedule(n_blocks, first, count, seed, ctypes.cast(buf, ctypes.c_void_p)),
           "ar_block_schedule")
    return [int(buf[i]) for i in range(count)]


def tune_layer(W: torch.Tensor, X: torch.Tensor, params: TuneParams, state: TuneState | None = None,
               workspace: torch.Tensor | None = None, want_loss_trace: bool = True,
               want_final_mse: bool = True, outputs=None, stream=None, timing: TuneTiming | None = None
               ) -> TuneResult:
    """Run ar_tune_layer on device tensors.  W fp32/bf16 [out, in]; X bf16 [n_rows, in].

    ``outputs`` may pass preallocated (codes, scale, zp, loss_trace, final_mse)
    tensors so that repeated calls allocate nothing.  With ``timing`` the timed
    variant runs (synchronising the stream) and fills it.
    """
    _dev(W, "W")
    _dev(X, "X", torch.bfloat16)
    out, inn = W.shape
    n_rows = X.shape[0]
    if X.shape[1] != inn:
        raise ValueError("X must be [n_rows, in]")
    need = tune_workspace_bytes(out, inn, n_rows, params)
    if need == 0:
        raise ArError(AR_EINVAL, "ar_tune_workspace_bytes")
    if workspace is None:
        workspace = torch.empty(need, dtype=torch.uint8, device=W.device)
    G = max(_groups(inn, params.group_size), 1)
    if outputs is None:
        codes = torch.empty((out, inn), dtype=torch.uint8, device=W.device)
        scale = torch.empty((out, G), dtype=torch.float32, device=W.device)
        zp = torch.empty((out, G), dtype=torch.int32, device=W.device)
        trace = torch.empty((max(params.iters, 1),), dtype=torch.float32, device=W.device) if want_loss_trace else None
        mse = torch.empty((1,), dtype=torch.float64, device=W.device) if want_final_mse else None
    else:
        codes, scale, zp, trace, mse = outputs
    st = ctypes.byref(state._c()) if state is not None else None
    args = (_ptr(W), _wdtype(W), out, inn, _ptr(X), n_rows, ctypes.byref(params), st, _ptr(workspace),
            workspace.numel(), _ptr(codes), _ptr(scale), _ptr(zp), _ptr(trace), _ptr(mse), _stream(stream))
    if timing is None:
        _check(_lib.ar_tune_layer(*args), "ar_tune_layer")
    else:
        _check(_lib.ar_tune_layer_timed(*args, ctypes.byref(timing)), "ar_tune_layer_timed")
    if state is not None:
        state.initialized = True
    return TuneResult(codes, scale, zp, trace[:params.iters] if trace is not None else None, mse, workspace)


def tune_layer_fp_target(W: torch.Tensor, X: torch.Tensor, X_target: torch.Tensor, params: TuneParams,
                         workspace: torch.Tensor | None = None, want_final_mse: bool = True,
                         stream=None, state: TuneState | None = None) -> TuneResult:
    """ar_tune_layer_fp_target on device tensors: the layer sees X (its input on the
    quantised path) and is tuned against the full-precision output X_target W^T.
    ``state`` as for tune_layer (inspection and resume)."""
    _dev(W, "W")
    _dev(X, "X", torch.bfloat16)
    _dev(X_target, "X_target", torch.bfloat16)
    out, inn = W.shape
    n_rows = X.shape[0]
    if X.shape != (n_rows, inn) or X_target.shape != X.shape:
        raise ValueError("X and X_target must be [n_rows, in]")
    wdt = _wdtype(W)
    need = int(_lib.ar_tune_fp_target_workspace_bytes(out, inn, n_rows, wdt, ctypes.byref(params)))
    if need == 0:
        raise ArError(AR_EUNSUPPORTED, "ar_tune_fp_target_workspace_bytes")
    if workspace is None or workspace.numel() < need:
        workspace = torch.empty(need, dtype=torch.uint8, device=W.device)
    G = max(_groups(inn, params.group_size), 1)
    codes = torch.empty((out, inn), dtype=torch.uint8, device=W.device)
    scale = torch.empty((out, G), dtype=torch.float32, device=W.device)
    zp = torch.empty((out, G), dtype=torch.int32, device=W.device)
    trace = torch.empty((max(params.iters, 1),), dtype=torch.float32, device=W.device)
    mse = torch.empty((1,), dtype=torch.float64, device=W.device) if want_final_mse else None
    st = ctypes.byref(state._c()) if state is not None else None
    _check(_lib.ar_tune_layer_fp_target(_ptr(W), wdt, out, inn, _ptr(X), _ptr(X_target), n_rows,
                                        ctypes.byref(params), st, _ptr(workspace), workspace.numel(),
                                        _ptr(codes), _ptr(scale), _ptr(zp), _ptr(trace), _ptr(mse),
                                        _stream(stream)), "ar_tune_layer_fp_target")
    if state is not None:
        state.initialized = True
    return TuneResult(codes, scale, zp, trace[:params.iters], mse, workspace)


def tune_row_losses(workspace: torch.Tensor, out: int, inn: int, n_rows: int, params: TuneParams,
                    stream=None) -> torch.Tensor:
    """Per-row batch losses of the last tune_layer call on ``workspace`` (same sizes and
    params): fp32 [iters, out], the sum over the step's block rows of R_bj^2."""
    dst = torch.empty((max(params.iters, 1), out), dtype=torch.float32, device=workspace.device)
    _check(_lib.ar_tune_row_losses(_ptr(workspace), workspace.numel(), out, inn, n_rows, ctypes.byref(params),
                                   _ptr(dst), _stream(stream)), "ar_tune_row_losses")
    return dst[:params.iters]


def tune_status(workspace: torch.Tensor, stream=None) -> int:
    """Device status of the last tuning call on this workspace (synchronises the stream)."""
    return int(_lib.ar_tune_status(_ptr(workspace), _stream(stream)))


def tune_layer_host(W, X, params: TuneParams, device="cuda", want_final_mse: bool = True, workspace=None,
                    stream=None):
    """Host arrays in, host arrays out, through ar_tune_layer_host: X goes to the
    device block by block, overlapped with the work.  W: fp32 or bf16 CPU tensor;
    X: bf16 CPU tensor [n_rows, in] (page-locked memory lets the copies overlap;
    other memory is pinned here first, which costs a host copy).  ``workspace`` may
    pass a device uint8 tensor of tune_host_workspace_bytes() bytes to reuse."""
    if W.device.type != "cpu" or X.device.type != "cpu":
        raise ValueError("tune_layer_host takes CPU tensors")
    if X.dtype != torch.bfloat16:
        raise TypeError("X must be bf16")
    W = W.contiguous()
    X = X.contiguous()
    if not X.is_pinned():
        X = X.pin_memory()
    if not W.is_pinned():
        W = W.pin_memory()
    out, inn = W.shape
    n_rows = X.shape[0]
    if X.shape[1] != inn:
        raise ValueError("X must be [n_rows, in]")
    wdt = _wdtype(W)
    need = tune_host_workspace_bytes(out, inn, n_rows, params, wdt)
    if need == 0:
        raise ArError(AR_EINVAL, "ar_tune_host_workspace_bytes")
    if workspace is None or workspace.numel() < need:
        workspace = torch.empty(need, dtype=torch.uint8, device=device)
    G = max(_groups(inn, params.group_size), 1)
    codes = torch.empty((out, inn), dtype=torch.uint8, pin_memory=True)
    scale = torch.empty((out, G), dtype=torch.float32, pin_memory=True)
    zp = torch.empty((out, G), dtype=torch.int32, pin_memory=True)
    trace = torch.empty((max(params.iters, 1),), dtype=torch.float32, pin_memory=True)
    mse = torch.empty((1,), dtype=torch.float64, pin_memory=True) if want_final_mse else None
    with torch.cuda.device(workspace.device):
        _check(_lib.ar_tune_layer_host(_ptr(W), wdt, out, inn, _ptr(X), n_rows, ctypes.byref(params),
                                       _ptr(workspace), workspace.numel(), _ptr(codes), _ptr(scale), _ptr(zp),
                                       _ptr(trace), _ptr(mse), _stream(stream)), "ar_tune_layer_host")
    return dict(codes=codes, scale=scale, zero_point=zp, loss_trace=trace[:params.iters],
                final_mse=float(mse.item()) if mse is not None else None)


def tune_host_workspace_bytes(out: int, inn: int, n_rows: int, params: TuneParams, w_dtype: int = AR_BF16) -> int:
    """Device workspace bytes of tune_layer_host (ar_tune_host_workspace_bytes)."""
    return int(_lib.ar_tune_host_workspace_bytes(out, inn, n_rows, w_dtype, ctypes.byref(params)))
