"""The decoder-block data flow of quant-aware layer-by-layer tuning (oracle side).

TEST INFRASTRUCTURE ONLY (see the package docstring).

"[llm-compressor] AutoRound ...", "enable_quanted_input 모드": each layer is tuned
on the output of the already quantised layers before it; the layer's weight is
replaced by W' = s*(q - zp) ("최종 양자화 적용", ``_fake_quantize_with_offset``).
Reading of the block (the pages show no attention arithmetic): q, k, v take x0;
o takes v'(x0); gate and up take h = x0 + o'(v'(x0)); down takes
silu(gate'(h)) * up'(h).  Activations are stored in bf16 between layers: each
linear output is computed exactly (fp64) and rounded once to bf16.
"""
from __future__ import annotations

import numpy as np

F32 = np.float32


def _bf16_round(x: np.ndarray) -> np.ndarray:
    """Nearest bf16 (ties to even) of fp64 values, via fp32 (exact for |x| in bf16's range
    whenever the fp32 rounding does not itself create a tie; both roundings are to nearest)."""
    x32 = np.asarray(x, dtype=np.float64).astype(np.float32)
    # round the fp64 value directly: pick the nearer of the two bf16 neighbours of x32
    b = x32.view(np.uint32).astype(np.uint64)
    lo = (b >> 16) << 16
    hi = lo + (1 << 16)
    lo_v = lo.astype(np.uint32).view(np.float32).astype(np.float64)
    hi_v = hi.astype(np.uint32).view(np.float32).astype(np.float64)
    x64 = np.asarray(x, dtype=np.float64)
    d_lo = np.abs(x64 - lo_v)
    d_hi = np.abs(hi_v - x64)
    even_lo = ((lo >> 16) & 1) == 0
    pick_hi = (d_hi < d_lo) | ((d_hi == d_lo) & ~even_lo)
    out = np.where(pick_hi, hi, lo).astype(np.uint32).view(np.float32)
    return out


def dequant(codes, scale, zero_point, group_size: int) -> np.ndarray:
    """W' = s*(q - zp) in fp32 (one rounding: q - zp is an exact small integer)."""
    codes = np.asarray(codes)
    out, inn = codes.shape
    g = inn if group_size == -1 else group_size
    s = np.repeat(np.asarray(scale, F32), g, axis=1)
    z = np.repeat(np.asarray(zero_point).astype(F32), g, axis=1)
    return s * (codes.astype(F32) - z)


def linear(X, Wq, add=None) -> np.ndarray:
    """bf16(X Wq^T + add): X bf16-exact values [n, in], Wq fp32 [out, in], add bf16-exact [n, out]."""
    Y = np.asarray(X, np.float64) @ np.asarray(Wq, np.float64).T
    if add is not None:
        Y = Y + np.asarray(add, np.float64)
    return _bf16_round(Y)


def silu_mul(a, b) -> np.ndarray:
    """bf16(silu(a) * b), silu(a) = a / (1 + exp(-a)), evaluated in fp64."""
    a = np.asarray(a, np.float64)
    return _bf16_round(a / (1.0 + np.exp(-a)) * np.asarray(b, np.float64))
