"""Seeded synthetic inputs for the AutoRound layer-tuning workloads.

This module draws random weights and calibration activations and nothing
else: it holds none of the tuning method's arithmetic.  Both the CUDA path and
the CPU oracle consume the bytes it produces, so data generation is never
under test.

Shapes and distributions follow the workloads of the AutoRound tuning loop:

* weights ~ N(0, std) with std 0.02 (LLaMA-7B-shaped layers) or 0.015
  (Qwen2.5-72B-shaped down_proj), stored as bf16 (fp32 for the tiny case);
* calibration activations: 128 samples x 2048 tokens = 262144 rows; every
  channel c has its own standard deviation sigma_c = exp(0.5 * z), z ~ N(0, 1)
  (a lognormal(0, 0.5) spread), and round(0.01 * in) seeded channels are
  scaled by 20 (activation outliers); rounded once to bf16;
* the tiny case: 512 x 256 activations ~ N(0, 1) with 4 seeded channels x20.

Every tensor has its own stream id under one seed, so changing one shape does
not change another tensor's values.  Two back-ends exist: numpy's Philox on the
host (small and medium sizes, reproducible on any machine) and torch's CUDA
generator (multi-GB activations for the large layers, generated in place on the
device).  A given test or benchmark always hands the same bytes to both sides.
"""
from __future__ import annotations

import dataclasses

import numpy as np

STREAM_W = 1
STREAM_X = 2
STREAM_SIGMA = 3
STREAM_OUTLIER = 4


def _rng(seed: int, stream: int) -> np.random.Generator:
    return np.random.Generator(np.random.Philox(np.random.SeedSequence([seed, stream])))


def bf16_round(x: np.ndarray) -> np.ndarray:
    """Round float32 values to the nearest bf16 (ties to even); returned as float32."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    b = x.view(np.uint32).astype(np.uint64)
    lsb = (b >> 16) & 1
    b = ((b + 0x7FFF + lsb) >> 16) << 16
    return b.astype(np.uint32).view(np.float32)


def bf16_bits(x: np.ndarray) -> np.ndarray:
    """bf16 bit patterns (uint16) of float32 values that are already bf16-exact."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    return (x.view(np.uint32) >> 16).astype(np.uint16)


def bf16_from_bits(b: np.ndarray) -> np.ndarray:
    return (np.ascontiguousarray(b, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32)


@dataclasses.dataclass(frozen=True)
class LayerWorkload:
    """One linear layer to tune: W is [out, in], X is [n_rows, in]."""

    name: str
    out: int
    inn: int
    n_rows: int
    batch_rows: int
    bits: int
    group_size: int
    sym: bool
    iters: int
    lr: float
    minmax_lr: float
    w_std: float
    w_dtype: str          # "f32" or "bf16"
    x_kind: str           # "tiny" (N(0,1), 4 channels x20) or "llm" (lognormal std, 1% x20)
    seed: int = 0

    @property
    def flops_per_step(self) -> float:
        # two dense contractions of batch_rows x out x in multiply-adds each
        return 4.0 * self.batch_rows * self.out * self.inn


TINY = LayerWorkload("tiny 256x256 W4 g64", 256, 256, 512, 512, 4, 64, False, 50,
                     0.005, 0.005, 0.02, "f32", "tiny")
Q_PROJ_7B = LayerWorkload("llama7b q_proj 4096x4096 W4 g128", 4096, 4096, 262144, 16384,
                          4, 128, False, 200, 0.005, 0.005, 0.02, "bf16", "llm")
# The q_proj layer with only 2 calibration blocks: the same per-step kernel shapes
# on about 1 GB of device memory (for profiler captures that replay kernels).
Q_PROJ_7B_2BLK = LayerWorkload("llama7b q_proj 4096x4096 W4 g128, 2 calibration blocks", 4096, 4096,
                               32768, 16384, 4, 128, False, 200, 0.005, 0.005, 0.02, "bf16", "llm")
DOWN_7B = LayerWorkload("llama7b down_proj 4096x11008 W2 g128", 4096, 11008, 262144, 16384,
                        2, 128, False, 200, 0.005, 0.005, 0.02, "bf16", "llm")
DOWN_72B = LayerWorkload("qwen2.5-72b down_proj 8192x29568 W2 g128", 8192, 29568, 262144, 16384,
                         2, 128, False, 200, 0.005, 0.005, 0.015, "bf16", "llm")

# The LLaMA-7B decoder block, tuned layer by layer (W3, g128, symmetric), each layer on
# the quantised block's activations at its input width (262144 calibration rows).
BLOCK_7B = LayerWorkload("llama7b decoder block (q,k,v,o 4096x4096; gate,up 11008x4096; down 4096x11008) W3 g128 sym",
                         4096, 4096, 262144, 16384, 3, 128, True, 200, 0.005, 0.005, 0.02, "bf16", "llm")
BLOCK_7B_LAYERS = [
    ("q_proj", 4096, 4096), ("k_proj", 4096, 4096), ("v_proj", 4096, 4096),
    ("o_proj", 4096, 4096), ("gate_proj", 11008, 4096), ("up_proj", 11008, 4096),
    ("down_proj", 4096, 11008),
]


def make_weight(out: int, inn: int, std: float, dtype: str = "bf16", seed: int = 0,
                stream: int = STREAM_W) -> np.ndarray:
    """W ~ N(0, std) as float32; bf16-exact values when dtype == 'bf16'."""
    w = _rng(seed, stream).standard_normal((out, inn), dtype=np.float32) * np.float32(std)
    return bf16_round(w) if dtype == "bf16" else w.astype(np.float32)


def outlier_channels(inn: int, count: int, seed: int = 0) -> np.ndarray:
    return np.sort(_rng(seed, STREAM_OUTLIER).permutation(inn)[:count])


def channel_sigma(inn: int, seed: int = 0) -> np.ndarray:
    z = _rng(seed, STREAM_SIGMA).standard_normal(inn)
    return np.exp(0.5 * z).astype(np.float32)


def channel_scale(inn: int, kind: str, seed: int = 0) -> np.ndarray:
    """Per-channel multiplier of the unit-normal activations (float32)."""
    if kind == "tiny":
        scale = np.ones(inn, np.float32)
        scale[outlier_channels(inn, 4, seed)] = 20.0
        return scale
    if kind == "llm":
        scale = channel_sigma(inn, seed)
        scale[outlier_channels(inn, int(round(0.01 * inn)), seed)] *= np.float32(20.0)
        return scale
    raise ValueError(f"unknown activation kind {kind!r}")


def make_activations(n_rows: int, inn: int, kind: str = "llm", seed: int = 0,
                     stream: int = STREAM_X) -> np.ndarray:
    """Host-side calibration activations, bf16-exact float32 [n_rows, inn]."""
    z = _rng(seed, stream).standard_normal((n_rows, inn), dtype=np.float32)
    return bf16_round(z * channel_scale(inn, kind, seed)[None, :])


STREAM_QNOISE = 5


def make_quantised_path_input(X_fp: np.ndarray, rel: float = 0.05, seed: int = 0) -> np.ndarray:
    """Stand-in for a layer's input on the quantised path (the output of layers
    already quantised before it): the full-precision input X_fp with seeded
    multiplicative noise of relative size ``rel``, rounded to bf16.  Used with
    X_fp as the target's input in the quant-aware, full-precision-target mode."""
    z = _rng(seed, STREAM_QNOISE).standard_normal(X_fp.shape, dtype=np.float32)
    return bf16_round(X_fp * (np.float32(1) + np.float32(rel) * z))


def make_activations_cuda(n_rows: int, inn: int, kind: str = "llm", seed: int = 0,
                          stream: int = STREAM_X, device="cuda"):
    """Device-side calibration activations as a torch bf16 tensor [n_rows, inn].

    Uses torch's CUDA generator seeded from (seed, stream); generated in row
    chunks so the fp32 temporary stays small.
    """
    import torch

    gen = torch.Generator(device=device)
    gen.manual_seed(int(np.random.SeedSequence([seed, stream]).generate_state(1)[0]))
    scale = torch.from_numpy(channel_scale(inn, kind, seed)).to(device)
    x = torch.empty((n_rows, inn), dtype=torch.bfloat16, device=device)
    chunk = max(1, (1 << 27) // max(inn, 1))
    for r0 in range(0, n_rows, chunk):
        r1 = min(n_rows, r0 + chunk)
        z = torch.randn((r1 - r0, inn), generator=gen, device=device, dtype=torch.float32)
        x[r0:r1] = (z * scale).to(torch.bfloat16)
    return x
