"""Layer-by-layer tuning of a LLaMA-style decoder block, each layer on the output of
the already quantised layers before it.

"[llm-compressor] AutoRound ...", "enable_quanted_input 모드": with quant-aware
calibration the input of a layer is the previous layer's quantised output, so the
quantisation error that accumulates through the block is what later layers are
tuned against; "on_event with SEQUENTIAL_EPOCH_END" walks a subgraph's linear
layers one at a time.  The pages show no attention arithmetic, so the block is
read as its linear data flow (single-key attention mixes nothing):

    q, k, v  tuned on x0
    o        tuned on v'(x0)
    gate, up tuned on h = x0 + o'(v'(x0))       (residual, no norm)
    down     tuned on silu(gate'(h)) * up'(h)

where L'(x) = x W'^T with W' = s*(q - zp) the layer's tuned fake-quantised weight.
Every layer's target is the full-precision output of the same layer on the same
input (the residual form of the tuning loss).  All arithmetic runs in libar
(ar_tune_layer, ar_dequant, ar_linear, ar_silu_mul); this module only sequences
the calls.
"""
from __future__ import annotations

import torch

from . import TuneParams, TuneTiming, dequant, linear, silu_mul, tune_layer, tune_workspace_bytes

BLOCK_LAYERS = ("q_proj", "k_proj", "v_proj", "o_proj", "gate_proj", "up_proj", "down_proj")


def block_workspace_bytes(weights: dict, n_rows: int, params: TuneParams) -> int:
    return max(tune_workspace_bytes(w.shape[0], w.shape[1], n_rows, params) for w in weights.values())


def tune_block(x0: torch.Tensor, weights: dict, params: TuneParams, workspace: torch.Tensor | None = None,
               keep_inputs: bool = False, timings: list | None = None):
    """Tune the seven projections of one block in order.

    x0: [n, hidden] bf16 calibration activations; weights: name -> [out, in] bf16 W.
    Returns (results: name -> TuneResult, inputs: name -> the activations the layer
    was tuned on, when keep_inputs).  With ``timings`` (a list) the timed variant of
    ar_tune_layer runs and appends one TuneTiming per layer.
    """
    if workspace is None:
        workspace = torch.empty(block_workspace_bytes(weights, x0.shape[0], params), dtype=torch.uint8,
                                device=x0.device)
    g = params.group_size
    results, inputs = {}, {}

    def tune(name, x):
        t = TuneTiming() if timings is not None else None
        r = tune_layer(weights[name], x, params, workspace=workspace, want_final_mse=False, timing=t)
        if timings is not None:
            timings.append(t)
        results[name] = r
        if keep_inputs:
            inputs[name] = x
        return r

    def quantised(name):
        r = results[name]
        hi, lo, _ = dequant(r.codes, r.scale, r.zero_point, g)
        return hi, lo

    for name in ("q_proj", "k_proj", "v_proj"):
        tune(name, x0)
    v_out = linear(x0, *quantised("v_proj"))
    tune("o_proj", v_out)
    h = linear(v_out, *quantised("o_proj"), add=x0)
    del v_out
    tune("gate_proj", h)
    tune("up_proj", h)
    a = silu_mul(linear(h, *quantised("gate_proj")), linear(h, *quantised("up_proj")))
    del h
    tune("down_proj", a)
    return results, inputs
