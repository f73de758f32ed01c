"""Benchmark of the AutoRound layer-tuning hot path on B200.

One benchmark step = one complete ``ar_tune_layer`` call on the LLaMA-7B-shaped
q_proj workload (W 4096x4096 bf16 ~N(0, 0.02), asymmetric W4 g128, 262144 x 4096
bf16 calibration activations with lognormal channel scales and 1% x20 outliers,
16384 rows per SignSGD step, 200 steps, lr = minmax_lr = 0.005), followed by
``ar_pack`` of its codes.  Every row of the hot path runs inside it: min-max
init, the fake-quant prologue, both tensor-core contractions with their fused
epilogues per step, the final codes and the final MSE pass, and packing.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                  [--workload q_proj|tiny|down_7b|down_72b]

Prints one JSON line (rank 0).  Metric: SignSGD steps per second (whole job).
With N GPUs the layer has N times the workload's output rows; each rank tunes
its row shard (shard.row_range) with no exchange in the loop and one all-gather
of the results per step, so the scaling is weak (NCCL; AR_BENCH_BACKEND=gloo runs
the same ranks over gloo, sharing GPUs, to test the path).  Also the layer tune time and
the fraction of the bf16 tensor-core peak.  ``--impl reference`` times the CPU oracle on a
bounded sample of the same workload on the host cores.
"""
from __future__ import annotations

import argparse
import dataclasses
import ctypes
import json
import os
import statistics
import subprocess
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from workloads import (BLOCK_7B, BLOCK_7B_LAYERS, DOWN_7B, DOWN_72B, Q_PROJ_7B, Q_PROJ_7B_2BLK,  # noqa: E402
                       TINY, make_activations, make_activations_cuda, make_weight)

WORKLOADS = {"q_proj": Q_PROJ_7B, "q_proj_2blk": Q_PROJ_7B_2BLK, "tiny": TINY, "down_7b": DOWN_7B,
             "down_72b": DOWN_72B, "block_7b": BLOCK_7B}
METRIC = "signsgd_steps_per_sec"


def _workload(args):
    """The named layer workload, with --group-size applied (-1: one group per row)."""
    c = WORKLOADS[args.workload]
    gs = getattr(args, "group_size", None)
    if gs is None or gs == c.group_size:
        return c
    label = "per-channel" if gs == -1 else f"g{gs}"
    name = c.name.replace(f" g{c.group_size}", f" {label}") if f" g{c.group_size}" in c.name else f"{c.name}, {label}"
    return dataclasses.replace(c, group_size=gs, name=name)
UNIT = "steps/s"


def _peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            d = json.load(f)
        return {"bf16_tflops": d["bf16_tflops"], "bf16_tflops_sustained": d["bf16_tflops_sustained"],
                "hbm_gbs": d["hbm_gbs"], "source": "measured"}
    except (OSError, KeyError, ValueError):
        return {"bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0, "hbm_gbs": 6650.0, "source": "fallback"}


class ClockSampler:
    """nvidia-smi clock and throttle-reason samples while the timed region runs."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.hw_slowdown,"
              "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
              "clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.index = index
        self.proc = None

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.index}", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "100"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None
        return self

    def __exit__(self, *exc):
        self.lines = []
        if self.proc is not None:
            time.sleep(0.25)
            self.proc.terminate()
            try:
                out, _ = self.proc.communicate(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
                out, _ = self.proc.communicate()
            self.lines = [l for l in out.splitlines() if l.strip()]

    def summary(self):
        sm, mx, watts, reasons = [], None, [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in getattr(self, "lines", []):
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 8:
                continue
            try:
                sm.append(float(parts[1]))
                mx = float(parts[2])
            except ValueError:
                continue
            try:
                watts.append(float(parts[3]))
            except ValueError:
                pass
            for name, val in zip(names, parts[4:8]):
                if val.lower() == "active":
                    reasons.add(name)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": mx, "reasons": sorted(reasons),
                "power_w": statistics.median(watts) if watts else None, "samples": len(sm)}


GEMM_SOURCES = ("gemm_sm100.cu", "ar_device.cuh", "ar_internal.h")


def _strip_comments(text: str) -> str:
    """C++ source without // and /* */ comments, indentation, trailing blanks or empty lines."""
    out, i, n = [], 0, len(text)
    while i < n:
        c = text[i]
        if c in "\"'":                                   # string or character literal
            j = i + 1
            while j < n and text[j] != c:
                j += 2 if text[j] == "\\" else 1
            out.append(text[i:j + 1])
            i = j + 1
        elif text.startswith("//", i):
            j = text.find("\n", i)
            i = n if j < 0 else j
        elif text.startswith("/*", i):
            j = text.find("*/", i + 2)
            i = n if j < 0 else j + 2
        else:
            out.append(c)
            i += 1
    lines = (line.strip() for line in "".join(out).splitlines())
    return "\n".join(line for line in lines if line)


def gemm_code_fingerprint() -> str:
    """First 16 hex digits of the sha256 of the GEMM kernel's code (its source and the
    device headers it includes, comments and blank lines removed): the ncu figures in
    profiles/traffic.txt hold while this is unchanged."""
    import hashlib
    h = hashlib.sha256()
    for name in GEMM_SOURCES:
        with open(os.path.join(ROOT, "signed_gradient_rounding_b200", "csrc", name), encoding="utf-8") as f:
            h.update(name.encode() + b"\0" + _strip_comments(f.read()).encode() + b"\0")
    return h.hexdigest()[:16]


def _recorded_traffic(key: str):
    """DRAM bytes per launch from profiles/traffic.txt, if the GEMM code is unchanged."""
    try:
        rec = {}
        for line in open(os.path.join(ROOT, "profiles", "traffic.txt")):
            parts = line.split()
            if len(parts) == 2 and not line.startswith("#"):
                rec[parts[0]] = parts[1]
        if gemm_code_fingerprint() != rec.get("gemm_code_sha256_16"):
            return None
        return int(rec[key]) if key in rec else None
    except (OSError, ValueError):
        return None


def _dist():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return world, rank, local


def run_block(args):
    """The LLaMA-7B decoder block tuned layer by layer, each layer on the quantised
    block's activations; one bench step = the whole block (7 x 200 SignSGD steps)."""
    import torch

    import signed_gradient_rounding_b200 as ar
    from signed_gradient_rounding_b200.block import block_workspace_bytes, tune_block

    world, rank, local = _dist()
    if world > 1:
        raise SystemExit("block_7b runs on one GPU")
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    c = BLOCK_7B
    weights = {name: torch.from_numpy(make_weight(o, i, c.w_std, c.w_dtype, seed=10 + j)).to(torch.bfloat16).to(dev)
               for j, (name, o, i) in enumerate(BLOCK_7B_LAYERS)}
    x0 = make_activations_cuda(c.n_rows, c.inn, c.x_kind, seed=0, device=dev)
    p = ar.make_params(bits=c.bits, group_size=c.group_size, sym=c.sym, iters=c.iters, lr=c.lr,
                       minmax_lr=c.minmax_lr, batch_rows=c.batch_rows, seed=0, algo=args.algo,
                       split=int(args.split))
    ws = torch.empty(block_workspace_bytes(weights, c.n_rows, p), dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream(dev)
    for _ in range(args.warmup):
        tune_block(x0, weights, p, workspace=ws)
    torch.cuda.synchronize()
    timings = []
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with ClockSampler(local) as clk:
        e0.record(stream)
        for _ in range(args.steps):
            tune_block(x0, weights, p, workspace=ws, timings=timings)
        e1.record(stream)
        torch.cuda.synchronize()
    ms = e0.elapsed_time(e1)
    if ar.tune_status(ws) != ar.AR_OK:
        raise RuntimeError("device status not OK after the timed region")
    peaks = _peaks()
    steps_total = len(BLOCK_7B_LAYERS) * c.iters * args.steps
    flops = 0.0
    for (name, o, i), t in zip(BLOCK_7B_LAYERS * args.steps, timings):
        pieces = (3 if t.algo == ar.AR_ALGO_GRAM else 2) if args.split else 1
        flops += c.iters * (pieces * 2.0 * o * i * i if t.algo == ar.AR_ALGO_GRAM
                            else 2 * pieces * 2.0 * c.batch_rows * o * i)
    step_ms = sum(t.residual_ms + t.update_ms for t in timings)
    return {"metric": METRIC, "value": steps_total / (ms / 1e3), "unit": UNIT, "n_gpus": 1,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms / args.steps,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
            "data": "synthetic",
            "config": {"workload": c.name, "layers": [list(x) for x in BLOCK_7B_LAYERS], "n_rows": c.n_rows,
                       "batch_rows": c.batch_rows, "iters_per_layer": c.iters, "bits": c.bits,
                       "group_size": c.group_size, "sym": c.sym, "bench_step": "one whole block (7 layers)",
                       "l2": "inputs larger than L2 (activations 2.1-5.8 GB)"},
            "block_tune_s": ms / args.steps / 1e3,
            "algos": sorted({("gram" if t.algo == ar.AR_ALGO_GRAM else "direct") for t in timings}),
            "fused_step_tflops": flops / (step_ms * 1e-3) / 1e12,
            "tensor_peak_frac": flops / (step_ms * 1e-3) / 1e12 / peaks["bf16_tflops_sustained"],
            "gpu_launches": sum(t.kernel_launches for t in timings) + 5 * args.steps,
            "clocks": clk.summary(), "e2e": None}


def run_fp_target(args):
    """The quant-aware input with a full-precision target (ar_tune_layer_fp_target)
    on one GPU: the layer's input on the quantised path is the target's input with
    5% seeded multiplicative noise.  The whole call is timed with CUDA events."""
    import torch

    import signed_gradient_rounding_b200 as ar

    world, rank, local = _dist()
    if world > 1:
        return None if rank else {"metric": METRIC, "unavailable": "--mode fp_target runs on one GPU"}
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    c = _workload(args)
    W = torch.from_numpy(make_weight(c.out, c.inn, c.w_std, c.w_dtype, seed=0))
    Wd = (W.to(torch.bfloat16) if c.w_dtype == "bf16" else W).to(dev)
    Xt = make_activations_cuda(c.n_rows, c.inn, c.x_kind, seed=0, device=dev)
    gen = torch.Generator(device=dev)
    gen.manual_seed(5)
    Xq = torch.empty_like(Xt)
    chunk = max(1, (1 << 27) // c.inn)
    for r0 in range(0, c.n_rows, chunk):
        r1 = min(c.n_rows, r0 + chunk)
        z = torch.randn((r1 - r0, c.inn), generator=gen, device=dev)
        Xq[r0:r1] = (Xt[r0:r1].float() * (1 + 0.05 * z)).to(torch.bfloat16)
    p = ar.make_params(bits=c.bits, group_size=c.group_size, sym=c.sym, iters=c.iters, lr=c.lr,
                       minmax_lr=c.minmax_lr, batch_rows=c.batch_rows, seed=0, algo=args.algo)
    need = int(ar._lib.ar_tune_fp_target_workspace_bytes(c.out, c.inn, c.n_rows, ar._wdtype(Wd), ctypes.byref(p)))
    if need == 0:
        raise SystemExit("full-precision-target mode: this form does not fit its workspace limit")
    ws = torch.empty(need, dtype=torch.uint8, device=dev)
    for _ in range(args.warmup):
        res = ar.tune_layer_fp_target(Wd, Xq, Xt, p, workspace=ws)
    torch.cuda.synchronize()
    if ar.tune_status(ws) != ar.AR_OK:
        raise RuntimeError("device status not OK after warm-up")
    stream = torch.cuda.current_stream(dev)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with ClockSampler(local) as clk:
        e0.record(stream)
        for _ in range(args.steps):
            res = ar.tune_layer_fp_target(Wd, Xq, Xt, p, workspace=ws)
            ar.pack(res.codes, c.bits)
        e1.record(stream)
        torch.cuda.synchronize()
    ms = e0.elapsed_time(e1)
    if ar.tune_status(ws) != ar.AR_OK:
        raise RuntimeError("device status not OK after the timed region")
    return {"metric": METRIC, "value": c.iters * args.steps / (ms / 1e3), "unit": UNIT, "n_gpus": 1,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms / args.steps,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
            "data": "synthetic",
            "config": {"workload": c.name, "mode": "quant-aware input, full-precision target",
                       "quantised_path_input": "target input x (1 + 0.05 N(0,1)), bf16", "algo": args.algo,
                       "n_rows": c.n_rows, "batch_rows": c.batch_rows, "iters": c.iters,
                       "bench_step": "one ar_tune_layer_fp_target call (all iters) + ar_pack"},
            "layer_tune_s": ms / args.steps / 1e3, "final_mse": float(res.final_mse.item()),
            "clocks": clk.summary(), "e2e": None}


def run_ours(args):
    import torch
    import torch.distributed as dist

    import signed_gradient_rounding_b200 as ar

    world, rank, local = _dist()
    # One process per GPU; AR_BENCH_BACKEND=gloo (with the final gather on the host)
    # lets the multi-rank path run where ranks share a GPU, as a test of the code path:
    # its times then mean nothing.
    backend = os.environ.get("AR_BENCH_BACKEND", "nccl")
    if backend not in ("nccl", "gloo"):
        raise SystemExit(f"AR_BENCH_BACKEND must be nccl or gloo, not {backend!r}")
    local = local % torch.cuda.device_count() if backend == "gloo" else local
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        import datetime
        if backend == "gloo":
            dist.init_process_group("gloo", timeout=datetime.timedelta(seconds=120))
        else:
            dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=dev)

    def all_max(x: float) -> float:
        t = torch.tensor([x], dtype=torch.float64, device=dev if backend == "nccl" else "cpu")
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        return float(t.item())
    from signed_gradient_rounding_b200.shard import row_range, tune_layer_sharded

    c = _workload(args)
    # One layer of out * world rows (weak scaling): rank r tunes its row_range shard
    # (out rows) on the same calibration activations and block schedule, with no
    # exchange during the loop; one all-gather of codes, scales and zero-points
    # over NCCL ends each step.  At world = 1 this is the workload's own layer.
    out_all = c.out * world
    a, b = row_range(out_all, rank, world)
    W_all = torch.from_numpy(make_weight(out_all, c.inn, c.w_std, c.w_dtype, seed=0))
    W = W_all[a:b].contiguous()
    Wd_all = (W_all.to(torch.bfloat16) if c.w_dtype == "bf16" else W_all).to(dev)
    del W_all
    Xd = make_activations_cuda(c.n_rows, c.inn, c.x_kind, seed=0, device=dev)
    p = ar.make_params(bits=c.bits, group_size=c.group_size, sym=c.sym, iters=c.iters, lr=c.lr,
                       minmax_lr=c.minmax_lr, batch_rows=c.batch_rows, seed=0, algo=args.algo,
                       split=int(args.split))
    rows = b - a
    ws = torch.empty(ar.tune_workspace_bytes(rows, c.inn, c.n_rows, p), dtype=torch.uint8, device=dev)
    G = c.inn // (c.inn if c.group_size == -1 else c.group_size)
    outs = (torch.empty((rows, c.inn), dtype=torch.uint8, device=dev),
            torch.empty((rows, G), dtype=torch.float32, device=dev),
            torch.empty((rows, G), dtype=torch.int32, device=dev),
            torch.empty((c.iters,), dtype=torch.float32, device=dev),
            torch.empty((1,), dtype=torch.float64, device=dev))
    stream = torch.cuda.current_stream(dev)
    timing_slot = [None]

    def compute(W_shard, X):
        res = ar.tune_layer(W_shard, X, p, workspace=ws, outputs=outs, timing=timing_slot[0])
        return res.codes, res.scale, res.zero_point

    def one_step(timing=None):
        timing_slot[0] = timing
        (codes, scale, zp), _ = tune_layer_sharded(Wd_all, Xd, compute)
        packed = ar.pack(codes, c.bits)
        return packed

    for _ in range(args.warmup):
        one_step()
    torch.cuda.synchronize()
    if ar.tune_status(ws) != ar.AR_OK:
        raise RuntimeError("device status not OK after warm-up")

    timings = []
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    with ClockSampler(local) as clk:
        e0.record(stream)
        for _ in range(args.steps):
            t = ar.TuneTiming()
            one_step(t)
            timings.append(t)
        e1.record(stream)
        torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    ms = e0.elapsed_time(e1)
    if ar.tune_status(ws) != ar.AR_OK:
        raise RuntimeError("device status not OK after the timed region")
    mse = float(outs[4].item())
    ms_max = all_max(ms) if world > 1 else ms

    # End to end through the host API: pinned host inputs copied in and the
    # results copied out inside the timed region, every step (this rank's shard).
    e2e = None
    if args.e2e_steps > 0:
        del Wd_all
        Wh = W.to(torch.bfloat16 if c.w_dtype == "bf16" else torch.float32).pin_memory()
        Xh = Xd.cpu().pin_memory()
        h2d = Wh.numel() * Wh.element_size() + Xh.numel() * Xh.element_size()
        d2h = rows * c.inn + 2 * rows * G * 4 + c.iters * 4 + 8
        del Xd
        torch.cuda.empty_cache()
        ar.tune_layer_host(Wh, Xh, p, device=dev)          # warm
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize()
        f0, f1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        f0.record(stream)
        for _ in range(args.e2e_steps):
            ar.tune_layer_host(Wh, Xh, p, device=dev)
        f1.record(stream)
        torch.cuda.synchronize()
        ems = f0.elapsed_time(f1)
        if world > 1:
            ems = all_max(ems)
        e2e = {"value": world * c.iters * args.e2e_steps / (ems / 1e3), "unit": UNIT,
               "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": int(d2h), "steps": args.e2e_steps}

    if world > 1:
        dist.destroy_process_group()
    if rank != 0:
        return None

    peaks = _peaks()
    algo = {ar.AR_ALGO_DIRECT: "direct", ar.AR_ALGO_GRAM: "gram"}[timings[0].algo]
    pieces = (3 if algo == "gram" else 2) if args.split else 1
    if algo == "gram":
        # one launch per step: G = D H_b, D and H_b as bf16 pairs (3 products)
        flops_upd = pieces * 2.0 * c.out * c.inn * c.inn
        flops_res = 0.0
    else:
        # two launches per step: R = X_b D^T and G = R^T X_b, operands as bf16 pairs
        flops_res = flops_upd = pieces * 2.0 * c.batch_rows * c.out * c.inn
    n_launch = sum(t.gemm_launches for t in timings)
    res_ms = sum(t.residual_ms for t in timings) / n_launch
    upd_ms = sum(t.update_ms for t in timings) / n_launch
    if res_ms > upd_ms:
        dom_name, dom_ms, dom_flops = "residual (kEpiStore)", res_ms, flops_res
        traffic = _recorded_traffic("direct_residual_bytes")
    else:
        dom_name, dom_ms, dom_flops = "update (kEpiUpdate)", upd_ms, flops_upd
        traffic = _recorded_traffic(f"{algo}_update_bytes")
        g_eff = c.inn if c.group_size == -1 else c.group_size
        if not (256 % g_eff == 0 or (g_eff == c.inn and c.inn <= 256)):
            # groups wider than an epilogue thread's columns: the step is the
            # kEpiUpdateWide launch plus group_finish_kernel (timed together); the
            # recorded traffic is the narrow-group kernel's
            dom_name, traffic = "update (kEpiUpdateWide) + group_finish_kernel", None
    achieved = dom_flops / (dom_ms * 1e-3) / 1e12
    layer_s = ms_max / args.steps / 1e3
    step_ms = res_ms + upd_ms
    step_tflops = (flops_res + flops_upd) / (step_ms * 1e-3) / 1e12
    launches = sum(t.kernel_launches for t in timings) + args.steps    # + one pack per step
    config = _config(c, world)
    line = {
        "metric": METRIC,
        "value": world * c.iters * args.steps / (ms_max / 1e3),
        "unit": UNIT,
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": ms_max / args.steps,
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "bf16",
        "data": "synthetic",
        "config": config,
        "bench_step": "one ar_tune_layer call (all iters) on this rank's row shard, the all-gather of "
                      "codes/scales/zero-points (N > 1), and ar_pack",
        "layer_tune_s": layer_s,
        "algo": algo,
        "split_operands": bool(args.split),
        "chunked_accumulation": args.split == 2,
        "step_ms": step_ms,
        "setup_ms": sum(t.setup_ms for t in timings) / len(timings),
        "executed_tflop_per_step": (flops_res + flops_upd) / 1e12,
        "fused_step_tflops": step_tflops,
        "tensor_peak_frac": step_tflops / peaks["bf16_tflops_sustained"],
        "direct_form_tflop_per_step": c.flops_per_step / 1e12,
        "final_mse": mse,
        "roofline": {"bound": "tensor", "kernel": f"gemm_kernel {algo} {dom_name}", "achieved": achieved,
                     "peak": peaks["bf16_tflops_sustained"], "unit": "TFLOP/s",
                     "frac": achieved / peaks["bf16_tflops_sustained"], "traffic": traffic,
                     "traffic_unit": "bytes per launch (ncu, profiles/traffic.txt)",
                     "peak_source": peaks["source"] + " sustained bf16",
                     "per_launch_ms": {"residual": res_ms, "update": upd_ms}},
        "gpu_launches": launches,
        "clocks": clk.summary(),
        "e2e": e2e,
    }
    if world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(c, Xd if args.e2e_steps == 0 else None, args.cpu_rows, args.cpu_steps)
    return line


def _config(c, world: int) -> dict:
    """The workload as both arms state it (the same keys and values in each)."""
    return {"workload": c.name if world == 1 else f"{c.name}, {c.out * world} output rows in {world} row shards",
            "out": c.out * world, "in": c.inn, "n_rows": c.n_rows, "batch_rows": c.batch_rows, "iters": c.iters,
            "bits": c.bits, "group_size": c.group_size, "sym": c.sym, "lr": c.lr, "minmax_lr": c.minmax_lr,
            "keep_best": True, "seed": 0,
            "l2": "inputs larger than L2: X is %.1f GB, one step reads a %.0f MB block"
                  % (c.n_rows * c.inn * 2 / 1e9, c.batch_rows * c.inn * 2 / 1e6),
            "parallelism": f"row shards x{world}; one all-gather of the results per step, none in the loop"}


def _threads():
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads", 0) for i in threadpool_info() if i.get("user_api") == "blas"]
        if n:
            return max(n)
    except Exception:
        pass
    return os.cpu_count()


def _cpu_model() -> str:
    """The host CPU's model name (Linux /proc/cpuinfo), or "" when unknown."""
    try:
        with open("/proc/cpuinfo", encoding="utf-8") as f:
            for line in f:
                if line.startswith("model name"):
                    return line.split(":", 1)[1].strip()
    except OSError:
        pass
    return ""


def _host_x(c, Xd=None):
    """The workload's activations on the host as bf16 bit patterns (same bytes as the GPU run)."""
    try:
        import torch
        if Xd is None and torch.cuda.is_available():
            Xd = make_activations_cuda(c.n_rows, c.inn, c.x_kind, seed=0)
        if Xd is not None:
            return Xd.view(torch.int16).cpu().numpy().view(np.uint16)
    except ImportError:
        pass
    from workloads import bf16_bits
    return bf16_bits(make_activations(c.n_rows, c.inn, c.x_kind, seed=0))


def cpu_baseline(c, Xd, rows: int, steps: int):
    """The oracle, as it stands, on `rows` sampled output rows for `steps` SignSGD
    steps of the same workload; rows tune independently and every row-step costs
    the same, so the rate scales to the full layer by rows / out."""
    import oracle
    X = _host_x(c, Xd)
    W = make_weight(c.out, c.inn, c.w_std, c.w_dtype, seed=0)
    sel = np.sort(np.random.default_rng(0).choice(c.out, min(rows, c.out), replace=False))
    t0 = time.perf_counter()
    oracle.tune_layer(W[sel], X, c.bits, c.group_size, c.sym, steps, c.lr, c.minmax_lr, c.batch_rows, 0,
                      want_final_mse=False)
    dt = time.perf_counter() - t0
    return {"value": steps * (len(sel) / c.out) / dt, "unit": UNIT, "cores": _threads(), "kind": "oracle",
            "sample": f"{len(sel)} of {c.out} output rows x {steps} steps on the full activations, "
                      f"{dt:.1f} s; rate scaled by rows/out (rows tune independently)",
            "host_cpu": os.cpu_count(), "cpu_model": _cpu_model()}


def run_reference(args):
    world, rank, _ = _dist()
    if rank != 0:
        return None
    c = _workload(args)
    import oracle
    X = _host_x(c)
    W = make_weight(c.out, c.inn, c.w_std, c.w_dtype, seed=0)
    sel = np.sort(np.random.default_rng(0).choice(c.out, min(args.cpu_rows, c.out), replace=False))

    def one_step():
        oracle.tune_layer(W[sel], X, c.bits, c.group_size, c.sym, args.cpu_steps, c.lr, c.minmax_lr,
                          c.batch_rows, 0, want_final_mse=False)

    for _ in range(args.warmup):
        one_step()
    t0 = time.perf_counter()
    for _ in range(args.steps):
        one_step()
    dt = time.perf_counter() - t0
    value = args.steps * args.cpu_steps * (len(sel) / c.out) / dt
    return {"impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": dt / args.steps * 1e3,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic",
            "config": _config(c, world),
            "bench_step": f"oracle.tune_layer on {len(sel)} sampled output rows x {args.cpu_steps} SignSGD steps",
            "cpu_baseline": {"value": value, "unit": UNIT, "cores": _threads(), "kind": "oracle",
                             "sample": f"each step: {len(sel)} of {c.out} output rows x {args.cpu_steps} "
                                       f"SignSGD steps; rate scaled by rows/out",
                             "host_cpu": os.cpu_count(), "cpu_model": _cpu_model()},
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", choices=sorted(WORKLOADS), default="q_proj")
    ap.add_argument("--e2e-steps", type=int, default=3)
    ap.add_argument("--cpu-rows", type=int, default=64)
    ap.add_argument("--cpu-steps", type=int, default=10)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--algo", choices=["auto", "direct", "gram"], default="auto")
    ap.add_argument("--split", type=int, default=1, choices=[0, 1, 2],
                    help="1: bf16-pair operands (default); 0: single bf16; 2: pairs and chunked K accumulation")
    ap.add_argument("--group-size", type=int, default=None,
                    help="override the workload's group size (-1: one group per row)")
    ap.add_argument("--mode", choices=["layer", "fp_target"], default="layer",
                    help="fp_target: quant-aware input with a full-precision target")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    if args.impl == "reference":
        line = run_reference(args)
    elif args.workload == "block_7b":
        line = run_block(args)
    elif args.mode == "fp_target":
        line = run_fp_target(args)
    else:
        line = run_ours(args)
    if line is not None:
        print(json.dumps(line), flush=True)


if __name__ == "__main__":
    main()
