"""GPU parity of the layer chain (quant-aware, layer-by-layer block tuning): the
dequantisation, the quantised linear layer, silu*mul, and a small decoder block
whose every layer is compared with the oracle tuned on the same input bytes."""
import numpy as np
import pytest
import torch

import oracle
from oracle import autoround as oar
from tests.free_running import code_bound, oracle_drift
from workloads import bf16_from_bits, make_activations, make_weight

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def ar():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    import signed_gradient_rounding_b200 as ar
    return ar


def _vals(t):
    """bf16 device tensor -> float32 numpy values."""
    return bf16_from_bits(t.view(torch.int16).cpu().numpy().view(np.uint16))


def _bf16_ulp_close(got, ref64, frac_max, abs_sum=None, rel=2.0 ** -19):
    """Every value within one bf16 step of the exact result plus the fp32 accumulation
    error (at most 2^-19 of the sum of |terms|, abs_sum), and at most frac_max of them
    not the correctly rounded one (the GPU's fp32 accumulation of bf16-pair weights
    sits close to exact, so only near-midpoint values may round the other way)."""
    got = got.astype(np.float64)
    exact = oracle.chain._bf16_round(ref64).astype(np.float64)
    ulp = np.abs(np.spacing(exact.astype(np.float32)).astype(np.float64)) * 65536
    slack = 0.0 if abs_sum is None else abs_sum * rel
    bad = np.abs(got - exact) > ulp * 1.0001 + slack + 1e-30
    assert not bad.any(), (f"{int(bad.sum())} values off: got {got[bad][:4]} exact {exact[bad][:4]} "
                           f"ulp {ulp[bad][:4]} slack {np.broadcast_to(slack, got.shape)[bad][:4]}")
    assert np.mean(got != exact) <= frac_max


def test_dequant_bitexact(ar):
    rng = np.random.default_rng(1)
    out, inn, g = 70, 320, 64
    codes = rng.integers(0, 8, (out, inn), dtype=np.uint8)
    scale = rng.uniform(1e-3, 1e-2, (out, inn // g)).astype(np.float32)
    zp = rng.integers(0, 8, (out, inn // g)).astype(np.int32)
    hi, lo, f32 = ar.dequant(torch.from_numpy(codes).cuda(), torch.from_numpy(scale).cuda(),
                             torch.from_numpy(zp).cuda(), g, want_f32=True)
    ref = oracle.chain.dequant(codes, scale, zp, g)
    assert np.array_equal(f32.cpu().numpy(), ref)
    assert np.array_equal(_vals(hi) + _vals(lo), ref) or np.all(
        np.abs(_vals(hi).astype(np.float64) + _vals(lo) - ref) <= np.abs(ref) * 2.0 ** -16)


@pytest.mark.parametrize("shape", [(300, 320, 200), (1024, 4096, 4096), (64, 256, 11008)])
@pytest.mark.parametrize("with_add", [False, True])
def test_linear(ar, shape, with_add):
    n, inn, out = shape
    rng = np.random.default_rng(n + out)
    X = make_activations(n, inn, "llm", seed=2)
    Wq = (rng.standard_normal((out, inn)) * 0.02).astype(np.float32)
    add = make_activations(n, out, "tiny", seed=3) if with_add else None
    Wt = torch.from_numpy(Wq).cuda()
    hi = Wt.to(torch.bfloat16)
    lo = (Wt - hi.float()).to(torch.bfloat16)
    Y = ar.linear(torch.from_numpy(X).to(torch.bfloat16).cuda(), hi, lo,
                  None if add is None else torch.from_numpy(add).to(torch.bfloat16).cuda())
    torch.cuda.synchronize()
    Wpair = hi.float().cpu().numpy().astype(np.float64) + lo.float().cpu().numpy()
    ref = X.astype(np.float64) @ Wpair.T + (0 if add is None else add.astype(np.float64))
    abs_sum = np.abs(X.astype(np.float64)) @ np.abs(Wpair).T
    _bf16_ulp_close(_vals(Y), ref, 0.02, abs_sum)


def test_silu_mul(ar):
    a = make_activations(512, 1024, "llm", seed=4)
    b = make_activations(512, 1024, "llm", seed=5)
    y = ar.silu_mul(torch.from_numpy(a).to(torch.bfloat16).cuda(), torch.from_numpy(b).to(torch.bfloat16).cuda())
    torch.cuda.synchronize()
    a64 = a.astype(np.float64)
    _bf16_ulp_close(_vals(y), a64 / (1 + np.exp(-a64)) * b, 0.02)


def test_small_block_layer_by_layer(ar):
    """A small decoder block (hidden 256, MLP 512, W3 g64 sym, 20 steps, 2 blocks of 512
    rows): every layer's tuning against the oracle on the same input bytes, and every
    chained activation against the oracle's chain from the GPU's own codes."""
    from signed_gradient_rounding_b200.block import tune_block
    hidden, mlp, n, B, g, bits, iters = 256, 512, 1024, 512, 64, 3, 20
    shapes = {"q_proj": (hidden, hidden), "k_proj": (hidden, hidden), "v_proj": (hidden, hidden),
              "o_proj": (hidden, hidden), "gate_proj": (mlp, hidden), "up_proj": (mlp, hidden),
              "down_proj": (hidden, mlp)}
    Ws = {k: make_weight(o, i, 0.02, "bf16", seed=10 + j) for j, (k, (o, i)) in enumerate(shapes.items())}
    x0 = make_activations(n, hidden, "llm", seed=9)
    p = ar.make_params(bits=bits, group_size=g, sym=True, iters=iters, batch_rows=B, seed=1)
    res, inputs = tune_block(torch.from_numpy(x0).to(torch.bfloat16).cuda(),
                             {k: torch.from_numpy(w).to(torch.bfloat16).cuda() for k, w in Ws.items()}, p,
                             keep_inputs=True)
    torch.cuda.synchronize()
    codes = {k: r.codes.cpu().numpy() for k, r in res.items()}
    wq = {k: oracle.chain.dequant(codes[k], res[k].scale.cpu().numpy(), res[k].zero_point.cpu().numpy(), g)
          for k in res}
    X = {k: _vals(v) for k, v in inputs.items()}
    # the chain, from the GPU's own tuned layers
    assert np.array_equal(X["q_proj"], x0) and np.array_equal(X["v_proj"], x0)
    v_out = X["o_proj"]
    wv = wq["v_proj"].astype(np.float64)
    # the GPU multiplies W' as a bf16 pair (~2^-17 relative): slack 2^-15 of sum |x w|
    _bf16_ulp_close(v_out, x0.astype(np.float64) @ wv.T, 0.02, np.abs(x0.astype(np.float64)) @ np.abs(wv).T,
                    2.0 ** -15)
    h = X["gate_proj"]
    wo = wq["o_proj"].astype(np.float64)
    _bf16_ulp_close(h, v_out.astype(np.float64) @ wo.T + x0, 0.02,
                    np.abs(v_out.astype(np.float64)) @ np.abs(wo).T + np.abs(x0), 2.0 ** -15)
    gl = oracle.chain.linear(h, wq["gate_proj"])
    ul = oracle.chain.linear(h, wq["up_proj"])
    a_ref = gl.astype(np.float64) / (1 + np.exp(-gl.astype(np.float64))) * ul
    got = X["down_proj"].astype(np.float64)
    # two bf16 roundings feed silu*mul; compare within a few bf16 steps
    assert np.max(np.abs(got - a_ref) / (np.abs(a_ref) + 1e-3)) < 0.05
    # every layer's tuning, on the GPU's input bytes
    for k in shapes:
        ref = oracle.tune_layer(Ws[k], X[k], bits, g, True, iters, 0.005, -1.0, B, 1)
        frac = float(np.mean(codes[k] != ref.codes))
        assert frac <= 0.005, f"{k}: {frac:.3%} of codes differ"
        mse_gpu = oar.layer_mse(Ws[k], wq[k], X[k])
        assert mse_gpu == pytest.approx(ref.final_mse, rel=0.02), k


def test_block_7b_full_size_sampled_rows(ar):
    """The LLaMA-7B decoder block at full size (262144 calibration rows, W3 g128 sym,
    200 steps per layer), as the benchmark runs it; per layer the oracle replays 16
    sampled rows on the GPU's own input bytes.  Full-size trajectories are chaotic
    (see test_gpu_parity), so the bars are the MSE (2%) and twice the oracle's drift
    against its own jittered run (tests/free_running.py)."""
    from signed_gradient_rounding_b200.block import tune_block
    from workloads import BLOCK_7B, BLOCK_7B_LAYERS, make_activations_cuda
    c = BLOCK_7B
    Ws = {name: make_weight(o, i, c.w_std, c.w_dtype, seed=10 + j) for j, (name, o, i) in enumerate(BLOCK_7B_LAYERS)}
    x0 = make_activations_cuda(c.n_rows, c.inn, c.x_kind, seed=0)
    p = ar.make_params(bits=c.bits, group_size=c.group_size, sym=True, iters=c.iters, batch_rows=c.batch_rows, seed=0)
    res, inputs = tune_block(x0, {k: torch.from_numpy(w).to(torch.bfloat16).cuda() for k, w in Ws.items()}, p,
                             keep_inputs=True)
    torch.cuda.synchronize()
    Xh = {}
    for name, o, i in BLOCK_7B_LAYERS:
        key = id(inputs[name])
        if key not in Xh:
            Xh[key] = inputs[name].view(torch.int16).cpu().numpy().view(np.uint16)
    del inputs, x0
    torch.cuda.empty_cache()
    keys = list(Xh)  # x0, v'(x0), h, silu(gate'(h)) * up'(h), in tuning order
    order = {"q_proj": 0, "k_proj": 0, "v_proj": 0, "o_proj": 1, "gate_proj": 2, "up_proj": 2, "down_proj": 3}
    for j, (name, o, i) in enumerate(BLOCK_7B_LAYERS):
        X = Xh[keys[order[name]]]
        rows = np.sort(np.random.default_rng(j).choice(o, 16, replace=False))
        ref = oracle.tune_layer(Ws[name][rows], X, c.bits, c.group_size, True, c.iters, c.lr, -1.0, c.batch_rows, 0,
                                want_final_mse=False)
        r = res[name]
        codes = r.codes.cpu().numpy()[rows]
        wq = oracle.chain.dequant(codes, r.scale.cpu().numpy()[rows], r.zero_point.cpu().numpy()[rows], c.group_size)
        mse_gpu = oar.layer_mse(Ws[name][rows], wq, X[:16384])
        mse_ref = oar.layer_mse(Ws[name][rows], ref.Wq, X[:16384])
        frac = float(np.mean(codes != ref.codes))
        drift = oracle_drift(ref, Ws[name][rows], X, c.bits, c.group_size, True, c.iters, c.lr, -1.0, c.batch_rows)
        print(f"block {name}: {frac:.3%} codes differ (oracle against its jittered self: {drift:.3%}), "
              f"mse {mse_gpu:.6g} vs oracle {mse_ref:.6g}")
        assert mse_gpu == pytest.approx(mse_ref, rel=0.02), name
        assert frac <= code_bound(drift, len(rows)), name
