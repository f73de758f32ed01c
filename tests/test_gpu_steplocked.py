"""Step-locked parity at full size: the GPU's own trajectory, checked one step at a time.

The tuning loop ("[llm-compressor] AutoRound ...", "on_event with
SEQUENTIAL_EPOCH_END") moves every V, alpha and beta by the sign of a gradient.
Run free, two correct implementations part ways wherever a gradient sign lies
within their rounding of zero, and the SignSGD iteration carries the difference
on.  This file removes that fork: at each checked step k it takes the GPU's own
state S_k (resumed runs are bit-identical to one run), lets the GPU take step k,
and lets the oracle take step k from the same S_k on sampled output rows (rows
tune independently).  It then requires, for every sampled row:

* the batch loss of step k (the number the keep-best choice compares) equal to
  the oracle's within the bound of the tensor cores' fp32 accumulation (see
  loss_rtol: 3e-5 in the Gram form, 1.2e-4 to 8.8e-4 in the direct form);
* the same move of every V whose gradient is clear of a tie (|G| above 1e-5 of
  the gradient's rms, the bar of test_one_step_signs), and of every alpha and
  beta whose group sum is clear of a tie (|d alpha| above 1e-5 of
  sum_k |G_k dW'_k/d alpha|, the scale of that sum's rounding);
* the same keep-best decision wherever the step loss is not within 1e-5 of the
  row's best so far, and the snapshot taken from the right state;
* codes, scales and zero-points of the applied state after the step bit-exact
  with the oracle's fake-quantisation of that state.

Free-running divergence (how far the final codes drift once ties have forked
the trajectories) is measured and printed by the full-size tests in
test_gpu_parity.py, which decompose it into rows whose best step differs and
rows that kept the same step.
"""
import ctypes
import dataclasses

import numpy as np
import pytest
import torch

import oracle
from workloads import DOWN_7B, DOWN_72B, Q_PROJ_7B, make_activations_cuda, make_weight

pytestmark = pytest.mark.gpu

TIE_G = 1e-5          # |G| below this fraction of rms(G): a tie of dV's sign
TIE_GROUP = 1e-5      # |d alpha| below this fraction of sum |G dW'/d alpha|: a tie
TIE_BEST = 1e-5       # step loss within this of the best so far: a keep-best tie


@pytest.fixture(scope="module")
def ar():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    import signed_gradient_rounding_b200 as ar
    return ar


def _np(t):
    return t.detach().cpu().numpy()


def _bits(Xd):
    return Xd.view(torch.int16).cpu().numpy().view(np.uint16)


@dataclasses.dataclass
class _Snap:
    V: np.ndarray
    alpha: np.ndarray
    beta: np.ndarray
    best: np.ndarray
    V_best: np.ndarray
    alpha_best: np.ndarray
    beta_best: np.ndarray


def _snap(st, rows_t) -> _Snap:
    return _Snap(*(_np(getattr(st, f).index_select(0, rows_t)) for f in
                   ("V", "alpha", "beta", "best_loss", "V_best", "alpha_best", "beta_best")))


def _quantised_path_input(Xt):
    """The layer's input on the quantised path for the full-precision-target mode: the
    target's input with 5% seeded multiplicative noise, in bf16 (as the full-size
    fp-target test and the benchmark make it)."""
    gen = torch.Generator(device="cuda")
    gen.manual_seed(5)
    Xq = torch.empty_like(Xt)
    chunk = (1 << 27) // Xt.shape[1]
    for r0 in range(0, Xt.shape[0], chunk):
        z = torch.randn((min(chunk, Xt.shape[0] - r0), Xt.shape[1]), generator=gen, device="cuda")
        Xq[r0:r0 + chunk] = (Xt[r0:r0 + chunk].float() * (1 + 0.05 * z)).to(torch.bfloat16)
    return Xq


def _step_locked(ar, c, algo, n_rows_sample, checkpoints, seed=0, fp_target=False):
    """Run workload ``c`` on the GPU step by step through the checkpoints and compare
    each checked step with the oracle's step from the GPU's state.  With fp_target the
    layer sees a noisy copy of the activations and is tuned against the full-precision
    output (ar_tune_layer_fp_target).  Returns a per-checkpoint summary (also printed)."""
    g = c.inn if c.group_size == -1 else c.group_size
    W = make_weight(c.out, c.inn, c.w_std, c.w_dtype, seed=seed)
    Wd = torch.from_numpy(W).to(torch.bfloat16).cuda()
    Xd = make_activations_cuda(c.n_rows, c.inn, c.x_kind, seed=seed)
    Xt = None
    if fp_target:
        Xt, Xd = Xd, _quantised_path_input(Xd)
    Xh = _bits(Xd)
    Xth = _bits(Xt) if fp_target else None
    rows = np.sort(np.random.default_rng(seed).choice(c.out, n_rows_sample, replace=False))
    rows_t = torch.from_numpy(rows).cuda()
    Wr = W[rows]
    wmin, wmax = oracle.group_minmax(Wr, g)
    n_blocks = c.n_rows // c.batch_rows
    sched = oracle.block_schedule(n_blocks, c.iters, seed)
    mlr = c.lr if c.minmax_lr < 0 else c.minmax_lr

    st = ar.TuneState.empty(c.out, c.inn, c.group_size)

    def params(iters, start):
        return ar.make_params(bits=c.bits, group_size=c.group_size, sym=c.sym, iters=iters, lr=c.lr,
                              minmax_lr=c.minmax_lr, batch_rows=c.batch_rows, seed=seed, start_step=start,
                              algo=algo)

    def need_bytes(p):
        if fp_target:
            return int(ar.lib.ar_tune_fp_target_workspace_bytes(c.out, c.inn, c.n_rows, ar.AR_BF16, ctypes.byref(p)))
        return ar.tune_workspace_bytes(c.out, c.inn, c.n_rows, p)

    def run(p):
        if fp_target:
            return ar.tune_layer_fp_target(Wd, Xd, Xt, p, workspace=ws, want_final_mse=False, state=st)
        return ar.tune_layer(Wd, Xd, p, state=st, workspace=ws, want_loss_trace=False, want_final_mse=False)

    need = max(need_bytes(params(it, 0)) for it in (0, 1, c.iters))
    ws = torch.empty(need, dtype=torch.uint8, device="cuda")
    # iters = 0 initialises the state (V = 0, alpha = beta = 1, best = +inf).
    run(params(0, 0))
    cache = {}
    summary = []
    cur = 0
    for k in checkpoints:
        if k > cur:
            run(params(k - cur, cur))
            cur = k
        s0 = _snap(st, rows_t)
        p1 = params(1, k)
        res = run(p1)
        assert ar.tune_status(ws) == ar.AR_OK
        loss_gpu = _np(ar.tune_row_losses(ws, c.out, c.inn, c.n_rows, p1)[0].index_select(0, rows_t))
        loss_gpu = loss_gpu.astype(np.float64) / c.batch_rows
        codes = _np(res.codes.index_select(0, rows_t))
        scale = _np(res.scale.index_select(0, rows_t))
        zp = _np(res.zero_point.index_select(0, rows_t))
        s1 = _snap(st, rows_t)
        cur = k + 1

        blk = sched[k]
        if blk not in cache:
            if len(cache) >= 4:
                cache.pop(next(iter(cache)))
            r0, r1 = blk * c.batch_rows, (blk + 1) * c.batch_rows
            cache[blk] = (oracle.autoround._rows_f64(Xh, r0, r1),
                          oracle.autoround._rows_f64(Xth, r0, r1) if fp_target else None)
        ref = oracle.sign_step(Wr, cache[blk][0], s0.V, s0.alpha, s0.beta, wmin, wmax, g, c.bits, c.sym, c.lr, mlr,
                               Xt_b=cache[blk][1], with_scale=True)

        rel = (loss_gpu - ref.row_loss) / ref.row_loss
        loss_err = float(np.max(np.abs(rel)))
        loss_bias = float(np.mean(rel))
        rms = float(np.sqrt(np.mean(ref.G ** 2)))
        v_diff = s1.V != ref.V
        v_bad = int(np.sum(v_diff & (np.abs(ref.G) > TIE_G * rms)))
        v_tie = float(np.max(np.abs(ref.G[v_diff]))) / rms if v_diff.any() else 0.0
        a_diff = s1.alpha != ref.alpha
        a_bad = int(np.sum(a_diff & (np.abs(ref.dalpha) > TIE_GROUP * ref.dalpha_abs)))
        b_diff = s1.beta != ref.beta
        b_bad = int(np.sum(b_diff & (np.abs(ref.dbeta) > TIE_GROUP * ref.dbeta_abs))) if not c.sym else 0
        best0 = s0.best.astype(np.float64)
        want = ref.row_loss < best0
        got = s1.best < s0.best
        near = np.abs(ref.row_loss - best0) <= TIE_BEST * np.where(np.isfinite(best0), best0, 1.0)
        best_bad = int(np.sum((want != got) & ~near))
        # the snapshot: improving rows keep S_k, the others keep their old best
        snap_ok = all(np.array_equal(s1.V_best[j], s0.V[j] if got[j] else s0.V_best[j]) and
                      np.array_equal(s1.alpha_best[j], s0.alpha[j] if got[j] else s0.alpha_best[j])
                      for j in range(len(rows)))
        # codes of the applied (best) state after the step: bit-exact with the oracle's
        sc, z = oracle.scale_zero_point(wmin, wmax, s1.alpha_best, s1.beta_best, c.bits, c.sym)
        fq = oracle.fake_quant(Wr, s1.V_best, sc, z, g, c.bits)
        codes_ok = (np.array_equal(codes, fq.q.astype(np.uint8)) and np.array_equal(scale, sc)
                    and np.array_equal(zp, z.astype(np.int32)))
        row = dict(k=k, loss_err=loss_err, loss_bias=loss_bias, v_diff=int(v_diff.sum()), v_bad=v_bad, v_tie=v_tie, a_diff=int(a_diff.sum()),
                   a_bad=a_bad, b_diff=int(b_diff.sum()), b_bad=b_bad, best_diff=int(np.sum(want != got)),
                   best_bad=best_bad, snap_ok=snap_ok, codes_ok=codes_ok,
                   moved=int(np.sum(s1.V != s0.V)), improved=int(np.sum(got)))
        summary.append(row)
    tot = {key: sum(r[key] for r in summary) for key in ("v_diff", "v_bad", "a_diff", "a_bad", "b_diff", "b_bad",
                                                         "best_diff", "best_bad", "moved", "improved")}
    worst = max(r["loss_err"] for r in summary)
    bias = float(np.mean([r["loss_bias"] for r in summary]))
    tie = max(r["v_tie"] for r in summary)
    print(f"\n{c.name} [{algo}{', full-precision target' if fp_target else ''}] step-locked over {len(summary)} steps x {len(rows)} rows: "
          f"V moves {tot['moved']}, differing {tot['v_diff']} (clear of a tie: {tot['v_bad']}; the largest "
          f"|G| among them {tie:.2e} of rms); "
          f"alpha differing {tot['a_diff']} ({tot['a_bad']}), beta {tot['b_diff']} ({tot['b_bad']}); "
          f"keep-best improvements {tot['improved']}, decisions differing {tot['best_diff']} ({tot['best_bad']}); "
          f"row-loss rel err max {worst:.2e}, mean signed {bias:.2e}")
    for r in summary:
        if r["v_diff"] or r["a_diff"] or r["b_diff"] or r["best_diff"] or not (r["snap_ok"] and r["codes_ok"]):
            print("   ", r)
    return summary


def loss_rtol(c, algo):
    """Bound on the relative error of the GPU's per-row batch loss.  Each addition into
    a tensor core's fp32 accumulator loses less than one unit in the last place
    (2^-23 of the running sum), so a sum built from N accumulation steps is off by
    less than N * 2^-23 relative, and a sum of squares by twice that.  Direct form:
    the residual R accumulates 2 products (the bf16 pair) x in/16 MMA steps.  Gram
    form: the loss d H_b d^T rests on H_b, summed in fp32 from chunks of at most 2048
    calibration rows (128 MMA steps each)."""
    steps = 2 * c.inn // 16 if algo == "direct" else 2048 // 16
    return 2.0 * steps * 2.0 ** -23


def _assert_locked(summary, rtol):
    for r in summary:
        assert r["loss_err"] <= rtol, r
        assert r["v_bad"] == 0 and r["a_bad"] == 0 and r["b_bad"] == 0, r
        assert r["best_bad"] == 0, r
        assert r["snap_ok"] and r["codes_ok"], r


@pytest.mark.parametrize("algo", ["gram", "direct"])
def test_q_proj_step_locked(ar, algo):
    """The 4096 x 4096 W4 g128 layer (the benchmarked workload): every one of the 200
    steps in the Gram form (the one the benchmark runs), every 10th in the direct form."""
    ks = list(range(Q_PROJ_7B.iters)) if algo == "gram" else list(range(0, Q_PROJ_7B.iters, 10)) + [199]
    _assert_locked(_step_locked(ar, Q_PROJ_7B, algo, 64, ks), loss_rtol(Q_PROJ_7B, algo))


def test_down_7b_step_locked(ar):
    """LLaMA-7B down_proj 4096 x 11008 W2 g128 (Gram form, as the full run picks)."""
    _assert_locked(_step_locked(ar, DOWN_7B, "gram", 64, [0, 50, 100, 150, 199]), loss_rtol(DOWN_7B, "gram"))


def test_down_72b_step_locked(ar):
    """Qwen2.5-72B down_proj 8192 x 29568 W2 g128 (direct form, as the full run picks)."""
    _assert_locked(_step_locked(ar, DOWN_72B, "direct", 32, [0, 50, 100, 150, 199]),
                   loss_rtol(DOWN_72B, "direct"))


def test_q_proj_per_channel_step_locked(ar):
    """The 4096 x 4096 W4 layer with one group per row (the wide-group path: the step
    kernel's per-segment partials and the group-finish kernel), Gram form."""
    c = dataclasses.replace(Q_PROJ_7B, group_size=-1, name="q_proj per-channel")
    _assert_locked(_step_locked(ar, c, "gram", 32, [0, 50, 100, 150, 199]), loss_rtol(c, "gram"))


@pytest.mark.parametrize("algo", ["gram", "direct"])
def test_q_proj_fp_target_step_locked(ar, algo):
    """The full-precision-target mode ("enable_quanted_input"): the layer sees a noisy
    copy of the activations and is tuned against the full-precision output, in both
    forms (Gram: C_b joins G; direct: E_b joins R)."""
    # the target's terms of the loss (|dX_b w_j^T|^2, or E_b inside R) accumulate over
    # K = in, as the direct form's residual does: its bound applies in both forms
    _assert_locked(_step_locked(ar, Q_PROJ_7B, algo, 32, [0, 50, 100, 150, 199], fp_target=True),
                   loss_rtol(Q_PROJ_7B, "direct"))
