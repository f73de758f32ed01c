"""AutoRound layer tuning, written out plainly (oracle side).

TEST INFRASTRUCTURE ONLY (see the package docstring for the sources and the
readings of the pages that this file follows).

Notation: W is [out, in]; a group is ``g`` consecutive columns of one row
(g = in when group_size is -1); Q = 2^bits - 1.  fp32 arrays hold the quantiser
state; every expression on fp32 arrays below is evaluated by numpy one IEEE
fp32 operation at a time.  Contractions and derivatives are fp64.
"""
from __future__ import annotations

import dataclasses

import numpy as np

from .schedule import block_schedule

F32 = np.float32
F64 = np.float64


def qmax(bits: int) -> np.float32:
    """Largest code, 2^bits - 1 ("[SGLang] AutoRound ...", 1. AutoRoundConfig: bits 2/3/4/8)."""
    if bits not in (2, 3, 4, 8):
        raise ValueError("bits must be one of 2, 3, 4, 8")
    return F32(2 ** bits - 1)


def _group(inn: int, group_size: int) -> int:
    g = inn if group_size == -1 else group_size
    if g <= 0 or inn % g:
        raise ValueError("group_size must be -1 or a positive divisor of in")
    return g


def _to_f32(a: np.ndarray) -> np.ndarray:
    """Accept fp32/fp64 values or uint16 bf16 bit patterns; return fp32."""
    a = np.asarray(a)
    if a.dtype == np.uint16:
        return (a.astype(np.uint32) << 16).view(np.float32)
    return a.astype(F32)


def _rows_f64(X: np.ndarray, r0: int, r1: int) -> np.ndarray:
    blk = X[r0:r1]
    if blk.dtype == np.uint16:
        return (blk.astype(np.uint32) << 16).view(np.float32).astype(F64)
    return blk.astype(F64)


def _expand(a: np.ndarray, g: int) -> np.ndarray:
    """Per-group [out, G] values broadcast to the elements [out, G*g]."""
    return np.repeat(a, g, axis=1)


# --------------------------------------------------------------------------
# forward: min-max init, scale / zero-point, offset fake-quant
# --------------------------------------------------------------------------

def group_minmax(W: np.ndarray, group_size: int):
    """Min-max statistics per group, widened to include 0.

    "[llm-compressor] AutoRound ...", "on_event with SEQUENTIAL_EPOCH_END":
    ``_init_scale_zp`` is min-max.  Reading: wmin = min(0, min W_grp),
    wmax = max(0, max W_grp), so 0 is always representable; taken from the
    original W and never updated.
    """
    W = _to_f32(W)
    out, inn = W.shape
    g = _group(inn, group_size)
    Wg = W.reshape(out, inn // g, g)
    wmin = np.minimum(Wg.min(axis=2), F32(0))
    wmax = np.maximum(Wg.max(axis=2), F32(0))
    return wmin, wmax


def scale_zero_point(wmin, wmax, alpha, beta, bits: int, sym: bool):
    """Scale and zero-point from the clip factors.

    Asymmetric: s = (alpha*wmax - beta*wmin) / Q and zp = clamp(rint(-beta*wmin / s), 0, Q),
    the clipped min-max range whose bounds are learned jointly with the rounding
    ("Introducing AutoRound ...", section 2).  An all-zero group gets s = 1.
    Symmetric (reading): amax = max(-wmin, wmax), s = 2*alpha*amax / Q,
    zp = 2^(bits-1); beta is unused.
    """
    Q = qmax(bits)
    wmin = _to_f32(wmin)
    wmax = _to_f32(wmax)
    alpha = _to_f32(alpha)
    beta = _to_f32(beta)
    if sym:
        amax = np.maximum(-wmin, wmax)
        s = (F32(2) * (alpha * amax)) / Q
        s = np.where(s == 0, F32(1), s).astype(F32)
        zp = np.full(s.shape, F32(2 ** (bits - 1)), dtype=F32)
    else:
        s = (alpha * wmax - beta * wmin) / Q
        s = np.where(s == 0, F32(1), s).astype(F32)
        zp = np.clip(np.rint(-(beta * wmin) / s), F32(0), Q).astype(F32)
    return s, zp


@dataclasses.dataclass
class FakeQuant:
    u: np.ndarray      # W / s
    t: np.ndarray      # u + V
    r: np.ndarray      # rint(t), ties to even
    p: np.ndarray      # r + zp
    q: np.ndarray      # clamp(p, 0, Q): the integer code
    m: np.ndarray      # 0 <= p <= Q (bool): the clamp's pass-through mask
    Wq: np.ndarray     # s * (q - zp)


def fake_quant(W, V, s, zp, group_size: int, bits: int) -> FakeQuant:
    """Offset rounding of every element.

    "[llm-compressor] AutoRound ...", section "논문 핵심 내용": w^ = s*round(w/s + V);
    ``_fake_quantize_with_offset``: q = clamp(round(W/s + zp + V), qmin, qmax),
    W' = s*(q - zp).  The rounding argument is formed as rint(W/s + V) + zp
    (equal in exact arithmetic; this fp32 order is the contract); round is
    torch.round, i.e. half to even.
    """
    W = _to_f32(W)
    V = _to_f32(V)
    g = _group(W.shape[1], group_size)
    Q = qmax(bits)
    se = _expand(_to_f32(s), g)
    ze = _expand(_to_f32(zp), g)
    u = W / se
    t = u + V
    r = np.rint(t)
    p = r + ze
    q = np.clip(p, F32(0), Q)
    m = (p >= 0) & (p <= Q)
    Wq = se * (q - ze)
    return FakeQuant(u, t, r, p, q, m, Wq)


def rtn(W, bits: int, group_size: int, sym: bool):
    """Round-to-nearest: V = 0, alpha = beta = 1 ("논문 핵심 내용": w^ = s*round(w/s)).

    Returns (codes uint8 [out, in], scale fp32 [out, G], zero-point int32 [out, G], W' fp32).
    """
    W = _to_f32(W)
    wmin, wmax = group_minmax(W, group_size)
    one = np.ones_like(wmin)
    s, zp = scale_zero_point(wmin, wmax, one, one, bits, sym)
    fq = fake_quant(W, np.zeros_like(W), s, zp, group_size, bits)
    return fq.q.astype(np.uint8), s, zp.astype(np.int32), fq.Wq


MSE_GRID = 51   # clip ratios p_i = (100 - i) / 100, i = 0 .. 50: 1.00 down to 0.50


def mse_init(W, group_size: int, bits: int, sym: bool):
    """Initial clip factors by an MSE grid search ("[llm-compressor] AutoRound ...",
    ``_init_scale_zp``: "Min-Max or MSE").

    The page names the option without spelling it out.  Reading: per group, try a
    common clip ratio p for both factors (alpha = beta = p; symmetric: alpha = p) on
    the grid p_i = fp32(100 - i) / fp32(100), i = 0 .. 50, i.e. 1.00 down to 0.50
    (the clip factors' range), and keep the p whose round-to-nearest weights
    (V = 0) have the smallest squared error sum_k (W'_k - W_k)^2.  The element
    arithmetic is the fp32 quantiser's; each square is exact in fp64 and the sum
    runs in fp64 over k in index order; the first minimum along the grid wins, so
    a tie keeps the wider range.

    Returns (p fp32 [out, G], err fp64 [out, G]: the squared error at p).
    """
    W = _to_f32(W)
    out, inn = W.shape
    g = _group(inn, group_size)
    wmin, wmax = group_minmax(W, g)
    zeros = np.zeros_like(W)
    best_p = np.ones(wmin.shape, dtype=F32)
    best_e = np.full(wmin.shape, np.inf)
    for i in range(MSE_GRID):
        p = F32(100 - i) / F32(100)
        a = np.full(wmin.shape, p, dtype=F32)
        sc, zp = scale_zero_point(wmin, wmax, a, a, bits, sym)
        d = fake_quant(W, zeros, sc, zp, g, bits).Wq - W              # fp32
        d2 = d.astype(F64).reshape(out, inn // g, g) ** 2             # exact squares
        e = np.cumsum(d2, axis=2)[:, :, -1]                            # sequential sum over k
        better = e < best_e
        best_e = np.where(better, e, best_e)
        best_p = np.where(better, p, best_p).astype(F32)
    return best_p, best_e


# --------------------------------------------------------------------------
# backward: straight-through derivatives of W' with respect to V, alpha, beta
# --------------------------------------------------------------------------

def step_gradients(W, V, alpha, beta, wmin, wmax, G, group_size: int, bits: int, sym: bool,
                   with_scale: bool = False):
    """Gradients of the loss at (V, alpha, beta), given G = dL/dW' up to a positive factor.

    The page's loop back-propagates through ``torch.round``; reading: a
    straight-through estimator -- every rint (the code's and the zero-point's)
    passes the gradient as the identity, and every clamp passes it only where its
    input lies inside the closed interval (torch.clamp's rule).

    Returns (sgn_dV fp32 [out, in] in {-1, 0, 1}, dalpha fp64 [out, G], dbeta fp64 [out, G]);
    with ``with_scale`` also the sums of the terms' magnitudes, sum_k |G*dW'/dalpha| and
    sum_k |G*dW'/dbeta| per group: the scale against which a rounding error in a
    group sum is measured (a sum far below it is a near-tie of its sign).
    With ds_a = ds/dalpha, ds_b = ds/dbeta:
      in range (m = 1):  W' = s*r, so dW'/dtheta = ds_theta * (r - W/s)  (zp cancels);
      clamped  (m = 0):  W' = s*(q - zp), so dW'/dtheta = ds_theta*(q - zp) - s*dzp/dtheta,
                         zp following z0 = -beta*wmin/s unless zp itself was clamped;
      dL/dV = G * s * m, and s > 0, so sign(dL/dV) = sign(G) * m.
    """
    W = _to_f32(W)
    out, inn = W.shape
    g = _group(inn, group_size)
    Q = qmax(bits)
    s, zp = scale_zero_point(wmin, wmax, alpha, beta, bits, sym)
    fq = fake_quant(W, V, s, zp, group_size, bits)

    Qd = float(Q)
    wmin64 = _to_f32(wmin).astype(F64)
    wmax64 = _to_f32(wmax).astype(F64)
    s64 = s.astype(F64)
    if sym:
        amax64 = np.maximum(-wmin64, wmax64)
        ds_a = 2.0 * amax64 / Qd
        ds_b = np.zeros_like(ds_a)
        dzp_a = np.zeros_like(ds_a)
        dzp_b = np.zeros_like(ds_a)
    else:
        ds_a = wmax64 / Qd
        ds_b = -wmin64 / Qd
        z0 = -_to_f32(beta).astype(F64) * wmin64 / s64
        rz = np.rint(-(_to_f32(beta) * _to_f32(wmin)) / s)   # the forward's pre-clamp zp
        zfree = ((rz >= 0) & (rz <= Q)).astype(F64)
        dzp_a = (-z0 * ds_a / s64) * zfree
        dzp_b = (-wmin64 / s64 - z0 * ds_b / s64) * zfree

    W64 = W.astype(F64)
    se = _expand(s64, g)
    ratio = W64 / se
    r = fq.r.astype(F64)
    qz = fq.q.astype(F64) - _expand(zp.astype(F64), g)
    m = fq.m
    dWa = np.where(m, _expand(ds_a, g) * (r - ratio), _expand(ds_a, g) * qz - se * _expand(dzp_a, g))
    dWb = np.where(m, _expand(ds_b, g) * (r - ratio), _expand(ds_b, g) * qz - se * _expand(dzp_b, g))
    G = np.asarray(G, dtype=F64)
    dalpha = (G * dWa).reshape(out, inn // g, g).sum(axis=2)
    dbeta = (G * dWb).reshape(out, inn // g, g).sum(axis=2)
    if sym:
        dbeta = np.zeros_like(dbeta)
    sgn_dV = (np.sign(G) * m).astype(F32)
    if not with_scale:
        return sgn_dV, dalpha, dbeta
    abs_a = np.abs(G * dWa).reshape(out, inn // g, g).sum(axis=2)
    abs_b = np.zeros_like(abs_a) if sym else np.abs(G * dWb).reshape(out, inn // g, g).sum(axis=2)
    return sgn_dV, dalpha, dbeta, abs_a, abs_b


# --------------------------------------------------------------------------
# the tuning loop
# --------------------------------------------------------------------------

@dataclasses.dataclass
class Step:
    """One SignSGD step of the tuning loop from a given state (see ``sign_step``)."""

    row_loss: np.ndarray     # fp64 [out]: batch MSE of each output row, mean_b (Y' - Y)_bj^2
    G: np.ndarray            # fp64 [out, in]: R^T X_b, dL/dW' up to the factor 2/(B*out)
    sgn_dV: np.ndarray       # fp32 [out, in]: sign(dL/dV) in {-1, 0, 1}
    dalpha: np.ndarray       # fp64 [out, G]
    dbeta: np.ndarray        # fp64 [out, G] (zeros when sym)
    dalpha_abs: np.ndarray | None  # fp64 [out, G]: sum_k |G*dW'/dalpha|, the scale of dalpha's rounding
    dbeta_abs: np.ndarray | None   # fp64 [out, G]
    V: np.ndarray            # fp32 [out, in]: the state after the update
    alpha: np.ndarray        # fp32 [out, G]
    beta: np.ndarray         # fp32 [out, G]


def sign_step(W, Xb, V, alpha, beta, wmin, wmax, group_size: int, bits: int, sym: bool, lr: float,
              minmax_lr: float, Xt_b=None, with_scale: bool = False, jitter=None) -> Step:
    """One step of the per-layer loop ("[llm-compressor] AutoRound ...", "on_event with
    SEQUENTIAL_EPOCH_END": fake-quantise, forward, MSE, backward, sign update).

    Xb: this step's calibration block as fp64 [B, in] (Xt_b: the target's inputs of
    the same rows, or None for Y = X_b W^T).  R = Y' - Y = X_b W'^T - X_b W^T (or
    X_b W'^T - Xt_b W^T), the row losses mean_b R_bj^2, G = R^T X_b, the
    straight-through gradients, then V <- clamp(V - lr*sign(dL/dV), -0.5, 0.5) and
    alpha, beta <- clamp(. - minmax_lr*sign(.), 0.5, 1), all from the same point.
    ``with_scale`` also fills dalpha_abs and dbeta_abs (otherwise None).
    ``jitter`` (sensitivity studies only, never parity): a callable applied to G
    before the sign decisions, see ``tune_layer(grad_jitter=...)``.
    """
    W = _to_f32(W)
    g = _group(W.shape[1], group_size)
    lr32 = F32(lr)
    mlr32 = F32(lr if minmax_lr < 0 else minmax_lr)
    s, zp = scale_zero_point(wmin, wmax, alpha, beta, bits, sym)
    Wq = fake_quant(W, V, s, zp, g, bits).Wq
    if Xt_b is None:
        R = Xb @ (Wq.astype(F64) - W.astype(F64)).T      # Y' - Y  [B, out]
    else:
        R = Xb @ Wq.astype(F64).T - Xt_b @ W.astype(F64).T
    row_loss = np.sum(R * R, axis=0) / Xb.shape[0]
    G = R.T @ Xb                                          # dL/dW' * (B*out/2)  [out, in]
    if jitter is not None:
        G = jitter(G)
    if with_scale:
        sgn_dV, dalpha, dbeta, abs_a, abs_b = step_gradients(W, V, alpha, beta, wmin, wmax, G, g, bits, sym,
                                                             with_scale=True)
    else:
        sgn_dV, dalpha, dbeta = step_gradients(W, V, alpha, beta, wmin, wmax, G, g, bits, sym)
        abs_a = abs_b = None
    V_new = np.clip(V - lr32 * sgn_dV, F32(-0.5), F32(0.5)).astype(F32)
    a_new = np.clip(alpha - mlr32 * np.sign(dalpha).astype(F32), F32(0.5), F32(1.0)).astype(F32)
    b_new = beta.copy() if sym else np.clip(beta - mlr32 * np.sign(dbeta).astype(F32), F32(0.5),
                                            F32(1.0)).astype(F32)
    return Step(row_loss, G, sgn_dV, dalpha, dbeta, abs_a, abs_b, V_new, a_new, b_new)


@dataclasses.dataclass
class TuneResult:
    codes: np.ndarray        # uint8 [out, in]: codes of the applied iterate
    scale: np.ndarray        # fp32 [out, G]
    zero_point: np.ndarray   # int32 [out, G]
    Wq: np.ndarray           # fp32 [out, in], the applied fake-quantised weight
    V: np.ndarray            # fp32 [out, in]: live state after the last update
    alpha: np.ndarray        # fp32 [out, G]
    beta: np.ndarray         # fp32 [out, G]
    loss_trace: np.ndarray   # fp64 [iters]: batch MSE at each step, before its update
    final_mse: float | None  # MSE over all calibration rows with the applied W'
    best_loss: np.ndarray    # fp64 [out]: per output row, lowest batch loss seen (inf if none)
    V_best: np.ndarray       # per row, the state at that row's best step (initial if none)
    alpha_best: np.ndarray
    beta_best: np.ndarray
    row_loss_trace: np.ndarray | None = None  # fp64 [iters, out]: each row's batch loss per step
    best_step: np.ndarray | None = None       # int64 [out]: step index (start_step-based) of the
                                              # applied best state; -1 if no step improved on best0


def tune_layer(W, X, bits: int, group_size: int, sym: bool, iters: int, lr: float,
               minmax_lr: float, batch_rows: int, seed: int, minmax_shrink: float = 1.0,
               keep_best: bool | int = True, V0=None, alpha0=None, beta0=None, start_step: int = 0,
               best0=None, want_final_mse: bool = True, init: str = "minmax", X_target=None,
               grad_jitter=None) -> TuneResult:
    """SignSGD tuning of one linear layer.

    "[llm-compressor] AutoRound ...", "on_event with SEQUENTIAL_EPOCH_END": per step,
    fake-quantise W, run the layer on a calibration batch, take the MSE against
    the full-precision output, back-propagate, then V <- clamp(V - lr*sign(dV), -0.5, 0.5)
    ("논문 핵심 내용": V <- V - eta*sign(grad_V L)).  The clip factors follow the
    same rule with minmax_lr (None -> lr, here minmax_lr < 0), clamped to [0.5, 1].
    All variables are updated together from gradients taken at the same point.
    One calibration block of ``batch_rows`` rows is used per step (see
    ``schedule.block_schedule``).  The bias cancels in Y' - Y and is not an input.

    Which iterate is applied at the end: the page's loop computes the step loss
    (``total_loss``) and then applies the final V.  With a constant lr the sign
    steps keep oscillating across rounding boundaries, and the final iterate can
    be worse than RTN.  Reading used by default (keep_best): the state with the
    lowest step loss is applied.  The loss is a sum over output rows, and a
    row's V, alpha and beta only enter its own term, so the choice is made per
    output row: row j keeps its state from the step where its batch loss
    mean_b (Y' - Y)_bj^2 was lowest.  This keeps every row's tuning independent
    of the others, and is never worse than one layer-wide choice.  Step 0, the
    min-max RTN state, is a candidate, so with one full batch the result is never
    worse than RTN.  keep_best=False applies the last state, as the page's
    listing does.  keep_best=2 makes one layer-wide choice instead: the state of
    the step whose layer batch loss (the sum over rows of the row losses) was
    lowest, every row together, as the page's loop would with its ``total_loss``
    tracked across steps.  The comparison is strict (a tie keeps the earlier
    state).  In that mode every entry of ``best_loss`` holds the layer's best.

    W: [out, in] fp32 values (or bf16 bit patterns); X: [n, in] bf16-exact values.
    ``start_step`` continues the block schedule of an interrupted run, with the
    live state passed in V0 / alpha0 / beta0 and the best state in
    best0 = (best_loss, V_best, alpha_best, beta_best).

    ``init``: "minmax" starts the clip factors at ``minmax_shrink`` (the page's
    ``minmax_shrink`` parameter); "mse" starts each group at its ``mse_init``
    ratio (minmax_shrink is then unused).

    ``X_target`` ([n, in], bf16-exact, optional): the inputs of the target output.
    The page's quant-aware mode (``enable_quanted_input``) feeds the layer the
    output of the already-quantised layers before it, while the target stays the
    captured full-precision output ``y_true``.  With X_target the batch residual
    is Y' - Y = X_b W'^T - X_target,b W^T, written out as those two products;
    without it Y = X_b W^T (the layer's own input on both sides).

    ``grad_jitter = (rel, seed)`` is not part of the method: it adds to every
    gradient G, before its sign is taken, seeded uniform noise in
    [-rel, rel] * rms(G).  That models an implementation whose gradients are exact
    only up to rel of their rms, so the loop's own drift from such an
    implementation can be measured (ties resolved the other way fork the SignSGD
    trajectory).  None (the default) is the method.
    """
    W = _to_f32(W)
    out, inn = W.shape
    n = X.shape[0]
    if X.shape[1] != inn:
        raise ValueError("X must be [n, in]")
    if batch_rows <= 0 or n % batch_rows:
        raise ValueError("n_rows must be a multiple of batch_rows")
    if iters < 0 or lr < 0:
        raise ValueError("iters and lr must be >= 0")
    g = _group(inn, group_size)
    lr32 = F32(lr)
    mlr32 = F32(lr if minmax_lr < 0 else minmax_lr)

    wmin, wmax = group_minmax(W, g)
    if init not in ("minmax", "mse"):
        raise ValueError("init must be 'minmax' or 'mse'")
    p0 = mse_init(W, g, bits, sym)[0] if init == "mse" else np.full(wmin.shape, F32(minmax_shrink))
    V = np.zeros_like(W) if V0 is None else _to_f32(V0).copy()
    alpha = p0.copy() if alpha0 is None else _to_f32(alpha0).copy()
    beta = p0.copy() if beta0 is None else _to_f32(beta0).copy()
    layer_wide = keep_best == 2 and keep_best is not True
    if best0 is None:
        best_loss = np.full(out, np.inf)
        V_best, a_best, b_best = V.copy(), alpha.copy(), beta.copy()
    else:
        best_loss = np.asarray(best0[0], dtype=F64).copy()
        V_best, a_best, b_best = (_to_f32(x).copy() for x in best0[1:])
    best_layer = float(best_loss[0]) if (layer_wide and out > 0) else np.inf

    sched = block_schedule(n // batch_rows, start_step + iters, seed)[start_step:]
    W64 = W.astype(F64)
    cache: dict[int, np.ndarray] = {}
    trace = np.zeros(iters, dtype=F64)
    row_trace = np.zeros((iters, out), dtype=F64)
    best_step = np.full(out, -1, dtype=np.int64)
    jitter = None
    if grad_jitter is not None:
        rel, jseed = grad_jitter
        jrng = np.random.default_rng(jseed)

        def jitter(G):
            rms = float(np.sqrt(np.mean(G * G)))
            return G + jrng.uniform(-1.0, 1.0, G.shape) * (rel * rms)
    for t in range(iters):
        blk = sched[t]
        if blk not in cache:
            cache[blk] = _rows_f64(X, blk * batch_rows, (blk + 1) * batch_rows)
        Xb = cache[blk]
        Xt_b = None if X_target is None else _rows_f64(X_target, blk * batch_rows, (blk + 1) * batch_rows)
        st = sign_step(W, Xb, V, alpha, beta, wmin, wmax, g, bits, sym, lr32, mlr32, Xt_b, jitter=jitter)
        row_loss = st.row_loss
        row_trace[t] = row_loss
        trace[t] = float(np.sum(row_loss)) / out
        if layer_wide:
            layer_loss = float(np.sum(row_loss))
            improved = layer_loss < best_layer
            if improved:
                best_layer = layer_loss
            better = np.full(out, improved)
            row_best = np.full(out, layer_loss)
        else:
            better = row_loss < best_loss
            row_best = row_loss
        best_loss = np.where(better, row_best, best_loss)
        best_step[better] = start_step + t
        V_best[better] = V[better]
        a_best[better] = alpha[better]
        b_best[better] = beta[better]
        V, alpha, beta = st.V, st.alpha, st.beta

    Va, aa, ba = (V_best, a_best, b_best) if keep_best else (V, alpha, beta)
    s, zp = scale_zero_point(wmin, wmax, aa, ba, bits, sym)
    fq = fake_quant(W, Va, s, zp, g, bits)
    mse = None
    if want_final_mse:
        D = fq.Wq.astype(F64) - W64
        acc = 0.0
        for r0 in range(0, n, batch_rows):
            Xb = cache.get(r0 // batch_rows)
            if Xb is None:
                Xb = _rows_f64(X, r0, r0 + batch_rows)
            if X_target is None:
                R = Xb @ D.T
            else:
                R = Xb @ fq.Wq.astype(F64).T - _rows_f64(X_target, r0, r0 + batch_rows) @ W64.T
            acc += float(np.sum(R * R))
        mse = acc / (n * out)
    return TuneResult(fq.q.astype(np.uint8), s, zp.astype(np.int32), fq.Wq, V, alpha, beta,
                      trace, mse, best_loss, V_best, a_best, b_best, row_trace, best_step)


def layer_mse(W, Wq, X) -> float:
    """Mean over rows and outputs of (X W'^T - X W^T)^2, from the two outputs directly
    (the page's ``(y_hat - y_true).pow(2).mean()``), in fp64."""
    X64 = _rows_f64(X, 0, X.shape[0])
    Y = X64 @ _to_f32(W).astype(F64).T
    Yq = X64 @ _to_f32(Wq).astype(F64).T
    return float(np.mean((Yq - Y) ** 2))
