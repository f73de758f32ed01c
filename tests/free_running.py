"""The free-running code bound of the full-size parity tests.

Over 200 SignSGD steps the tuning loop is chaotic: a gradient sign that sits
within rounding of zero and is resolved the other way moves one offset by 2*lr,
and the trajectories part from there on.  test_gpu_steplocked.py shows, one
step at a time from the GPU's own state, that every move of the GPU equals the
oracle's except where |G| is within TIE_BAND of its rms.  How far two runs that
differ only there drift apart is a property of the loop itself; it is measured
here with the oracle alone, by running it once more with every gradient jittered
by seeded uniform noise of TIE_BAND * rms(G) (oracle.tune_layer's grad_jitter),
and the GPU's free-running drift must stay within MARGIN times that, plus the
granularity of the row sample: a row whose best step (keep-best) differs from the
oracle's differs in 20-45% of its codes (measured), so one such row among n
sampled rows moves the fraction by about ROW_GRANULE / n.  The bound is never
below the stated 0.5%.
"""
import numpy as np

import oracle

CODE_TOL = 0.005   # the stated bar: at most 0.5% of the codes differ
TIE_BAND = 1e-5    # the tie band of the step-locked checks (fraction of rms(G))
MARGIN = 2.0
ROW_GRANULE = 0.5  # about half of one sampled row's codes


def oracle_drift(ref, W_rows, X, bits, group_size, sym, iters, lr, minmax_lr, batch_rows, seed=0, **kw):
    """Fraction of codes by which the jittered oracle run differs from ``ref``."""
    jit = oracle.tune_layer(W_rows, X, bits, group_size, sym, iters, lr, minmax_lr, batch_rows, seed,
                            want_final_mse=False, grad_jitter=(TIE_BAND, 1), **kw)
    return float(np.mean(jit.codes != ref.codes))


def code_bound(drift: float, n_rows: int) -> float:
    """The free-running code bound for a sample of n_rows output rows."""
    return max(CODE_TOL, MARGIN * drift + ROW_GRANULE / n_rows)
