"""The quantiser's fast correctly rounded division against CUDA's IEEE division.

The fake-quantiser needs u = W/s rounded once to fp32 (its integer codes follow
from rint(u + V)).  When every weight of the layer is zero or at least 2^-100 in
magnitude, it forms u from the group's correctly rounded reciprocal with one
fma residual correction (Markstein, 1990).  Here both forms run through
ar_selftest_division over:
  * every finite bf16 weight against scales drawn the way the quantiser makes
    them (min-max ranges of N(0, sigma) groups, clip factors in [0.5, 1],
    2^b - 1 levels) and against edge scales (powers of two, all-ones
    significands, values next to powers of two);
  * random fp32 numerators of every exponent against random normal scales;
and every pair must agree bit for bit.
"""
import numpy as np
import pytest
import torch

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def ar():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    import signed_gradient_rounding_b200 as ar
    return ar


def _run(ar, a: np.ndarray, b: np.ndarray):
    import ctypes
    ad = torch.from_numpy(a.astype(np.float32)).cuda()
    bd = torch.from_numpy(b.astype(np.float32)).cuda()
    bad = torch.zeros(1, dtype=torch.int64, device="cuda")
    first = torch.zeros(2, dtype=torch.float32, device="cuda")
    st = ar._lib.ar_selftest_division(ctypes.c_void_p(ad.data_ptr()), ad.numel(), ctypes.c_void_p(bd.data_ptr()),
                                      bd.numel(), ctypes.c_void_p(bad.data_ptr()), ctypes.c_void_p(first.data_ptr()),
                                      None)
    assert st == ar.AR_OK
    torch.cuda.synchronize()
    return int(bad.item()), first.cpu().numpy()


def _realistic_scales(n, seed):
    rng = np.random.default_rng(seed)
    out = []
    for bits in (2, 3, 4, 8):
        Q = np.float32(2 ** bits - 1)
        sigma = np.float32(10.0) ** rng.uniform(-4, 0, n).astype(np.float32)
        w = rng.standard_normal((n, 128)).astype(np.float32) * sigma[:, None]
        wmin = np.minimum(w.min(axis=1), 0).astype(np.float32)
        wmax = np.maximum(w.max(axis=1), 0).astype(np.float32)
        al = rng.uniform(0.5, 1.0, n).astype(np.float32)
        be = rng.uniform(0.5, 1.0, n).astype(np.float32)
        out.append(((al * wmax - be * wmin) / Q).astype(np.float32))
    return np.concatenate(out)


def _edge_scales():
    e = np.arange(-60, 61, dtype=np.float32)
    pw = np.float32(2.0) ** e
    ones = np.float32(2.0) ** e * np.float32(2 - 2 ** -23)           # 1.11...1 significands
    nxt = np.nextafter(pw, np.float32(np.inf)).astype(np.float32)
    prv = np.nextafter(pw, np.float32(0)).astype(np.float32)
    thirds = (np.float32(1) / np.float32(3)) * pw
    return np.concatenate([pw, ones, nxt, prv, thirds, -pw[:8]]).astype(np.float32)


def _all_bf16():
    bits = np.arange(1 << 16, dtype=np.uint32) << 16
    x = bits.view(np.float32)
    return x[np.isfinite(x)]


def test_every_bf16_weight_realistic_scales(ar):
    bad, first = _run(ar, _all_bf16(), _realistic_scales(256, 0))
    assert bad == 0, f"{bad} mismatches, first at a={first[0]!r} b={first[1]!r}"


def test_every_bf16_weight_edge_scales(ar):
    bad, first = _run(ar, _all_bf16(), _edge_scales())
    assert bad == 0, f"{bad} mismatches, first at a={first[0]!r} b={first[1]!r}"


def test_random_fp32(ar):
    rng = np.random.default_rng(7)
    a = rng.integers(0, 1 << 32, 1 << 20, dtype=np.uint64).astype(np.uint32).view(np.float32)
    a = a[np.isfinite(a)]
    b = rng.integers(0, 1 << 32, 1 << 12, dtype=np.uint64).astype(np.uint32).view(np.float32)
    b = b[np.isfinite(b)]
    bad, first = _run(ar, a, b)
    assert bad == 0, f"{bad} mismatches, first at a={first[0]!r} b={first[1]!r}"


@pytest.mark.parametrize("algo", ["direct", "gram"])
def test_tuning_with_tiny_and_zero_weights(ar, algo):
    """A layer with nonzero weights below 2^-100 takes the IEEE division in every
    pass (the fast form's domain check fails); with a zero group as well, the
    tuned result still meets the parity bars against the oracle."""
    import oracle
    from workloads import TINY, make_activations, make_weight
    c = TINY
    W = make_weight(c.out, c.inn, c.w_std, "f32", seed=3)
    W[5, 3] = np.float32(1e-35)              # below 2^-100: no fast division anywhere
    W[6, 10] = np.float32(-3e-38)
    W[7, 64:128] = 0.0                       # an all-zero group
    X = make_activations(c.n_rows, c.inn, c.x_kind, seed=3)
    p = ar.make_params(bits=c.bits, group_size=c.group_size, iters=30, batch_rows=c.batch_rows, algo=algo)
    res = ar.tune_layer(torch.from_numpy(W).cuda(), torch.from_numpy(X).to(torch.bfloat16).cuda(), p)
    assert ar.tune_status(res.workspace) == ar.AR_OK
    ref = oracle.tune_layer(W, X, c.bits, c.group_size, False, 30, 0.005, -1.0, c.batch_rows, 0)
    codes = res.codes.cpu().numpy()
    assert float(np.mean(codes != ref.codes)) <= 0.005
    assert float(res.final_mse.item()) == pytest.approx(ref.final_mse, rel=0.02)
    assert np.all(codes[7, 64:128] == ref.codes[7, 64:128])
