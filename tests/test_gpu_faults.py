"""Failure detection on the GPU, without a GPU fault.

* Canaries: every output is written through a view into a larger buffer whose
  padding before and after holds a fixed pattern; after each call the padding
  must be untouched (no store lands outside its output).
* Injected host failures (the AR_FAULT test hook): the call returns its status,
  outputs filled with a canary pattern are untouched, and the next call without
  the hook gives the same results as a call that never saw a failure.
* Device bounds checks (AR_CHECKS=1): a clean run is bit-identical to an
  unchecked one and reports AR_OK; with AR_FAULT=bounds the step kernels are told
  V and D are one element shorter than they are, refuse that store instead of
  making it, and the workspace status reads AR_ECHECK -- the context stays usable.
None of these makes a kernel trap, fault or hang.
"""
import numpy as np
import pytest
import torch

from workloads import make_activations, make_weight

pytestmark = pytest.mark.gpu

PAD = 256
CANARY = 0xA5


@pytest.fixture(scope="module")
def ar():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    import signed_gradient_rounding_b200 as ar
    return ar


def _guarded(shape, dtype):
    """A tensor of `shape` viewed inside a byte buffer with PAD canary bytes on each side."""
    n = int(np.prod(shape)) * torch.empty((), dtype=dtype).element_size()
    raw = torch.full((n + 2 * PAD,), CANARY, dtype=torch.uint8, device="cuda")
    return raw, raw[PAD:PAD + n].view(dtype).view(shape)


def _canaries_intact(raw):
    head, tail = raw[:PAD], raw[-PAD:]
    return bool((head == CANARY).all().item() and (tail == CANARY).all().item())


CASES = {
    "gram_g128": dict(out=200, inn=384, n=1536, B=512, bits=4, g=128, algo="gram"),
    "direct_g64": dict(out=200, inn=320, n=1024, B=512, bits=3, g=64, algo="direct"),
    "gram_per_channel": dict(out=130, inn=384, n=1024, B=512, bits=2, g=-1, algo="gram"),
}


def _case(ar, name, iters=12):
    c = CASES[name]
    W = torch.from_numpy(make_weight(c["out"], c["inn"], 0.02, "bf16", seed=61)).to(torch.bfloat16).cuda()
    X = torch.from_numpy(make_activations(c["n"], c["inn"], "llm", seed=61)).to(torch.bfloat16).cuda()
    p = ar.make_params(bits=c["bits"], group_size=c["g"], iters=iters, batch_rows=c["B"], algo=c["algo"])
    return c, W, X, p


def _guarded_outputs(c, p):
    G = c["inn"] // (c["inn"] if c["g"] == -1 else c["g"])
    specs = [((c["out"], c["inn"]), torch.uint8), ((c["out"], G), torch.float32), ((c["out"], G), torch.int32),
             ((p.iters,), torch.float32), ((1,), torch.float64)]
    raws, views = zip(*(_guarded(s, d) for s, d in specs))
    return list(raws), tuple(views)


@pytest.mark.parametrize("name", sorted(CASES))
def test_tuning_outputs_stay_inside_their_buffers(ar, name):
    c, W, X, p = _case(ar, name)
    ref = ar.tune_layer(W, X, p)
    raws, outs = _guarded_outputs(c, p)
    res = ar.tune_layer(W, X, p, outputs=outs)
    assert ar.tune_status(res.workspace) == ar.AR_OK
    assert all(_canaries_intact(r) for r in raws)
    assert torch.equal(outs[0], ref.codes) and torch.equal(outs[1], ref.scale)
    assert torch.equal(outs[2], ref.zero_point) and torch.equal(outs[4], ref.final_mse)


def test_rtn_and_pack_outputs_stay_inside_their_buffers(ar):
    W = torch.from_numpy(make_weight(37, 96, 0.02, "bf16", seed=62)).to(torch.bfloat16).cuda()
    codes, scale, zp = ar.rtn(W, 3, 32)
    rc, c2 = _guarded((37, 96), torch.uint8)
    rs, s2 = _guarded((37, 3), torch.float32)
    rz, z2 = _guarded((37, 3), torch.int32)
    assert ar.lib.ar_rtn(ar._ptr(W), ar.AR_BF16, 37, 96, 3, 32, 0, ar._ptr(c2), ar._ptr(s2), ar._ptr(z2),
                         ar._stream(None)) == ar.AR_OK
    rp, p2 = _guarded((37, 96 * 3 // 32), torch.int32)
    assert ar.lib.ar_pack(ar._ptr(c2), 37, 96, 3, ar._ptr(p2), ar._stream(None)) == ar.AR_OK
    torch.cuda.synchronize()
    assert all(_canaries_intact(r) for r in (rc, rs, rz, rp))
    assert torch.equal(c2, codes) and torch.equal(s2, scale) and torch.equal(z2, zp)
    assert torch.equal(p2, ar.pack(codes, 3))


@pytest.mark.parametrize("fault,status", [("param", 1), ("alloc", 3), ("launch", 4)])
@pytest.mark.parametrize("name", ["gram_g128", "direct_g64"])
def test_injected_failure_leaves_outputs_and_recovers(ar, monkeypatch, name, fault, status):
    c, W, X, p = _case(ar, name)
    ref = ar.tune_layer(W, X, p)
    torch.cuda.synchronize()
    raws, outs = _guarded_outputs(c, p)
    monkeypatch.setenv("AR_FAULT", fault)
    with pytest.raises(ar.ArError) as e:
        ar.tune_layer(W, X, p, workspace=ref.workspace, outputs=outs)
    assert e.value.status == status
    torch.cuda.synchronize()
    # nothing was written: every byte of every output buffer still holds the canary
    assert all(bool((r == CANARY).all().item()) for r in raws)
    monkeypatch.delenv("AR_FAULT")
    res = ar.tune_layer(W, X, p, workspace=ref.workspace, outputs=outs)
    assert ar.tune_status(res.workspace) == ar.AR_OK
    assert torch.equal(outs[0], ref.codes) and torch.equal(outs[1], ref.scale)
    assert torch.equal(outs[2], ref.zero_point) and torch.equal(outs[3], ref.loss_trace)


@pytest.mark.parametrize("name", sorted(CASES))
def test_checked_run_is_identical(ar, monkeypatch, name):
    c, W, X, p = _case(ar, name)
    ref = ar.tune_layer(W, X, p)
    torch.cuda.synchronize()
    monkeypatch.setenv("AR_CHECKS", "1")
    res = ar.tune_layer(W, X, p)
    assert ar.tune_status(res.workspace) == ar.AR_OK
    assert torch.equal(res.codes, ref.codes) and torch.equal(res.scale, ref.scale)
    assert torch.equal(res.zero_point, ref.zero_point) and torch.equal(res.loss_trace, ref.loss_trace)


@pytest.mark.parametrize("name", sorted(CASES))
def test_bounds_check_refuses_and_reports(ar, monkeypatch, name):
    c, W, X, p = _case(ar, name)
    ref = ar.tune_layer(W, X, p)
    torch.cuda.synchronize()
    monkeypatch.setenv("AR_CHECKS", "1")
    monkeypatch.setenv("AR_FAULT", "bounds")
    bad = ar.tune_layer(W, X, p, workspace=ref.workspace)
    assert ar.tune_status(bad.workspace) == ar.AR_ECHECK
    monkeypatch.delenv("AR_FAULT")
    monkeypatch.delenv("AR_CHECKS")
    # the status word is per call: the next call on the same workspace starts clean
    res = ar.tune_layer(W, X, p, workspace=ref.workspace)
    assert ar.tune_status(res.workspace) == ar.AR_OK
    assert torch.equal(res.codes, ref.codes) and torch.equal(res.scale, ref.scale)
