"""Row-sharded tuning of one layer with libar: the N > 1 path, run here on one GPU.

The tuning loss is a sum over output rows and a row's V, alpha and beta enter only
its own term ("[llm-compressor] AutoRound ...", "on_event with
SEQUENTIAL_EPOCH_END": the per-layer loss |W'x - Wx|^2), so rows tune
independently and a layer splits into row shards with no exchange during the
loop.  Two spawned processes, each one gloo rank on cuda:0, tune their
shard.row_range slice of one layer with libar's tune_layer and all-gather the
results (CPU tensors over gloo); the gathered codes, scales and zero-points must
equal one libar run over all rows bit for bit.  The two processes share the GPU
but never wait on each other's kernels: the only exchange is the final gather,
on the host.
"""
import datetime
import os
import socket

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

pytestmark = pytest.mark.gpu

CASES = {
    "gram_g128": dict(out=512, inn=1024, n=4096, B=1024, bits=4, g=128, algo="gram", iters=24),
    "direct_per_channel": dict(out=384, inn=512, n=2048, B=512, bits=2, g=-1, algo="direct", iters=24),
}


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _inputs(c):
    from workloads import make_activations, make_weight
    W = make_weight(c["out"], c["inn"], 0.02, "bf16", seed=51)
    X = make_activations(c["n"], c["inn"], "llm", seed=51)
    return W, X


def _params(ar, c):
    return ar.make_params(bits=c["bits"], group_size=c["g"], iters=c["iters"], batch_rows=c["B"], seed=3,
                          algo=c["algo"])


def _worker(rank, world, port, name, q):
    import torch.distributed as dist

    import signed_gradient_rounding_b200 as ar
    from signed_gradient_rounding_b200.shard import tune_layer_sharded

    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    torch.cuda.set_device(0)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=120))
    c = CASES[name]
    W, X = _inputs(c)
    Xd = torch.from_numpy(X).to(torch.bfloat16).cuda()
    p = _params(ar, c)

    def compute(W_shard, X_dev):
        res = ar.tune_layer(W_shard.to(torch.bfloat16).cuda(), X_dev, p, want_final_mse=False)
        assert ar.tune_status(res.workspace) == ar.AR_OK
        return res.codes.cpu(), res.scale.cpu(), res.zero_point.cpu()

    (codes, scale, zp), rng = tune_layer_sharded(torch.from_numpy(W), Xd, compute)
    if rank == 0:
        q.put((codes.numpy(), scale.numpy(), zp.numpy(), rng))
    dist.barrier()
    dist.destroy_process_group()


@pytest.mark.parametrize("name", sorted(CASES))
def test_two_ranks_on_libar_equal_one_run(name):
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, name, q)) for r in range(2)]
    for pr in procs:
        pr.start()
    try:
        codes, scale, zp, rng = q.get(timeout=300)
    finally:
        for pr in procs:
            pr.join(timeout=120)
    assert all(pr.exitcode == 0 for pr in procs)

    import signed_gradient_rounding_b200 as ar
    c = CASES[name]
    W, X = _inputs(c)
    ref = ar.tune_layer(torch.from_numpy(W).to(torch.bfloat16).cuda(), torch.from_numpy(X).to(torch.bfloat16).cuda(),
                        _params(ar, c), want_final_mse=False)
    assert ar.tune_status(ref.workspace) == ar.AR_OK
    assert rng == (0, c["out"])
    assert np.array_equal(codes, ref.codes.cpu().numpy())
    assert np.array_equal(scale, ref.scale.cpu().numpy())
    assert np.array_equal(zp, ref.zero_point.cpu().numpy())
