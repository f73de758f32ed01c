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


def test_bench_two_ranks_runs_its_multi_rank_path():
    """bench.py --gpus 2 under torchrun: both ranks tune their row shard of one
    512-row layer, all-gather the results and reduce their times; the backend is
    gloo (AR_BENCH_BACKEND) because both ranks share this one GPU, so the line's
    times mean nothing here, only that the path runs and reports the whole layer."""
    import json
    import subprocess
    import sys
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    env = dict(os.environ, AR_BENCH_BACKEND="gloo")
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node", "2",
           "--master-addr", "127.0.0.1", "--master-port", str(_free_port()), "bench.py", "--gpus", "2",
           "--steps", "2", "--warmup", "3", "--workload", "tiny", "--e2e-steps", "1"]
    out = subprocess.run(["timeout", "-k", "30", "300", *cmd], cwd=root, env=env, capture_output=True,
                         text=True)
    assert out.returncode == 0, out.stderr[-3000:]
    lines = [ln for ln in out.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1, out.stdout[-3000:]
    line = json.loads(lines[0])
    assert line["n_gpus"] == 2 and line["scaling"] == "weak"
    assert line["config"]["out"] == 512 and "2 row shards" in line["config"]["workload"]
    assert line["value"] > 0 and line["e2e"]["value"] > 0
    assert line["gpu_launches"] > 0
    assert np.isfinite(line["final_mse"])
