"""The N > 1 path on CPU: two gloo ranks tune row shards of one layer and gather.

The per-rank compute here is the oracle (CPU), which makes the check exact:
the gathered result must equal one oracle run over all rows, because rows tune
independently.  On B200s the same sharding and gather run with libar and NCCL.
"""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from signed_gradient_rounding_b200.shard import row_range, tune_layer_sharded


def test_row_range_partitions():
    for out in (1, 127, 128, 300, 4096, 11008):
        for world in (1, 2, 3, 8):
            ranges = [row_range(out, r, world) for r in range(world)]
            assert ranges[0][0] == 0 and ranges[-1][1] == out
            for (a0, b0), (a1, b1) in zip(ranges, ranges[1:]):
                assert b0 == a1
            lens = [b - a for a, b in ranges]
            full = [x for x in lens if x > 0]
            assert all(x % 128 == 0 for x in lens[:-1] if x > 0) or out < 128 * world


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, W, X, result_q, group_size=32):
    import oracle
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    import datetime
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))

    def compute(Wr, Xr):
        res = oracle.tune_layer(Wr.numpy(), Xr.numpy(), 4, group_size, False, 12, 0.005, 0.005, 32, 4,
                                want_final_mse=False)
        return (torch.from_numpy(res.codes), torch.from_numpy(res.scale), torch.from_numpy(res.zero_point))

    (codes, scale, zp), rng = tune_layer_sharded(torch.from_numpy(W), torch.from_numpy(X), compute)
    # the max-over-ranks reduction the benchmark uses for its timings
    t = torch.tensor([float(rank + 1)], dtype=torch.float64)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    if rank == 0:
        result_q.put((codes.numpy(), scale.numpy(), zp.numpy(), rng, float(t.item())))
    dist.barrier()
    dist.destroy_process_group()


@pytest.mark.parametrize("group_size", [32, -1], ids=["g32", "per-channel"])
def test_two_gloo_ranks_gather_equals_single_run(group_size):
    import oracle
    from workloads import bf16_round, make_weight
    W = make_weight(300, 64, 0.02, "f32", seed=3)
    X = bf16_round(np.random.default_rng(4).standard_normal((96, 64)).astype(np.float32))
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, W, X, q, group_size)) for r in range(2)]
    for p in procs:
        p.start()
    codes, scale, zp, rng, tmax = q.get(timeout=240)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    ref = oracle.tune_layer(W, X, 4, group_size, False, 12, 0.005, 0.005, 32, 4, want_final_mse=False)
    assert rng == (0, 300)
    assert np.array_equal(codes, ref.codes)
    assert np.array_equal(scale, ref.scale)
    assert np.array_equal(zp, ref.zero_point)
    assert tmax == 2.0
