"""Row-sharded tuning of one layer over several GPUs (one process per GPU).

The tuning loss is a sum over output rows, and a row's V, alpha and beta only
enter its own term, so the rows of W tune independently: rank r tunes a
contiguous slice of rows with the same calibration activations and the same
block schedule, with no exchange during the loop.  The only collective is one
all-gather of the results at the end (optional: a caller may keep them sharded).

The tuning itself is the ``compute`` callable (libar's ``tune_layer`` on a GPU);
the sharding and the gather are plain ``torch.distributed`` and run under any
backend (NCCL on B200s, gloo in the CPU tests).
"""
from __future__ import annotations

import torch
import torch.distributed as dist

ROW_TILE = 128  # the M tile of the contractions: shards are multiples of it where possible


def row_range(out: int, rank: int, world: int, align: int = ROW_TILE) -> tuple[int, int]:
    """Contiguous, balanced [start, stop) rows of ``rank`` out of ``world``, in units of
    ``align`` rows (the last shard takes the remainder)."""
    if world < 1 or not 0 <= rank < world:
        raise ValueError("bad rank/world")
    units = -(-out // align)
    base, extra = divmod(units, world)
    u0 = rank * base + min(rank, extra)
    u1 = u0 + base + (1 if rank < extra else 0)
    return min(out, u0 * align), min(out, u1 * align)


def _gather_rows(local: torch.Tensor, out: int, world: int, group=None) -> torch.Tensor:
    """All-gather row slices of different lengths (padded to the longest).  Under the
    gloo backend device tensors travel through host memory."""
    rows_max = max(row_range(out, r, world)[1] - row_range(out, r, world)[0] for r in range(world))
    staged = local.is_cuda and dist.get_backend(group) == "gloo"
    dev = local.device
    if staged:
        local = local.cpu()
    pad = torch.zeros((rows_max,) + tuple(local.shape[1:]), dtype=local.dtype, device=local.device)
    pad[:local.shape[0]] = local
    bufs = [torch.empty_like(pad) for _ in range(world)]
    dist.all_gather(bufs, pad, group=group)
    if staged:
        bufs = [b.to(dev) for b in bufs]
    parts = []
    for r in range(world):
        a, b = row_range(out, r, world)
        parts.append(bufs[r][:b - a])
    return torch.cat(parts, dim=0)


def tune_layer_sharded(W: torch.Tensor, X: torch.Tensor, compute, gather: bool = True, group=None):
    """Tune this rank's row shard of W with ``compute(W_shard, X) -> (codes, scale, zp)``;
    return the full (codes, scale, zp) when ``gather`` else this rank's shard and its
    row range."""
    world = dist.get_world_size(group) if dist.is_initialized() else 1
    rank = dist.get_rank(group) if dist.is_initialized() else 0
    out = W.shape[0]
    a, b = row_range(out, rank, world)
    codes, scale, zp = compute(W[a:b].contiguous(), X)
    if not gather or world == 1:
        return (codes, scale, zp), (a, b)
    return tuple(_gather_rows(t, out, world, group) for t in (codes, scale, zp)), (0, out)
