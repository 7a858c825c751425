"""Row sharding for running the MX path on several GPUs, one process per GPU.

MX blocks (32 elements) and macro blocks (128) never cross a row, so a tensor
of shape [rows, cols] splits into contiguous row ranges that ranks quantize
independently: there is no data exchange on the path. The one step with an
exchange is the error statistics of a sharded tensor (one all-reduce of
three numbers); the others are for timing (a barrier and a maximum).
"""

from __future__ import annotations

import torch


def shard_rows(rows: int, world: int, rank: int):
    """Contiguous, balanced [start, end) row range of `rank` among `world`."""
    if world < 1 or not 0 <= rank < world:
        raise ValueError("bad rank / world size")
    base, extra = divmod(rows, world)
    start = rank * base + min(rank, extra)
    return start, start + base + (1 if rank < extra else 0)


def max_over_ranks(values, device=None):
    """Element-wise maximum of a list of floats over all ranks (identity if not distributed)."""
    import torch.distributed as dist
    vals = [float(v) for v in values]
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return vals
    t = torch.tensor(vals, dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return t.tolist()


def global_error_stats(totals, n_local, device=None):
    """MSE and SQNR (dB) of a row-sharded tensor from each rank's block-error
    totals {sum d^2, sum x^2} over its n_local elements: one all-reduce (sum)
    of [sum d^2, sum x^2, n] (NCCL for device tensors, gloo on the host), then
    MSE = sum d^2 / N and SQNR = 10 log10(sum x^2 / sum d^2)."""
    import math

    import torch.distributed as dist
    vals = [float(totals[0]), float(totals[1]), float(n_local)]
    if dist.is_available() and dist.is_initialized() and dist.get_world_size() > 1:
        t = torch.tensor(vals, dtype=torch.float64, device=device)
        dist.all_reduce(t, op=dist.ReduceOp.SUM)
        vals = t.tolist()
    sd, sx, n = vals
    mse = sd / n if n else float("nan")
    sqnr = 10 * math.log10(sx / sd) if sd > 0 else float("inf")
    return mse, sqnr
