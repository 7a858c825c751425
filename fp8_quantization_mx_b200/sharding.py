"""Row sharding for running the MX path on several GPUs, one process per GPU.

MX blocks (32 elements) and macro blocks (128) never cross a row, so a tensor
of shape [rows, cols] splits into contiguous row ranges that ranks quantize
independently: there is no data exchange on the path. The only collectives
are for timing (a barrier and a maximum over ranks).
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
