"""Multi-rank host logic on CPU (gloo, world size 2).

Each rank quantizes its contiguous row shard with the oracle; gathering the
shards must reproduce the whole-tensor result bit for bit (rows are
independent, so no exchange is needed), and the timing reduction returns the
maximum over ranks.
"""

import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from fp8_quantization_mx_b200.sharding import max_over_ranks, shard_rows


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _worker(rank, world, port, x_bits, scaling, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    import oracle
    r0, r1 = shard_rows(x_bits.shape[0], world, rank)
    c, s, m = oracle.quantize(np.ascontiguousarray(x_bits[r0:r1]), 0, scaling)
    parts = [None] * world
    dist.all_gather_object(parts, (r0, r1, c, s, m))
    t = max_over_ranks([float(rank + 1), -float(rank)])
    if rank == 0:
        out.put((parts, t))
    dist.barrier()
    dist.destroy_process_group()


def test_shard_rows_partition():
    for rows in (0, 1, 7, 196608):
        for world in (1, 2, 3, 8):
            spans = [shard_rows(rows, world, r) for r in range(world)]
            assert spans[0][0] == 0 and spans[-1][1] == rows
            assert all(a[1] == b[0] for a, b in zip(spans, spans[1:]))
            sizes = [e - s for s, e in spans]
            assert max(sizes) - min(sizes) <= 1
    with pytest.raises(ValueError):
        shard_rows(10, 2, 2)


@pytest.mark.parametrize("scaling", [0, 3, 16])
def test_two_rank_shards_match_whole_tensor(oracle_mod, scaling):
    from fp8_quantization_mx_b200 import inputs
    x = inputs.bf16_bits_numpy(inputs.heavy_tail(rows=37, cols=512, seed=9))
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, x, scaling, q)) for r in range(2)]
    for p in procs:
        p.start()
    parts, t = q.get(timeout=120)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    c_full, s_full, m_full = oracle_mod.quantize(x, 0, scaling)
    for r0, r1, c, s, m in parts:
        assert np.array_equal(c, c_full[r0:r1]) and np.array_equal(s, s_full[r0:r1])
        if m_full is not None:
            assert np.array_equal(m, m_full[r0:r1])
    assert sum(p[1] - p[0] for p in parts) == 37
    assert t == [2.0, 0.0]


def _err_worker(rank, world, port, x_bits, scaling, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    import oracle
    from fp8_quantization_mx_b200.sharding import global_error_stats
    r0, r1 = shard_rows(x_bits.shape[0], world, rank)
    _, sd, sx = oracle.block_error(np.ascontiguousarray(x_bits[r0:r1]), 0, scaling, want_blocks=False)
    mse, sqnr = global_error_stats((sd, sx), (r1 - r0) * x_bits.shape[1])
    out.put((rank, mse, sqnr))
    dist.barrier()
    dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 3])
def test_sharded_error_stats_equal_the_whole_tensor(oracle_mod, world):
    """The one exchange on the path: each rank's {sum d^2, sum x^2, n}
    all-reduced gives the whole tensor's MSE and SQNR."""
    from fp8_quantization_mx_b200 import inputs
    x = inputs.bf16_bits_numpy(inputs.heavy_tail(rows=41, cols=512, seed=10))
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_err_worker, args=(r, world, port, x, 3, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = [q.get(timeout=120) for _ in range(world)]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    _, sd, sx = oracle_mod.block_error(x, 0, 3, want_blocks=False)
    mse_full, sqnr_full = sd / x.size, 10 * np.log10(sx / sd)
    for _, mse, sqnr in res:
        assert np.isclose(mse, mse_full, rtol=1e-12) and np.isclose(sqnr, sqnr_full, rtol=1e-12)


def _bat_worker(rank, world, port, x_bits, params, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    import oracle
    r0, r1 = shard_rows(x_bits.shape[0], world, rank)
    A, B, bmin, bmax = params
    c, s, _ = oracle.bat_quantize(np.ascontiguousarray(x_bits[r0:r1]), A.shape[0], A, B, bmin, bmax)
    parts = [None] * world
    dist.all_gather_object(parts, (r0, r1, c, s))
    if rank == 0:
        out.put(parts)
    dist.barrier()
    dist.destroy_process_group()


def test_two_rank_batquant_shards_match_whole_tensor(oracle_mod):
    """BATQuant's parameters belong to column blocks: every rank passes the
    same A, B and thresholds with its own rows, and the gathered result is
    the whole tensor's."""
    from fp8_quantization_mx_b200 import inputs
    x = inputs.bf16_bits_numpy(inputs.outlier_act(rows=29, cols=256, seed=5))
    params = tuple(None if t is None else t.numpy() for t in inputs.bat_params(8, 256 // 32, seed=2))
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_bat_worker, args=(r, 2, port, x, params, q)) for r in range(2)]
    for p in procs:
        p.start()
    parts = q.get(timeout=120)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    A, B, bmin, bmax = params
    c_full, s_full, _ = oracle_mod.bat_quantize(x, 8, A, B, bmin, bmax)
    for r0, r1, c, s in parts:
        assert np.array_equal(c, c_full[r0:r1]) and np.array_equal(s, s_full[r0:r1])
    assert sum(p[1] - p[0] for p in parts) == 29
