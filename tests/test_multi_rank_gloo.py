"""Multi-rank host logic of the benchmark (replicas, no data-path collective), on CPU with gloo.

Two ranks report different timings and violation counts; both must end with the max
of every timing and the sum of the violations, which is what rank 0 prints.  A second
check runs a batch-invariant stand-in op on each rank's own shard of rows and confirms
that a row's bits are the same whichever rank processed it, in whatever batch.
"""
import os
import socket

import numpy as np
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import bench
from invariant_deterministic_rmsnorm_b200 import inputs


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        times = [10.0 + rank, 20.0 - rank, 5.0 * (rank + 1)]
        got, viol = bench.reduce_over_ranks(times, rank + 2, world, torch.device("cpu"))
        # each rank processes its own shard of a global batch with a row-wise op
        rows = inputs.normal(3, (16, 32))
        shard = rows[rank::world]
        out = np.tanh(shard) * np.float32(0.5)
        q.put((rank, got, viol, [(int(i), out[j].tobytes()) for j, i in enumerate(range(rank, 16, world))]))
    finally:
        dist.destroy_process_group()


def test_two_rank_reduction_and_row_sharding():
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    results = [q.get(timeout=120) for _ in range(world)]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, got, viol, _ in results:
        assert got == [11.0, 20.0, 10.0]
        assert viol == 2 + 3
    rows = inputs.normal(3, (16, 32))
    solo = {i: (np.tanh(rows[i:i + 1]) * np.float32(0.5))[0].tobytes() for i in range(16)}
    for _, _, _, outs in results:
        for i, b in outs:
            assert b == solo[i]
