"""Multi-rank host logic of bench.py on CPU: world-size-2 gloo ranks.

The layer is data-parallel over independent batches (weak scaling, no
data-path collective); what crosses ranks is the timing protocol: a barrier
on both sides of the timed region and the max over ranks of the device time.
These tests run that protocol with gloo on CPU.
"""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world),
                      LOCAL_RANK=str(rank))
    import datetime
    import bench
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        r, w, l = bench.dist_env()
        assert (r, w, l) == (rank, world, rank)
        bench.barrier(w, torch.device("cpu"))
        my_ms = 10.0 * (rank + 1)                  # rank 1 is the slow one
        mx = bench.reduce_max(my_ms, w, torch.device("cpu"))
        bench.barrier(w, torch.device("cpu"))
        # the reference arm: only rank 0 works and prints; the others return nothing
        ref = None
        if rank != 0:
            ref = bench.run_reference(None, None, rank, w)
        q.put((rank, mx, ref))
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_and_barriers_gloo():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    got = sorted(q.get(timeout=5) for _ in range(2))
    assert [g[1] for g in got] == [20.0, 20.0]      # every rank sees the slowest rank's time
    assert got[1][2] is None                        # rank 1 does no reference work


def test_single_rank_reduce_is_identity():
    import bench
    assert bench.reduce_max(3.5, 1) == 3.5
    bench.barrier(1)


def test_weak_scaling_value_counts_all_ranks():
    # value = tokens processed by all ranks / max-over-ranks time
    T, world, ms = 32768, 4, 2.5
    assert abs(T * world / (ms * 1e-3) - 52_428_800.0) < 1.0
