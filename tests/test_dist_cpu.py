"""Multi-rank host logic on CPU: world-size-2 gloo ranks.

The layer is data-parallel over independent batches (weak scaling, no
data-path collective); what crosses ranks is the timing protocol (a barrier
on both sides of the timed region and the max over ranks of the device time)
and, optionally, the balance loss of the whole batch (one all-reduce of the
2E statistics).  These tests run both with gloo on CPU; the statistics come
from the oracle in place of the kernels.
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


class _OracleLayer:
    """Stands in for MoELayer on CPU: the statistics and the loss come from the oracle."""

    def __init__(self, idx, P, E, K, alpha, seq_len=0):
        import types
        self.idx, self.P, self.E, self.K, self.alpha = idx, P, E, K, alpha
        self.s = types.SimpleNamespace(E=E, seq_len=seq_len)
        self.cfg = types.SimpleNamespace(T=P.shape[0])

    def balance_stats(self, out=None):
        from oracle import moe_oracle as O
        st = torch.tensor(O.balance_stats(self.idx, self.P, self.E), dtype=torch.float64)
        if out is None:
            return st
        out.copy_(st)
        return out

    def balance_loss_from_stats(self, stats, T_total):
        from oracle import moe_oracle as O
        self.aux = torch.tensor([O.balance_loss_from_stats(stats.numpy(), self.K, T_total, self.alpha)],
                                dtype=torch.float32)
        return self.aux


def _batch(T, E, K, seed):
    import numpy as np
    from oracle import moe_oracle as O
    rng = np.random.default_rng(seed)
    skew = np.zeros(E)
    skew[0] = 2.0                                   # rank 1's half leans on expert 0
    l = rng.standard_normal((2 * T, E))
    l[T:] += skew
    P = O.softmax_scores(l)
    idx, _ = O.topk_route(P, K)
    return P, idx


def _loss_worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    import datetime
    from sparse_moe_layer_03_b200.layer import global_balance_loss
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        T, E, K, alpha = 40, 8, 2, 0.01
        P, idx = _batch(T, E, K, 71)
        mine = slice(rank * T, (rank + 1) * T)
        layer = _OracleLayer(idx[mine], P[mine], E, K, alpha)
        own = float(layer.balance_loss_from_stats(layer.balance_stats(), T)[0])
        glob = float(global_balance_loss(layer)[0])
        again = float(global_balance_loss(layer)[0])            # reuses the stats buffer
        q.put((rank, own, glob, again))
    finally:
        dist.destroy_process_group()


def test_global_balance_loss_gloo():
    from oracle import moe_oracle as O
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_loss_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    got = sorted(q.get(timeout=5) for _ in range(2))
    T, E, K, alpha = 40, 8, 2, 0.01
    P, idx = _batch(T, E, K, 71)
    whole = O.balance_loss(O.expert_counts(idx, E), P, K, alpha)
    for rank, own, glob, again in got:
        assert abs(glob - whole) <= 1e-6 * whole and glob == again
    assert got[0][2] == got[1][2]                   # every rank holds the same value
    # the ranks' own losses differ from the batch's, and so does their mean
    assert abs((got[0][1] + got[1][1]) / 2 - whole) > 1e-3 * whole


def test_global_balance_loss_single_process_and_seq_len():
    from sparse_moe_layer_03_b200.layer import global_balance_loss
    from oracle import moe_oracle as O
    T, E, K, alpha = 40, 8, 2, 0.01
    P, idx = _batch(T, E, K, 72)
    layer = _OracleLayer(idx[:T], P[:T], E, K, alpha)
    assert not dist.is_initialized()
    got = float(global_balance_loss(layer)[0])      # no process group: the call's own loss
    assert abs(got - O.balance_loss(O.expert_counts(idx[:T], E), P[:T], K, alpha)) < 1e-9
    with pytest.raises(ValueError):
        global_balance_loss(_OracleLayer(idx[:T], P[:T], E, K, alpha, seq_len=10))
