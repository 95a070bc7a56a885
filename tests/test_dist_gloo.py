"""Multi-rank host logic on CPU (gloo, world size 2): shard coverage, the
max-over-ranks timing reduction, and the weight-gradient all-reduce of a
d = 64 ensemble split across ranks (each rank differentiates its shard with
the CPU oracle; the reduced dW must equal the single-process one)."""
import os
import socket

import numpy as np
import pytest
import torch.multiprocessing as mp

from discrete_adjoint_b200.dist import shard


def test_shard_covers_every_trajectory_once():
    for n in (0, 1, 7, 1000, 1 << 20):
        for world in (1, 2, 3, 8):
            seen = []
            for r in range(world):
                s, c = shard(n, r, world)
                seen.extend(range(s, s + c))
            assert seen == list(range(n))
    with pytest.raises(ValueError):
        shard(10, 2, 2)


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    import torch
    import torch.distributed as dist

    import oracle
    import workloads as W
    from discrete_adjoint_b200.dist import allreduce_shared_grad, max_over_ranks, shard

    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        prob = W.node64(12, dtype="f64").as_dtype("f64")
        s, c = shard(prob.n, rank, world)
        mine = prob.subset(np.arange(s, s + c))
        om = oracle.record(mine, 64, nthreads=1)
        g = oracle.grad(mine, om, nthreads=1)
        dW = torch.tensor(g["dW"])
        allreduce_shared_grad(dW)
        t = max_over_ranks([float(rank + 1), -float(rank)])
        out[rank] = (dW.numpy().copy(), t)
    finally:
        dist.destroy_process_group()


def test_weight_gradient_allreduce_two_ranks():
    import oracle
    import workloads as W
    world = 2
    mgr = mp.get_context("spawn").Manager()
    out = mgr.dict()
    mp.start_processes(_worker, args=(world, _free_port(), out), nprocs=world, join=True, start_method="spawn")
    prob = W.node64(12, dtype="f64").as_dtype("f64")
    om = oracle.record(prob, 64, nthreads=1)
    ref = oracle.grad(prob, om, nthreads=1)["dW"]
    for r in range(world):
        dW, t = out[r]
        assert np.abs(dW - ref).max() <= 1e-12 * np.abs(ref).max()
        assert t == [2.0, 0.0]
