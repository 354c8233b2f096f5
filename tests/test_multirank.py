"""The N > 1 bench path on CPU: two gloo ranks, as torchrun would start them.

Each rank times its own independent layer (seed + rank, no data-path
collective); the job time is the max over ranks and the job-wide ms/layer is
that max divided by the number of layers finished per step (one per rank).
"""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world),
                      LOCAL_RANK=str(rank))
    import bench
    from tests import gen
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        assert bench.dist_env() == (rank, world, rank)
        w = bench.layer_workload(gen.WORKLOADS["llama3_8b_128k"], rank)
        ms = bench.reduce_max([10.0 + rank, 3.0 - rank], dist, torch.device("cpu"))
        dist.barrier()
        out[rank] = (w.seed, ms[0], ms[1], bench.job_value(ms[0], world))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_independent_layers_and_max_timing():
    world = 2
    port = _free_port()
    with mp.get_context("spawn").Manager() as m:
        out = m.dict()
        mp.spawn(_rank_main, args=(world, port, out), nprocs=world, join=True)
        res = dict(out)
    base_seed = __import__("tests.gen", fromlist=["WORKLOADS"]).WORKLOADS["llama3_8b_128k"].seed
    assert res[0][0] == base_seed and res[1][0] == base_seed + 1  # independent layers
    for r in range(world):
        assert res[r][1] == pytest.approx(11.0)   # max over ranks
        assert res[r][2] == pytest.approx(3.0)
        assert res[r][3] == pytest.approx(5.5)    # job-wide ms per layer


def test_single_rank_is_identity():
    import bench
    assert bench.reduce_max([1.5, 2.5], None, torch.device("cpu")) == [1.5, 2.5]
    assert bench.job_value(7.0, 1) == 7.0
