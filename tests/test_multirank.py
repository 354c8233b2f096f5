"""The N > 1 path on CPU: gloo ranks, as torchrun would start them.

One layer is split across ranks by (batch element, KV group) units with no
exchange step (block_sparse_attention_band_b200.shard).  These tests check the
host logic every rank runs: the units of all ranks tile the layer exactly
once, each run's pointer offsets and per-sequence lengths address its own
heads, and the job time is the max over ranks while counts are summed.
"""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from block_sparse_attention_band_b200 import shard


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


SHAPES = [(1, 32, 8, 131072, None), (3, 4, 2, 1000, [1000, 1, 513]), (2, 6, 3, 640, None)]


def _rank_main(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world),
                      LOCAL_RANK=str(rank))
    import bench
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        assert bench.dist_env() == (rank, world, rank)
        mine = []
        for (b, hq, hkv, n, lens) in SHAPES:
            runs = shard.shard_runs(b, hkv, world, rank)
            mine.append([(r.batch, r.kv0, r.kv1, shard.run_offsets(r, hq, hkv, n), shard.run_seqlens(r, lens))
                         for r in runs])
        gathered = [None] * world
        dist.all_gather_object(gathered, mine)
        ms = bench.reduce_max([10.0 + rank, 3.0 - rank], dist, torch.device("cpu"))
        cnt = bench.reduce_sum([1.0 + rank, 5.0], dist, torch.device("cpu"))
        dist.barrier()
        out[rank] = (gathered, ms, cnt)
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 3])
def test_gloo_ranks_tile_the_layer_once(world):
    port = _free_port()
    with mp.get_context("spawn").Manager() as m:
        out = m.dict()
        mp.spawn(_rank_main, args=(world, port, out), nprocs=world, join=True)
        res = dict(out)
    for r in range(world):
        assert res[r][0] == res[0][0]  # every rank computes the same partition
        assert res[r][1] == pytest.approx([10.0 + world - 1, 3.0])   # max over ranks
        assert res[r][2] == pytest.approx([sum(1.0 + x for x in range(world)), 5.0 * world])  # sums
    gathered = res[0][0]
    for si, (b, hq, hkv, n, lens) in enumerate(SHAPES):
        g = hq // hkv
        nb = -(-n // 128)
        words = (nb + 31) // 32
        covered = np.zeros((b, hkv), dtype=int)
        for rank_runs in gathered:
            for (bi, kv0, kv1, off, sl) in rank_runs[si]:
                covered[bi, kv0:kv1] += 1
                assert off["hq"] == (kv1 - kv0) * g and off["hkv"] == kv1 - kv0
                assert off["q"] == (bi * hq + kv0 * g) * n * 128       # first Q row of the run
                assert off["kv"] == (bi * hkv + kv0) * n * 128         # first K / V row
                assert off["mask"] == (bi * hq + kv0 * g) * nb * words
                assert sl == (None if lens is None else [lens[bi]])
        assert np.all(covered == 1), f"shape {si}: units covered {covered.tolist()}"
        # contiguous and balanced: rank r holds floor(U (r+1)/world) - floor(U r/world) units
        units = b * hkv
        for r, rank_runs in enumerate(gathered):
            assert sum(kv1 - kv0 for (_, kv0, kv1, _, _) in rank_runs[si]) == \
                units * (r + 1) // world - units * r // world


def test_single_rank_is_the_whole_layer_and_views_are_the_heads():
    import bench
    assert bench.reduce_max([1.5, 2.5], None, torch.device("cpu")) == [1.5, 2.5]
    assert bench.reduce_sum([1.5, 2.5], None, torch.device("cpu")) == [1.5, 2.5]
    assert shard.shard_runs(1, 8, 1, 0) == [shard.Run(0, 0, 8)]
    assert shard.shard_runs(1, 8, 16, 15) == [shard.Run(0, 7, 8)]
    assert shard.shard_runs(1, 2, 4, 0) == []  # more ranks than units: idle ranks
    q = torch.arange(2 * 8 * 3 * 2).reshape(2, 8, 3, 2)
    k = torch.arange(2 * 2 * 3 * 2).reshape(2, 2, 3, 2)
    run = shard.Run(1, 1, 2)
    qs, ks, vs, ms, os_ = shard.run_views(run, 4, q, k, k, None, q)
    assert torch.equal(qs, q[1:2, 4:8]) and torch.equal(ks, k[1:2, 1:2]) and ms is None
    assert qs.is_contiguous() and ks.is_contiguous()
    assert qs.flatten()[0].item() == shard.run_offsets(run, 8, 2, 3, head_dim=2)["q"]
    with pytest.raises(ValueError):
        shard.shard_runs(1, 8, 2, 2)
