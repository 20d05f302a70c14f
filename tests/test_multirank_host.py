"""The benchmark's multi-rank host logic on CPU with gloo, world size 2: every rank times
its own replica; the job time is the max over ranks and the value counts every rank's tokens."""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, results):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    import bench
    from datetime import timedelta
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=timedelta(seconds=60))
    try:
        assert bench.dist_env() == (world, rank, rank)
        dev = torch.device("cpu")
        bench.barrier(dev)
        my_ms = 100.0 + 50.0 * rank           # rank 1 is the slow one
        mx = bench.reduce_max(my_ms, dev)
        agg = bench.aggregate(tokens_per_rank=4096, world=world, max_ms_total=mx, steps=10)
        results[rank] = (mx, agg["value"], agg["ms_per_step"])
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_and_aggregate_gloo():
    world = 2
    port = _free_port()
    mgr = mp.get_context("spawn").Manager()
    results = mgr.dict()
    mp.start_processes(_worker, args=(world, port, results), nprocs=world, join=True,
                       start_method="spawn")
    assert len(results) == world
    for rank in range(world):
        mx, value, ms = results[rank]
        assert mx == 150.0
        assert ms == 15.0
        assert value == pytest.approx(4096 * 2 * 10 / 0.150)


def test_single_rank_defaults(monkeypatch):
    import bench
    for k in ("WORLD_SIZE", "RANK", "LOCAL_RANK"):
        monkeypatch.delenv(k, raising=False)
    assert bench.dist_env() == (1, 0, 0)
    assert bench.reduce_max(3.5, torch.device("cpu")) == 3.5
    agg = bench.aggregate(64, 1, 20.0, 4)
    assert agg["ms_per_step"] == 5.0 and agg["value"] == pytest.approx(64 * 4 / 0.020)
