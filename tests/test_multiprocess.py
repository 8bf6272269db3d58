"""The N > 1 host logic of the benchmark, on CPU: world_size-2 gloo process groups.

The head shards as independent replicas (one per GPU, no collective on the data path); what crosses
ranks is the timing and the work count: the job's time is the slowest rank's (max over ranks) and its
work the sum over ranks.  Each rank draws its own query pool, and the reference arm runs on rank 0
only."""

import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        import bench
        from clustered_retrieval_classification_b200 import synth
        t_ms = [3.5, 7.25][rank]
        calls = [100, 300][rank]
        out[rank * 4 + 0] = bench.max_over_ranks(t_ms, True)
        out[rank * 4 + 1] = bench.sum_over_ranks(calls, True)
        cfg = synth.scaled(synth.CONFIGS["llama"], v=4096, c=256, d=64, p=8, name="mp")
        q = torch.from_numpy(bench.rank_queries(cfg, 4, rank).astype(np.float64).ravel().copy())
        gathered = [torch.zeros_like(q) for _ in range(world)]
        dist.all_gather(gathered, q)
        out[rank * 4 + 2] = float(torch.equal(gathered[0], gathered[1]))
        out[rank * 4 + 3] = float(torch.equal(gathered[rank], q))
    finally:
        dist.destroy_process_group()


def test_two_rank_timing_and_work_reductions():
    world = 2
    out = torch.zeros(world * 4, dtype=torch.float64).share_memory_()
    mp.start_processes(_worker, args=(world, _free_port(), out), nprocs=world, join=True,
                       start_method="spawn")
    for r in range(world):
        assert out[r * 4 + 0] == 7.25          # max over ranks: the slowest rank's time
        assert out[r * 4 + 1] == 400           # sum over ranks: all the work done
        assert out[r * 4 + 2] == 0.0           # the ranks' query pools differ
        assert out[r * 4 + 3] == 1.0


def test_reference_arm_runs_on_rank_zero_only(monkeypatch):
    import bench
    monkeypatch.setenv("RANK", "1")

    class Args:
        batch, steps, warmup, gpus = 1, 1, 1, 2
    assert bench.run_reference(Args()) is None  # returns at once: no work, no output
