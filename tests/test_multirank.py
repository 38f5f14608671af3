"""The N > 1 host logic of bench.py on CPU: two `gloo` ranks (world size 2).

Each rank runs its own replica on its own data (weak scaling, no data-path
collective); the only collective is the max of the ranks' times, and the
job's throughput is the units all ranks processed over that max.  The
reference arm runs on rank 0 alone.
"""

import os
import socket
import sys

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, results):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    import datetime

    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        import bench
        from rotation_w4a4_quantization_b200 import synthetic as syn

        # per-rank times: the max goes to every rank
        mx = bench.max_over_ranks([1.0 + rank, 10.0 - rank, 3.0], dist)
        # each rank's inputs come from its own seeds (the bench's seed offsets)
        x = syn.activations("tiny_int4", rows=4, seed_offset=rank * bench.RING_MAX)
        gathered = [torch.empty_like(x.float()) for _ in range(world)]
        dist.all_gather(gathered, x.float())
        distinct = not torch.equal(gathered[0], gathered[1])
        results[rank] = (mx.tolist(), distinct)
    finally:
        dist.destroy_process_group()


def test_two_rank_max_and_distinct_inputs():
    world = 2
    port = _free_port()
    ctx = mp.get_context("spawn")
    manager = ctx.Manager()
    results = manager.dict()
    mp.start_processes(_rank_main, args=(world, port, results), nprocs=world, join=True, start_method="spawn")
    assert sorted(results.keys()) == [0, 1]
    for r in range(world):
        mx, distinct = results[r]
        assert mx == [2.0, 10.0, 3.0]
        assert distinct


def test_job_rate_counts_every_rank():
    import bench
    # 1 GB per rank in 2 ms on each of 4 ranks: 2 TB/s for the job
    assert bench.job_rate(1e9, 4, 2.0) == pytest.approx(2e12)
    assert bench.max_over_ranks([3.0, 4.0]).tolist() == [3.0, 4.0]


def test_reference_arm_runs_on_rank0_only(capsys):
    import argparse

    import bench
    args = argparse.Namespace(workload="q_proj_int4", steps=1, warmup=0, y_dtype="bf16", gpus=2)
    bench.run_reference(args, world=2, rank=1)
    assert capsys.readouterr().out == ""
