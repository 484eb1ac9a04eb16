"""The multi-rank bench path on CPU: two gloo ranks, no GPU.

With N > 1 every rank runs its own clip (weak scaling): the only collectives are
the barrier around the timed region and the max over ranks of the device time.
These tests run those helpers with world_size 2 and check the per-rank inputs.
"""
import os
import socket
import sys

import numpy as np
import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out_dir):
    import datetime

    import torch
    import torch.distributed as dist

    import bench
    from structured_attention_video_b200 import synth

    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        bench.rank_barrier(world)
        # every rank reports a different time; all of them must see the largest
        slowest = bench.max_over_ranks(1.0 + rank, world, torch.device("cpu"))
        # the reference arm does its work on rank 0 only and returns at once elsewhere
        wl = synth.WORKLOADS["tiny"]
        if rank != 0:
            bench.run_reference(None, wl, world, rank)
        # each rank's clip: the same shapes, its own seed
        pos = synth.positional_code(wl.f, wl.h, wl.w, wl.d)
        x = synth.make_head(wl, 0, 0, rank, pos)
        np.savez(os.path.join(out_dir, "rank%d.npz" % rank), slowest=slowest, q=x["q"])
        bench.rank_barrier(world)
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_max_time_and_distinct_clips(tmp_path):
    world = 2
    mp.start_processes(_rank_main, args=(world, _free_port(), str(tmp_path)), nprocs=world,
                       join=True, start_method="spawn")
    r0 = np.load(tmp_path / "rank0.npz")
    r1 = np.load(tmp_path / "rank1.npz")
    assert float(r0["slowest"]) == 2.0 and float(r1["slowest"]) == 2.0
    assert r0["q"].shape == r1["q"].shape
    assert not np.array_equal(r0["q"], r1["q"])


def test_job_throughput_counts_every_rank():
    import bench
    one = bench.job_throughput(1, 1e12, 1.0)
    assert one == pytest.approx(1000.0)
    assert bench.job_throughput(4, 1e12, 1.0) == pytest.approx(4 * one)
