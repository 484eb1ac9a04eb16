"""Splitting one clip across ranks by (batch, head, tile) units.

Every unit is independent from the aggregated query to its output rows, so the
ranks of one job can each compute a contiguous range of units of the same clip,
with no data-path collective.  These tests check, on the CPU with two gloo
ranks, that the ranks' ranges cover every unit exactly once and that the output
rows they write are disjoint and cover each head's N rows; the GPU test in
test_parity_gpu.py checks that calls over a partition reproduce the full call
bit for bit."""
import os
import socket
import sys

import numpy as np
import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402
from structured_attention_video_b200 import synth  # noqa: E402


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out_dir, name):
    import datetime

    import torch.distributed as dist

    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        wl = synth.WORKLOADS[name]
        total = wl.B * wl.H * wl.tiles
        mine = bench.unit_partition(total, world, rank)
        ranges = [None] * world
        dist.all_gather_object(ranges, mine)
        if rank == 0:
            np.save(os.path.join(out_dir, "ranges.npy"), np.array(ranges))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("name", ["720p", "14b", "480p_chunk"])
def test_two_gloo_ranks_partition_the_units(tmp_path, name):
    world = 2
    mp.start_processes(_rank_main, args=(world, _free_port(), str(tmp_path), name),
                       nprocs=world, join=True, start_method="spawn")
    wl = synth.WORKLOADS[name]
    ranges = np.load(tmp_path / "ranges.npy")
    covered = np.zeros(wl.B * wl.H * wl.tiles, np.int64)
    for b, e in ranges:
        covered[b:e] += 1
    assert (covered == 1).all()
    # the output rows of the two ranks are disjoint and cover every row of every head
    owner = np.full((wl.B * wl.H, wl.N), -1, np.int64)
    for r, (b, e) in enumerate(ranges):
        for unit in range(b, e):
            bh, rows = bench.unit_rows(wl, unit)
            assert (owner[bh, rows] == -1).all()
            owner[bh, rows] = r
    assert (owner >= 0).all()


@pytest.mark.parametrize("world", [1, 3, 7, 8, 48, 50])
def test_partition_is_contiguous_and_balanced(world):
    total = 48
    ranges = [bench.unit_partition(total, world, r) for r in range(world)]
    assert ranges[0][0] == 0 and ranges[-1][1] == total
    for (b0, e0), (b1, _) in zip(ranges, ranges[1:]):
        assert e0 == b1
    sizes = [e - b for b, e in ranges]
    assert max(sizes) - min(sizes) <= 1


def test_unit_rows_follow_the_tile_partition():
    wl = synth.WORKLOADS["720p"]
    bh, rows = bench.unit_rows(wl, 3 * wl.tiles + 3)
    assert bh == 3
    assert rows.size == (wl.b1 - (3 * wl.b1) // 4) * wl.b2        # the last tile: 237 rows
    assert rows.min() == ((3 * wl.b1) // 4) * wl.b2 and rows.max() == wl.N - 1
