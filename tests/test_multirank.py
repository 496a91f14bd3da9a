"""The benchmark's N > 1 host path on CPU: two gloo ranks, each with its own
batch, timings reduced to the slowest rank (no GPU, no data-path collective)."""
import os
import socket

import numpy as np
import pytest
import torch.distributed as dist
import torch.multiprocessing as mp

import bench
from mxfp4_microscaled_quantization_b200 import workloads as wl


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out_dir):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        w = wl.Workload("t", 1, 2, 96, 64, 64, "gaussian")
        Q, _, _ = wl.make_qkv(w, seed=bench.rank_seed(rank))
        my_times = [10.0 + rank, 3.0 - rank]
        red = bench.max_over_ranks(my_times, dist, "cpu")
        np.save(os.path.join(out_dir, f"q{rank}.npy"), Q)
        np.save(os.path.join(out_dir, f"red{rank}.npy"), np.array(red))
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_weak_scaling(tmp_path):
    world = 2
    mp.start_processes(_worker, args=(world, _free_port(), str(tmp_path)), nprocs=world, start_method="spawn")
    q0, q1 = np.load(tmp_path / "q0.npy"), np.load(tmp_path / "q1.npy")
    assert q0.shape == q1.shape and not np.array_equal(q0, q1)  # each rank its own batch
    for r in range(world):
        np.testing.assert_array_equal(np.load(tmp_path / f"red{r}.npy"), [11.0, 3.0])  # slowest rank per entry


def test_max_over_ranks_without_process_group():
    assert bench.max_over_ranks([1.5, 2.0]) == [1.5, 2.0]


def _shard_worker(rank, world, port, out_dir):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        w = wl.Workload("t", 1, 5, 64, 64, 64, "gaussian")
        lo, hi = bench.head_range(w.H, rank, world)
        Q, K, V = (a[:, lo:hi] for a in wl.make_qkv(w, seed=0))
        np.save(os.path.join(out_dir, f"shard_q{rank}.npy"), Q)
        red = bench.max_over_ranks([float(hi - lo)], dist, "cpu")
        np.save(os.path.join(out_dir, f"shard_red{rank}.npy"), np.array(red))
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_head_sharding(tmp_path):
    """--shard heads: the ranks' head slices of one problem put back together are the
    whole problem, and the slowest (largest) shard is what every rank reports."""
    world = 2
    mp.start_processes(_shard_worker, args=(world, _free_port(), str(tmp_path)), nprocs=world, start_method="spawn")
    full, _, _ = wl.make_qkv(wl.Workload("t", 1, 5, 64, 64, 64, "gaussian"), seed=0)
    parts = [np.load(tmp_path / f"shard_q{r}.npy") for r in range(world)]
    np.testing.assert_array_equal(np.concatenate(parts, axis=1), full)
    for r in range(world):
        np.testing.assert_array_equal(np.load(tmp_path / f"shard_red{r}.npy"), [3.0])


@pytest.mark.parametrize("H", [1, 5, 24, 40])
@pytest.mark.parametrize("world", [1, 2, 3, 4, 8])
def test_head_range_partitions_the_heads(H, world):
    ranges = [bench.head_range(H, r, world) for r in range(world)]
    assert ranges[0][0] == 0 and ranges[-1][1] == H
    assert all(a[1] == b[0] for a, b in zip(ranges, ranges[1:]))
    sizes = [hi - lo for lo, hi in ranges]
    assert max(sizes) - min(sizes) <= 1 and min(sizes) >= 0
