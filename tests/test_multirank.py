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


def _ulysses_worker(rank, world, port, out_dir):
    import torch

    import oracle
    from mxfp4_microscaled_quantization_b200 import ulysses

    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        Q, K, V = wl.gaussian_qkv(1, 4, 192, 64, seed=3)
        n = 192 // world
        local = lambda a: torch.from_numpy(np.ascontiguousarray(a[:, :, rank * n:(rank + 1) * n]).view(np.int16))  # noqa: E731

        def oracle_attend(q, k, v, kv_tile):  # the CPU oracle stands in for the GPU kernel
            bits = lambda t: np.ascontiguousarray(t.numpy()).view(np.uint16)  # noqa: E731
            return torch.from_numpy(oracle.attention(bits(q), bits(k), bits(v), kv_tile, rule="uos", pnq=True))

        o = ulysses.sequence_parallel_attention(local(Q), local(K), local(V), attend=oracle_attend, kv_tile=64)
        np.save(os.path.join(out_dir, f"o{rank}.npy"), o.numpy())
        dist.barrier()
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 4])
def test_gloo_sequence_parallel_attention_equals_single_rank(world, tmp_path):
    """Ulysses: tokens split over the ranks, all-to-all to heads, attention (the
    oracle here, on CPU), all-to-all back; the ranks' token blocks put together
    equal the single-rank result, bit for bit (same heads, same key-tile order)."""
    import oracle

    mp.start_processes(_ulysses_worker, args=(world, _free_port(), str(tmp_path)), nprocs=world,
                       start_method="spawn")
    Q, K, V = wl.gaussian_qkv(1, 4, 192, 64, seed=3)
    ref = oracle.attention(Q, K, V, 64, rule="uos", pnq=True)
    got = np.concatenate([np.load(tmp_path / f"o{r}.npy") for r in range(world)], axis=2)
    np.testing.assert_array_equal(got, ref)


def test_sequence_layout_transforms_are_identity_on_one_rank():
    import torch

    from mxfp4_microscaled_quantization_b200 import ulysses

    x = torch.arange(2 * 4 * 6 * 8, dtype=torch.float32).reshape(2, 4, 6, 8)
    assert ulysses.seq_to_head(x) is x and ulysses.head_to_seq(x) is x


def test_bench_gpus_flag_starts_its_own_ranks():
    """`bench.py --gpus 2` outside torchrun starts two ranks on this node itself
    (here the reference arm, which runs on the host: rank 0 times the oracle and
    prints the one JSON line, rank 1 exits without work)."""
    import json
    import subprocess
    import sys

    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    env = {k: v for k, v in os.environ.items() if k not in ("RANK", "WORLD_SIZE", "LOCAL_RANK", "MASTER_ADDR",
                                                            "MASTER_PORT")}
    res = subprocess.run([sys.executable, os.path.join(root, "bench.py"), "--gpus", "2", "--impl", "reference",
                          "--steps", "1", "--warmup", "3", "--ref-step-budget", "0.2"], capture_output=True,
                         text=True, env=env, cwd=root, timeout=600)
    assert res.returncode == 0, res.stderr[-2000:]
    lines = [ln for ln in res.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1, res.stdout
    line = json.loads(lines[0])
    assert line["impl"] == "reference" and line["n_gpus"] == 2 and line["steps"] == 1
    assert line["config"] == bench.config_dict(bench.WORKLOAD, 2, "replicas")
