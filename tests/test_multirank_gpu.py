"""The sharded multi-GPU paths with the CUDA kernel inside them.

Two processes, each a gloo rank, share cuda:0: the exchanges (the all-to-alls
of the sequence-parallel scheme) move host tensors over gloo, and the
attention on each rank is mxattn_forward on the GPU.  The kernels of the two
ranks are independent launches that never wait on each other.  Checked: the
ranks' pieces of O put together equal the single-process forward bit for bit
(heads are independent and every rank walks every key tile in order), and
stay within the target's tolerance of the CPU oracle (rel-Frobenius <= 1e-3,
max-abs <= 2e-2).
"""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import bench
import oracle
from mxfp4_microscaled_quantization_b200 import workloads as wl

pytestmark = pytest.mark.gpu

B, H, N, d, T = 1, 4, 1000, 128, 128


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _inputs():
    return wl.gaussian_qkv(B, H, N, d, seed=11)


def _to_torch(a):
    return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16)


def _worker(rank, world, port, out_dir, mode):
    from mxfp4_microscaled_quantization_b200 import mxattn as mx
    from mxfp4_microscaled_quantization_b200 import ulysses

    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        torch.cuda.set_device(0)
        Q, K, V = _inputs()
        if mode == "sequence":
            n = N // world
            local = [_to_torch(a[:, :, rank * n:(rank + 1) * n]) for a in (Q, K, V)]

            def gpu_attend(q, k, v, **kw):  # this rank's heads on the GPU; the exchange stays on the host
                return mx.mxattn_forward(q.cuda(), k.cuda(), v.cuda(), **kw).cpu()

            o = ulysses.sequence_parallel_attention(*local, attend=gpu_attend, kv_tile=T, pnq=True, rule="uos")
        else:
            lo, hi = bench.head_range(H, rank, world)
            q, k, v = (_to_torch(a[:, lo:hi]).cuda() for a in (Q, K, V))
            o = mx.mxattn_forward(q, k, v, T, True, "uos").cpu()
        torch.cuda.synchronize()
        np.save(os.path.join(out_dir, f"{mode}_o{rank}.npy"), o.numpy())
        dist.barrier()
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("mode,axis", [("sequence", 2), ("heads", 1)])
def test_two_ranks_on_one_gpu_match_single_process(mode, axis, tmp_path):
    from mxfp4_microscaled_quantization_b200 import mxattn as mx

    world = 2
    mp.start_processes(_worker, args=(world, _free_port(), str(tmp_path), mode), nprocs=world, start_method="spawn")
    got = np.concatenate([np.load(tmp_path / f"{mode}_o{r}.npy") for r in range(world)], axis=axis)
    Q, K, V = _inputs()
    single = mx.mxattn_forward(*(_to_torch(a).cuda() for a in (Q, K, V)), T, True, "uos").cpu().numpy()
    np.testing.assert_array_equal(got, single)
    R = oracle.attention(Q, K, V, T, rule="uos", pnq=True)
    g = got.astype(np.float64)
    rel = np.linalg.norm(g - R) / np.linalg.norm(R)
    mabs = float(np.max(np.abs(g - R)))
    assert rel <= 1e-3 and mabs <= 2e-2, f"{mode}: rel-Frobenius {rel:.3e}, max-abs {mabs:.3e}"
