"""mxattn_forward_noalloc against mxattn_forward.

Some callers of this library cannot allocate device memory themselves: a host
framework that owns every device byte through its own pool and forbids raw
cudaMalloc, or a latency-critical loop that must not pay for cudaMalloc's
implicit device synchronization.  mxattn_forward_noalloc serves them by running
the same kernels on a fixed 16 MiB scratch array that lives inside the library.
Two calls in a row (different inputs, one shared scratch) must each match
mxattn_forward with a caller-owned workspace within the parity tolerance, and a
shape whose workspace does not fit must be refused before anything runs.

This file is collected last on purpose, so a run that stops at the first
failure has already run every other test.
"""
import ctypes

import numpy as np
import pytest
import torch

from mxfp4_microscaled_quantization_b200 import mxattn as mx
from mxfp4_microscaled_quantization_b200 import workloads as wl

pytestmark = pytest.mark.gpu

REL_FROB = 1e-3
MAX_ABS = 2e-2


def _dev(bits):
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).cuda().view(torch.bfloat16)


def _noalloc_via_c_abi(q, k, v, kv_tile, pnq, rule):
    B, H, N, d = q.shape
    out = torch.empty((B, H, N, d), dtype=torch.float32, device="cuda")
    ptr = lambda t: ctypes.c_void_p(t.data_ptr())  # noqa: E731
    status = mx.lib().mxattn_forward_noalloc(ptr(q), ptr(k), ptr(v), B, H, N, d, kv_tile, 1 if pnq else 0,
                                             mx.RULES[rule], ctypes.c_float(0.0), ptr(out),
                                             ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert status == 0, mx.status_string(status)
    return out


@pytest.mark.parametrize("shape,kv_tile,pnq,rule", [((1, 4, 1000, 128), 128, True, "uos"),
                                                    ((2, 3, 333, 64), 64, False, "ocp")])
def test_noalloc_matches_forward_on_two_calls_in_a_row(shape, kv_tile, pnq, rule):
    B, H, N, d = shape
    assert mx.mxattn_workspace_size(B, H, N, d) <= mx.NOALLOC_MAX_WORKSPACE
    for seed in (21, 22):  # the second call reuses the scratch the first one left behind
        Q, K, V = wl.gaussian_qkv(B, H, N, d, seed=seed)
        q, k, v = _dev(Q), _dev(K), _dev(V)
        got = _noalloc_via_c_abi(q, k, v, kv_tile, pnq, rule)
        ws = mx.new_workspace(B, H, N, d)
        ref = mx.mxattn_forward(q, k, v, kv_tile, pnq, rule, workspace=ws)
        assert mx.mxattn_workspace_status(ws) == 0
        g = got.cpu().numpy().astype(np.float64)
        r = ref.cpu().numpy().astype(np.float64)
        assert np.all(np.isfinite(g))
        rel = np.linalg.norm(g - r) / np.linalg.norm(r)
        assert rel <= REL_FROB and np.max(np.abs(g - r)) <= MAX_ABS, f"seed {seed}: rel-Frobenius {rel:.3e}"


def test_noalloc_refuses_shapes_larger_than_its_scratch():
    B, H, N, d = 1, 40, 32760, 128
    assert mx.mxattn_workspace_size(B, H, N, d) > mx.NOALLOC_MAX_WORKSPACE
    fake = ctypes.c_void_p(1 << 20)
    status = mx.lib().mxattn_forward_noalloc(fake, fake, fake, B, H, N, d, 128, 1, 1, ctypes.c_float(0.0), fake,
                                             None)
    assert status == 2  # MXATTN_ERR_UNSUPPORTED, nothing launched
