"""mxattn_forward_noalloc against mxattn_forward.

Some callers of this library cannot allocate device memory themselves: a host
framework that owns every device byte through its own pool and forbids raw
cudaMalloc, or a latency-critical loop that must not pay for cudaMalloc's
implicit device synchronization.  mxattn_forward_noalloc serves them by running
the same kernels on a fixed 16 MiB scratch array that lives inside the library.

The scratch is shared by every call and keeps the previous call's contents, so
the tests run calls back to back -- two in a row on one shape, and a sequence
that changes N, d, kv_tile, the rule and PNQ between calls -- and require each
result to be bit-identical to mxattn_forward with a caller-owned workspace
(the same kernels on the same inputs).  Argument errors must come back with the
same codes as mxattn_forward, and a shape whose workspace does not fit must be
refused before anything runs.

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

OK, INVALID, UNSUPPORTED = 0, 1, 2


def _dev(bits):
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).cuda().view(torch.bfloat16)


def _ptr(t):
    return ctypes.c_void_p(t.data_ptr())


def _stream():
    return ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)


def _noalloc_via_c_abi(q, k, v, kv_tile, pnq, rule):
    B, H, N, d = q.shape
    out = torch.full((B, H, N, d), float("nan"), dtype=torch.float32, device="cuda")
    status = mx.lib().mxattn_forward_noalloc(_ptr(q), _ptr(k), _ptr(v), B, H, N, d, kv_tile, 1 if pnq else 0,
                                             mx.RULES[rule], ctypes.c_float(0.0), _ptr(out), _stream())
    assert status == OK, mx.status_string(status)
    return out


def _check_against_forward(shape, kv_tile, pnq, rule, seed):
    B, H, N, d = shape
    assert mx.mxattn_workspace_size(B, H, N, d) <= mx.NOALLOC_MAX_WORKSPACE
    Q, K, V = wl.gaussian_qkv(B, H, N, d, seed=seed)
    q, k, v = _dev(Q), _dev(K), _dev(V)
    got = _noalloc_via_c_abi(q, k, v, kv_tile, pnq, rule)
    ws = mx.new_workspace(B, H, N, d)
    ref = mx.mxattn_forward(q, k, v, kv_tile, pnq, rule, workspace=ws)
    assert mx.mxattn_workspace_status(ws) == 0
    torch.cuda.synchronize()
    assert torch.isfinite(got).all()
    assert torch.equal(got, ref), (f"shape {shape} kv_tile {kv_tile} pnq {pnq} {rule}: max |diff| "
                                   f"{(got - ref).abs().max().item():.3e}")


@pytest.mark.parametrize("shape,kv_tile,pnq,rule", [((1, 4, 1000, 128), 128, True, "uos"),
                                                    ((2, 3, 333, 64), 64, False, "ocp")])
def test_noalloc_matches_forward_on_two_calls_in_a_row(shape, kv_tile, pnq, rule):
    for seed in (21, 22):  # the second call reuses the scratch the first one left behind
        _check_against_forward(shape, kv_tile, pnq, rule, seed)


def test_noalloc_matches_forward_when_the_shape_changes_between_calls():
    """Large then small N, d = 128 then 64 and back, both tiles, rules and PNQ
    settings: a call must not read anything a larger previous call left behind."""
    seq = [((1, 8, 8000, 128), 128, True, "uos"),
           ((1, 1, 100, 64), 64, True, "uos"),
           ((1, 2, 4097, 128), 64, False, "ocp"),
           ((2, 1, 33, 128), 128, True, "ocp"),
           ((1, 3, 1500, 64), 128, False, "uos"),
           ((1, 1, 1, 128), 128, True, "uos")]
    for i, (shape, kv_tile, pnq, rule) in enumerate(seq):
        _check_against_forward(shape, kv_tile, pnq, rule, seed=40 + i)


def test_noalloc_refuses_shapes_larger_than_its_scratch():
    B, H, N, d = 1, 40, 32760, 128
    assert mx.mxattn_workspace_size(B, H, N, d) > mx.NOALLOC_MAX_WORKSPACE
    fake = ctypes.c_void_p(1 << 20)
    status = mx.lib().mxattn_forward_noalloc(fake, fake, fake, B, H, N, d, 128, 1, 1, ctypes.c_float(0.0), fake,
                                             None)
    assert status == UNSUPPORTED  # nothing launched


@pytest.mark.parametrize("B,H,N,d,kv_tile,pnq,rule,want", [
    (1, 1, (1 << 24) + 1, 128, 128, 1, 1, UNSUPPORTED),  # N beyond the limit
    (1, 1, 256, 96, 128, 1, 1, UNSUPPORTED),             # d
    (1, 1, 256, 128, 32, 1, 1, UNSUPPORTED),             # kv_tile
    (1, 1, 256, 128, 128, 2, 1, INVALID),                # pnq
    (1, 1, 256, 128, 128, 1, 7, INVALID),                # rule
    (0, 1, 256, 128, 128, 1, 1, INVALID),                # B
    (1, 1, 0, 128, 128, 1, 1, INVALID),                  # N
])
def test_noalloc_argument_errors_match_forward(B, H, N, d, kv_tile, pnq, rule, want):
    """Nothing is launched for these (every check precedes any launch), so fake pointers are safe."""
    fake = ctypes.c_void_p(1 << 20)
    got = mx.lib().mxattn_forward_noalloc(fake, fake, fake, B, H, N, d, kv_tile, pnq, rule, ctypes.c_float(0.0),
                                          fake, None)
    ref = mx.lib().mxattn_forward(fake, fake, fake, B, H, N, d, kv_tile, pnq, rule, ctypes.c_float(0.0), fake,
                                  fake, ctypes.c_size_t(1 << 40), None)
    assert got == want and ref == want, (got, ref, want)
