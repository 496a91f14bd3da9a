"""Seeded synthetic inputs for MXFP4 attention (shared by the CUDA path's tests,
the oracle's tests and the benchmark).

This module holds only random-number generation and array shaping: no part of
the quantization or attention arithmetic lives here, so both the CUDA path and
the CPU oracle can take their inputs from it without sharing method code.

Every tensor is drawn on the host with numpy's PCG64 (`default_rng`), in
float32, then rounded to bfloat16 with round-to-nearest-even.  Q, K and V use
independent sub-streams `seed`, `seed + 1`, `seed + 2`.

The workloads stand in for the self-attention of the video diffusion
transformers (Wan2.2, HunyuanVideo) that the MXAttention abstract evaluates on;
those models, their weights and the VBench prompts are not used.
"""
from __future__ import annotations

import dataclasses
import math

import numpy as np

__all__ = [
    "Workload",
    "WORKLOADS",
    "f32_to_bf16_bits",
    "bf16_bits_to_f32",
    "gaussian_qkv",
    "outlier_qkv",
    "video_dit_qkv",
    "student_t_matrix",
    "student_t_qkv",
    "make_qkv",
]


@dataclasses.dataclass(frozen=True)
class Workload:
    """One attention problem: shapes, tile and the input recipe's name."""

    name: str
    B: int
    H: int
    N: int
    d: int
    kv_tile: int
    recipe: str  # "gaussian" | "outlier" | "video"
    frames: int = 0
    rows: int = 0
    cols: int = 0

    @property
    def flops(self) -> float:
        """Algorithmic work 4*B*H*N^2*d (QK^T and PV, one multiply-add = 2 flops)."""
        return 4.0 * self.B * self.H * float(self.N) ** 2 * self.d


# The four attention workloads.  The fifth workload (the standalone quantize
# sweep) is `student_t_matrix`.
WORKLOADS = {
    "tiny": Workload("tiny", 1, 1, 256, 64, 64, "gaussian"),
    "outlier": Workload("outlier", 1, 8, 4096, 128, 128, "outlier"),
    "video_dit": Workload("video_dit", 1, 40, 32760, 128, 128, "video", 21, 30, 52),
    "long_video_dit": Workload("long_video_dit", 1, 24, 75600, 128, 128, "video", 21, 45, 80),
}


def f32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round float32 values to bfloat16 (nearest, ties to even); returns uint16 bit patterns."""
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32).astype(np.uint64)
    rounded = (u + 0x7FFF + ((u >> 16) & 1)) >> 16
    return rounded.astype(np.uint16)


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    """Widen bfloat16 bit patterns (uint16) to float32 exactly."""
    return (np.asarray(b, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32)


def gaussian_qkv(B, H, N, d, seed=0):
    """Q, K, V drawn i.i.d. N(0, 1); returns three uint16 (bf16 bits) arrays [B, H, N, d]."""
    out = []
    for t in range(3):
        rng = np.random.default_rng(seed + t)
        out.append(f32_to_bf16_bits(rng.standard_normal((B, H, N, d), dtype=np.float32)))
    return tuple(out)


def outlier_qkv(B, H, N, d, seed=0, frac=0.02, factor=20.0):
    """Outlier-channel inputs: Q, K ~ N(0, 1) with round(frac*d) channels per head
    (the same channels for Q and K, chosen per head from `seed`) multiplied by
    `factor`; V ~ N(0, 1)."""
    n_out = int(round(frac * d))
    pick = np.random.default_rng(seed)
    chans = np.stack([pick.choice(d, n_out, replace=False) for _ in range(B * H)])
    out = []
    for t in range(3):
        rng = np.random.default_rng(seed + t)
        x = rng.standard_normal((B, H, N, d), dtype=np.float32)
        if t < 2:
            xv = x.reshape(B * H, N, d)
            for bh in range(B * H):
                xv[bh][:, chans[bh]] *= np.float32(factor)
        out.append(f32_to_bf16_bits(x))
    return tuple(out)


def _smooth_lowrank_head(rng, frames, rows, cols, d, rank=16, sigma=2.0, noise=0.3):
    from scipy.ndimage import gaussian_filter1d

    z = rng.standard_normal((frames, rows, cols, rank), dtype=np.float32)
    for ax in range(3):
        z = gaussian_filter1d(z, sigma, axis=ax, mode="reflect", truncate=4.0)
    z = z.reshape(frames * rows * cols, rank)
    z /= z.std(axis=0, keepdims=True)
    a = rng.standard_normal((rank, d), dtype=np.float32) * np.float32(1.0 / math.sqrt(rank))
    x = z @ a
    x += rng.standard_normal(x.shape, dtype=np.float32) * np.float32(noise)
    amp = math.exp(rng.uniform(math.log(0.5), math.log(4.0)))
    x *= np.float32(amp)
    return x


def video_dit_qkv(B, H, frames, rows, cols, d, seed=0):
    """Video-DiT-like inputs: per (tensor, head) a rank-16 latent field over the
    (frame, row, col) token grid, Gaussian-smoothed with sigma 2 along all three
    axes (truncated at 4 sigma, reflecting boundary), each latent channel
    re-standardised to unit std, projected to d channels with A ~ N(0, 1/16),
    plus N(0, 0.3^2) noise, times an amplitude drawn log-uniform in [0.5, 4].
    Token index is f*rows*cols + r*cols + c."""
    N = frames * rows * cols
    out = []
    for t in range(3):
        rng = np.random.default_rng(seed + t)
        arr = np.empty((B, H, N, d), dtype=np.uint16)
        for b in range(B):
            for h in range(H):
                arr[b, h] = f32_to_bf16_bits(_smooth_lowrank_head(rng, frames, rows, cols, d))
        out.append(arr)
    return tuple(out)


def student_t_matrix(n_elems, cols=4096, seed=0, nu=3.0, scale=0.5):
    """Quantize-sweep input: bf16 [n_elems // cols, cols] with values 0.5 * StudentT(nu=3)."""
    assert n_elems % cols == 0
    rng = np.random.default_rng(seed)
    rows = n_elems // cols
    out = np.empty((rows, cols), dtype=np.uint16)
    step = max(1, (1 << 24) // cols)
    for r0 in range(0, rows, step):
        r1 = min(rows, r0 + step)
        x = rng.standard_t(nu, size=(r1 - r0, cols)).astype(np.float32) * np.float32(scale)
        out[r0:r1] = f32_to_bf16_bits(x)
    return out


def student_t_qkv(B, H, N, d, seed=0, nu=3.0):
    """Heavy-tailed inputs: Q, K, V drawn i.i.d. StudentT(nu), nu = 3 by default."""
    out = []
    for t in range(3):
        rng = np.random.default_rng(seed + t)
        out.append(f32_to_bf16_bits(rng.standard_t(nu, size=(B, H, N, d)).astype(np.float32)))
    return tuple(out)


def make_qkv(w: Workload, seed=0):
    """Inputs of workload `w` as three uint16 (bf16 bits) arrays [B, H, N, d]."""
    if w.recipe == "gaussian":
        return gaussian_qkv(w.B, w.H, w.N, w.d, seed)
    if w.recipe == "outlier":
        return outlier_qkv(w.B, w.H, w.N, w.d, seed)
    if w.recipe == "video":
        assert w.frames * w.rows * w.cols == w.N
        return video_dit_qkv(w.B, w.H, w.frames, w.rows, w.cols, w.d, seed)
    raise ValueError(f"unknown recipe {w.recipe!r}")
