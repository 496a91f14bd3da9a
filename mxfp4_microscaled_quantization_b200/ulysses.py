"""Sequence-parallel attention across GPUs (the all-to-all scheme known as
Ulysses): the host-side exchange around the fused kernel.

A video diffusion transformer run with sequence parallelism holds, on each of
P ranks, Q, K and V for its own N/P tokens and all H heads.  Attention needs
all N tokens of a head, so one all-to-all regroups the tensors by head (rank r
gets heads [r H/P, (r+1) H/P) over every token), each rank runs the attention
on its heads, and a second all-to-all returns the output to the token layout.
Heads are independent and every rank sees every key in ascending order, so the
result equals the single-GPU forward, key-tile order (and thus PNQ) included.

The exchanges use torch.distributed all-to-all (NCCL between GPUs); the
attention is any callable on [B, h, N, d] tensors, by default the library's
mxattn_forward.
"""
from __future__ import annotations

import torch
import torch.distributed as dist


def _world(group):
    return dist.get_world_size(group) if dist.is_initialized() else 1


def _exchange(send: torch.Tensor, group) -> torch.Tensor:
    """all_to_all of the P equal blocks along dim 0 of a contiguous tensor, moved
    as raw bytes (so any element type goes through every backend)."""
    recv = torch.empty_like(send)
    dist.all_to_all_single(recv.view(torch.uint8), send.view(torch.uint8), group=group)
    return recv


def seq_to_head(x: torch.Tensor, group=None) -> torch.Tensor:
    """[B, H, n, d] (this rank's n = N/P tokens, all heads) -> [B, H/P, N, d]
    (this rank's heads, all tokens in global order)."""
    P = _world(group)
    if P == 1:
        return x
    B, H, n, d = x.shape
    if H % P:
        raise ValueError(f"{H} heads do not split over {P} ranks")
    h = H // P
    send = x.reshape(B, P, h, n, d).permute(1, 0, 2, 3, 4).contiguous()  # [P, B, h, n, d]: block j goes to rank j
    recv = _exchange(send, group)                                          # [P, B, h, n, d]: block i came from rank i
    return recv.permute(1, 2, 0, 3, 4).reshape(B, h, P * n, d)


def head_to_seq(o: torch.Tensor, group=None) -> torch.Tensor:
    """Inverse of seq_to_head: [B, H/P, N, d] -> [B, H, N/P, d]."""
    P = _world(group)
    if P == 1:
        return o
    B, h, N, d = o.shape
    if N % P:
        raise ValueError(f"{N} tokens do not split over {P} ranks")
    n = N // P
    send = o.reshape(B, h, P, n, d).permute(2, 0, 1, 3, 4).contiguous()  # [P, B, h, n, d]: token block j to rank j
    recv = _exchange(send, group)                                          # [P, B, h, n, d]: head group i from rank i
    return recv.permute(1, 0, 2, 3, 4).reshape(B, P * h, n, d)


def sequence_parallel_attention(q, k, v, attend=None, group=None, **kwargs):
    """Attention over a sequence split across the ranks of `group`.

    q, k, v: [B, H, N/P, d] -- this rank's contiguous block of tokens (rank r
    holds tokens [r N/P, (r+1) N/P)); H and N must divide by P.  Returns this
    rank's block of O, [B, H, N/P, d].  `attend(q, k, v, **kwargs)` runs on
    [B, H/P, N, d]; by default mxattn_forward (kv_tile, pnq, rule, ... pass
    through kwargs)."""
    if attend is None:
        from . import mxattn

        attend = mxattn.mxattn_forward
    qh, kh, vh = (seq_to_head(t, group) for t in (q, k, v))
    return head_to_seq(attend(qh, kh, vh, **kwargs), group)
