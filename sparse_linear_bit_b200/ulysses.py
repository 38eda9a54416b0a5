"""Ulysses context parallelism around the SageSLA forward.

Each of P ranks holds a contiguous range of N / P tokens of every head ([B, H,
N/P, d]).  ``seq_to_heads`` regroups them with one all-to-all into every token of
the rank's H / P heads ([B, H/P, N, d]); the attention runs per head on that;
``heads_to_seq`` returns the output to the token sharding.  The block
permutations around each all-to-all run in ``sla_ulysses_permute`` (CUDA); the
exchange is ``torch.distributed.all_to_all_single`` (NCCL over NVLink on GPUs).
"""
from __future__ import annotations

import ctypes
from typing import Callable, Optional

import torch
import torch.distributed as dist

from . import _ok, _ptr, _stream, lib, sla_forward, workspace

lib.sla_ulysses_permute.argtypes = [ctypes.c_void_p, ctypes.c_void_p] + [ctypes.c_int] * 7 + [ctypes.c_void_p]
lib.sla_ulysses_permute.restype = ctypes.c_int


def cuda_permute(src: torch.Tensor, dst: torch.Tensor, B: int, H: int, P: int, n_local: int, d: int, mode: int,
                 stream=None) -> None:
    _ok(lib.sla_ulysses_permute(_ptr(src), _ptr(dst), B, H, P, n_local, d, src.element_size(), mode,
                                _stream(stream)), "sla_ulysses_permute")


Permute = Callable[[torch.Tensor, torch.Tensor, int, int, int, int, int, int], None]


def seq_to_heads(x: torch.Tensor, group=None, permute: Optional[Permute] = None) -> torch.Tensor:
    """[B, H, N/P, d] (this rank's tokens of every head) -> [B, H/P, N, d] (every token of
    this rank's heads: heads r*H/P .. (r+1)*H/P - 1 on rank r)."""
    P = dist.get_world_size(group)
    B, H, n, d = x.shape
    if H % P:
        raise ValueError(f"{H} heads do not split over {P} ranks")
    permute = permute or cuda_permute
    send = torch.empty((P, B, H // P, n, d), dtype=x.dtype, device=x.device)
    recv = torch.empty_like(send)
    permute(x, send, B, H, P, n, d, 0)
    dist.all_to_all_single(recv, send, group=group)
    out = torch.empty((B, H // P, P * n, d), dtype=x.dtype, device=x.device)
    permute(recv, out, B, H, P, n, d, 1)
    return out


def heads_to_seq(y: torch.Tensor, group=None, permute: Optional[Permute] = None) -> torch.Tensor:
    """Inverse of seq_to_heads: [B, H/P, N, d] -> [B, H, N/P, d]."""
    P = dist.get_world_size(group)
    B, Hp, N, d = y.shape
    if N % P:
        raise ValueError(f"{N} tokens do not split over {P} ranks")
    n, H = N // P, Hp * P
    permute = permute or cuda_permute
    send = torch.empty((P, B, Hp, n, d), dtype=y.dtype, device=y.device)
    recv = torch.empty_like(send)
    permute(y, send, B, H, P, n, d, 2)
    dist.all_to_all_single(recv, send, group=group)
    out = torch.empty((B, H, n, d), dtype=y.dtype, device=y.device)
    permute(recv, out, B, H, P, n, d, 3)
    return out


def sla_forward_ulysses(q, k, v, blk_q, blk_k, topk, phi, quant, ws=None, group=None, stream=None):
    """The SageSLA forward on token-sharded [B, H, N/P, d] inputs: all-to-all to the rank's
    heads, sla_forward on [B, H/P, N, d], all-to-all back.  Returns [B, H, N/P, d]."""
    qh, kh, vh = (seq_to_heads(x, group) for x in (q, k, v))
    B, Hp, N, d = qh.shape
    if ws is None:
        ws = workspace(B, Hp, N, d, blk_q, blk_k, topk, quant, device=q.device)
    oh = torch.empty_like(qh)
    sla_forward(qh, kh, vh, oh, blk_q, blk_k, topk, phi, quant, ws, stream=stream)
    return heads_to_seq(oh, group)
