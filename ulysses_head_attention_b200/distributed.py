"""Ulysses' two all-to-alls between processes, one GPU per SP rank.

Blog "Ulysses Sequence Parallelism: Training with Million-Token Contexts",
"How Ulysses works", steps 3 and 5; Transformers docs "Ulysses sequence
parallelism" (the seq-sharded -> head-sharded -> seq-sharded figure).

Rank r of a P-process group holds its seq shard x (b, n/P, H, d): tokens
[r n/P, (r+1) n/P) with every head.  The first all-to-all leaves it all n
tokens of its heads [r H/P, (r+1) H/P), laid out (b, n, H/P, d) exactly like
rank r's slice of the one-GPU ``ulysses_seq_to_head`` output; the second is
the inverse.  Each is three steps:

  pack      ulysses_transpose_runs: (b n/P, P, H/P d) -> (P, b n/P, H/P d):
            chunk s holds this rank's tokens of rank s's heads;
  exchange  torch.distributed.all_to_all_single (NCCL between GPUs): chunk s
            goes to rank s, the chunk from rank s lands in slot s;
  unpack    ulysses_transpose_runs: (P, b, n/P H/P d) -> (b, P, n/P H/P d),
            i.e. (b, n, H/P, d) with rank s's tokens at [s n/P, (s+1) n/P).

The pack and unpack run on this package's CUDA kernels; the exchange is
NCCL's all-to-all.  ``transpose`` and ``exchange`` can be replaced (the CPU
tests of the step order use numpy and gloo stand-ins); the product path
always uses the defaults.
"""
from __future__ import annotations

from typing import Callable, Optional

import torch

from . import ulysses_transpose_runs

Transpose = Callable[[torch.Tensor, torch.Tensor, int, int, int], None]
Exchange = Callable[[torch.Tensor, torch.Tensor, object], None]


def _cuda_transpose(src: torch.Tensor, dst: torch.Tensor, A: int, B: int, run_bytes: int) -> None:
    ulysses_transpose_runs(src, dst, A, B, run_bytes)


def _nccl_exchange(recv: torch.Tensor, send: torch.Tensor, group) -> None:
    import torch.distributed as dist
    dist.all_to_all_single(recv, send, group=group)


def _group_size(group) -> int:
    import torch.distributed as dist
    return dist.get_world_size(group)


def seq_to_head(x_seq: torch.Tensor, group=None, out: Optional[torch.Tensor] = None,
                transpose: Transpose = _cuda_transpose, exchange: Exchange = _nccl_exchange) -> torch.Tensor:
    """First all-to-all: this rank's (b, n/P, H, d) shard -> (b, n, H/P, d)."""
    P = _group_size(group)
    b, m, H, d = x_seq.shape
    if H % P:
        raise ValueError("the head count must be divisible by the group size")
    h = H // P
    es = x_seq.element_size()
    send = torch.empty((P, b, m, h, d), dtype=x_seq.dtype, device=x_seq.device)
    recv = torch.empty_like(send)
    if out is None:
        out = torch.empty((b, m * P, h, d), dtype=x_seq.dtype, device=x_seq.device)
    elif tuple(out.shape) != (b, m * P, h, d) or out.dtype != x_seq.dtype:
        raise ValueError("out has the wrong shape or dtype")
    transpose(x_seq.contiguous(), send, b * m, P, h * d * es)      # pack
    exchange(recv, send, group)                                    # all-to-all
    transpose(recv, out, P, b, m * h * d * es)                     # unpack
    return out


def head_to_seq(x_head: torch.Tensor, group=None, out: Optional[torch.Tensor] = None,
                transpose: Transpose = _cuda_transpose, exchange: Exchange = _nccl_exchange) -> torch.Tensor:
    """Second all-to-all (and the backward of the first): (b, n, H/P, d) -> (b, n/P, H, d)."""
    P = _group_size(group)
    b, n, h, d = x_head.shape
    if n % P:
        raise ValueError("the sequence length must be divisible by the group size")
    m = n // P
    es = x_head.element_size()
    send = torch.empty((P, b, m, h, d), dtype=x_head.dtype, device=x_head.device)
    recv = torch.empty_like(send)
    if out is None:
        out = torch.empty((b, m, h * P, d), dtype=x_head.dtype, device=x_head.device)
    elif tuple(out.shape) != (b, m, h * P, d) or out.dtype != x_head.dtype:
        raise ValueError("out has the wrong shape or dtype")
    transpose(x_head.contiguous(), send, b, P, m * h * d * es)     # (b, P, m h d) -> (P, b, m h d)
    exchange(recv, send, group)                                    # chunk s: rank s's heads of my tokens
    transpose(recv, out, P, b * m, h * d * es)                     # (P, b m, h d) -> (b m, P, h d)
    return out
