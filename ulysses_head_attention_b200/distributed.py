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

K and V with fewer kv heads than ranks (H_kv < P, P a multiple of H_kv; the
pages are silent on this case) go through ``kv_seq_to_head`` and
``kv_head_to_seq``: rank s receives all n tokens of kv head s H_kv/P, the
one its query heads read, and the gradients of the P/H_kv copies of a head
are summed on the way back (the one-GPU ``ulysses_kv_seq_to_head`` /
``ulysses_kv_head_to_seq`` contract, split over processes).  The copies are
made and summed by the library's kv re-layout kernels, applied to one kv
head's block of rows at a time.

The pack and unpack run on this package's CUDA kernels; the exchange is
NCCL's all-to-all.  ``transpose``, ``replicate``, ``reduce`` and
``exchange`` can be replaced (the CPU tests of the step order use numpy and
gloo stand-ins); the product path always uses the defaults.
"""
from __future__ import annotations

from typing import Callable, Optional

import torch

from . import ulysses_kv_head_to_seq, ulysses_kv_seq_to_head, ulysses_transpose_runs

Transpose = Callable[[torch.Tensor, torch.Tensor, int, int, int], None]
Exchange = Callable[[torch.Tensor, torch.Tensor, object], None]
Copies = Callable[[torch.Tensor, torch.Tensor, int, int, int], None]


def _cuda_transpose(src: torch.Tensor, dst: torch.Tensor, A: int, B: int, run_bytes: int) -> None:
    ulysses_transpose_runs(src, dst, A, B, run_bytes)


def _cuda_replicate(src: torch.Tensor, dst: torch.Tensor, R: int, T: int, d: int) -> None:
    """dst[c] = src for c < R: src (T, d) rows, dst (R, T, d).  The kv copy
    kernel with R ranks and one kv head: every rank receives the one head's
    T tokens, read as R shards of T/R tokens."""
    ulysses_kv_seq_to_head(src.view(R, 1, T // R, 1, d), dst.view(R, 1, T, 1, d))


def _cuda_reduce(src: torch.Tensor, dst: torch.Tensor, R: int, T: int, d: int) -> None:
    """dst = sum over c < R of src[c] (ascending, float32 accumulation): src
    (R, T, d), dst (T, d).  The kv sum kernel with R ranks holding copies of
    one kv head; its output shards of T/R tokens are dst's rows in order."""
    ulysses_kv_head_to_seq(src.view(R, 1, T, 1, d), dst.view(R, 1, T // R, 1, d))


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


def kv_seq_to_head(x_seq: torch.Tensor, group=None, out: Optional[torch.Tensor] = None,
                   transpose: Transpose = _cuda_transpose, replicate: Copies = _cuda_replicate,
                   exchange: Exchange = _nccl_exchange) -> torch.Tensor:
    """First all-to-all for K or V: (b, n/P, H_kv, d) -> (b, n, H_kv/P, d), or
    (b, n, 1, d) holding kv head r H_kv/P when H_kv < P (P a multiple of H_kv).

      pack       (b n/P, H_kv, d) -> (H_kv, b n/P, d): one block of rows per kv head;
      copy       send slots [g R, (g+1) R) <- R copies of head g's block (R = P/H_kv);
      exchange   slot s goes to rank s;
      unpack     (P, b, n/P d) -> (b, P, n/P d) = (b, n, 1, d).
    """
    P = _group_size(group)
    b, m, H, d = x_seq.shape
    if H % P == 0:
        return seq_to_head(x_seq, group, out, transpose, exchange)
    if P % H:
        raise ValueError("the kv head count must be a multiple or a divisor of the group size")
    R, T = P // H, b * m
    if T % R:
        raise ValueError("b * n/P must be a multiple of (group size / kv heads)")
    es = x_seq.element_size()
    if out is None:
        out = torch.empty((b, m * P, 1, d), dtype=x_seq.dtype, device=x_seq.device)
    elif tuple(out.shape) != (b, m * P, 1, d) or out.dtype != x_seq.dtype:
        raise ValueError("out has the wrong shape or dtype")
    packed = torch.empty((H, b, m, d), dtype=x_seq.dtype, device=x_seq.device)
    send = torch.empty((P, b, m, d), dtype=x_seq.dtype, device=x_seq.device)
    recv = torch.empty_like(send)
    transpose(x_seq.contiguous(), packed, T, H, d * es)             # pack by kv head
    for g in range(H):
        replicate(packed[g], send[g * R:(g + 1) * R], R, T, d)      # a copy for each rank reading head g
    exchange(recv, send, group)                                      # all-to-all
    transpose(recv, out, P, b, m * d * es)                           # unpack
    return out


def kv_head_to_seq(x_head: torch.Tensor, H_kv: int, group=None, out: Optional[torch.Tensor] = None,
                   transpose: Transpose = _cuda_transpose, reduce: Copies = _cuda_reduce,
                   exchange: Exchange = _nccl_exchange) -> torch.Tensor:
    """Backward of kv_seq_to_head, for dK / dV: (b, n, H_kv/P or 1, d) ->
    (b, n/P, H_kv, d); with H_kv < P the gradients of a head's R = P/H_kv
    copies are summed (ascending rank, float32 accumulation).

      pack       (b, P, n/P d) -> (P, b, n/P d): slot s = this rank's rows of rank s's tokens;
      exchange   slot r of the result = rank r's gradient (of head r H_kv/P) for this rank's tokens;
      sum        head g = sum of slots [g R, (g+1) R);
      unpack     (H_kv, b n/P, d) -> (b n/P, H_kv, d).
    """
    P = _group_size(group)
    if H_kv % P == 0:
        return head_to_seq(x_head, group, out, transpose, exchange)
    if P % H_kv:
        raise ValueError("the kv head count must be a multiple or a divisor of the group size")
    b, n, one, d = x_head.shape
    if one != 1 or n % P:
        raise ValueError("x_head must be (b, n, 1, d) with n divisible by the group size")
    m = n // P
    R, T = P // H_kv, b * m
    if T % R:
        raise ValueError("b * n/P must be a multiple of (group size / kv heads)")
    es = x_head.element_size()
    if out is None:
        out = torch.empty((b, m, H_kv, d), dtype=x_head.dtype, device=x_head.device)
    elif tuple(out.shape) != (b, m, H_kv, d) or out.dtype != x_head.dtype:
        raise ValueError("out has the wrong shape or dtype")
    send = torch.empty((P, b, m, d), dtype=x_head.dtype, device=x_head.device)
    recv = torch.empty_like(send)
    summed = torch.empty((H_kv, b, m, d), dtype=x_head.dtype, device=x_head.device)
    transpose(x_head.contiguous(), send, b, P, m * d * es)           # pack by destination
    exchange(recv, send, group)                                      # all-to-all
    for g in range(H_kv):
        reduce(recv[g * R:(g + 1) * R], summed[g], R, T, d)          # sum the copies of head g
    transpose(summed, out, H_kv, T, d * es)                          # unpack
    return out
