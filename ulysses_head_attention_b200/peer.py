"""Ulysses' two all-to-alls between processes by peer stores, one GPU per rank.

Blog "Ulysses Sequence Parallelism: Training with Million-Token Contexts",
"How Ulysses works", steps 3 and 5; "Communication complexity".

Instead of packing, calling a collective and unpacking (distributed.py), each
rank stores its chunks straight into its peers' receive buffers with the
library's push kernels (ulysses_seq_to_head_push / ulysses_head_to_seq_push:
plain stores through peer-mapped pointers over NVLink, no staging copy), and
each destination waits on one flag per source (ulysses_wait_flags, bounded in
time) before it reads.

Buffers and flags, per rank, opened by every peer through CUDA IPC handles:
  recv_head[2]  (b, n, H/P, d)   the head-sharded result of seq_to_head
  recv_seq[2]   (b, n/P, H, d)   the seq-sharded result of head_to_seq
  flags         (4, P) uint32    rows: data seq->head, data head->seq,
                                 free seq->head, free head->seq
Receive buffers alternate between two copies by epoch, so a rank may push
epoch e while its peers still read epoch e - 1.  Before it pushes epoch e
into copy e % 2, a rank waits until every peer has released epoch e - 2 of
that copy ("free" row); a rank releases epoch e - 1 on all peers when it
starts exchange e in the same direction, after every kernel it enqueued on
the received buffer (stream order).  So a buffer is never overwritten while
it is read, and no kernel waits on a launch of its own GPU that has not been
enqueued before it.

``ops`` bundles the device operations (push, wait, release) and ``ipc`` the
handle export / open; the defaults call the library.  The CPU tests replace
both (numpy stores into shared memory, gloo for the handle exchange); the
product path always uses the library.
"""
from __future__ import annotations

import torch

from . import (alloc_workspace, ulysses_head_to_seq_push, ulysses_ipc_close, ulysses_ipc_handle, ulysses_ipc_open,
               ulysses_release_flags, ulysses_seq_to_head_push, ulysses_wait_flags, ulysses_workspace_status)

DATA_S2H, DATA_H2S, FREE_S2H, FREE_H2S = 0, 1, 2, 3


class CudaIpc:
    """CUDA IPC through the library: handles of local allocations, peer addresses of remote ones."""

    def handle(self, t: torch.Tensor) -> bytes:
        return ulysses_ipc_handle(t)

    def open(self, handle: bytes, like: torch.Tensor) -> int:
        return ulysses_ipc_open(handle)

    def close(self, addr: int) -> None:
        ulysses_ipc_close(addr)


class CudaOps:
    """The device operations of the exchange, on the current CUDA stream."""

    def __init__(self, device, limit_ns: int):
        self.limit_ns = limit_ns
        self.status = alloc_workspace(256, device)
        self.counters = alloc_workspace(4096, device)

    def push_s2h(self, x, dsts, flags, rank, P, epoch):
        ulysses_seq_to_head_push(x, dsts, flags, rank, P, epoch, self.counters)

    def push_h2s(self, x, dsts, flags, rank, P, epoch):
        ulysses_head_to_seq_push(x, dsts, flags, rank, P, epoch, self.counters)

    def wait(self, flags_row: torch.Tensor, epoch: int):
        ulysses_wait_flags(flags_row, epoch, self.limit_ns, self.status)

    def release(self, slot_addrs, epoch: int):
        """Store epoch into each address (a peer's flag slot for this rank)."""
        ulysses_release_flags(slot_addrs, epoch)

    def check(self):
        if ulysses_workspace_status(self.status) != 0:
            raise TimeoutError("a peer exchange wait gave up: a peer did not deliver in time")


class PeerExchange:
    """Ulysses' all-to-alls for one tensor shape (b, n, H, d) over a process group."""

    def __init__(self, group, b: int, n: int, H: int, d: int, dtype=torch.bfloat16, device=None,
                 ops=None, ipc=None, alloc=None, limit_ns: int = 10_000_000_000):
        import torch.distributed as dist
        self.group = group
        self.P = dist.get_world_size(group)
        self.rank = dist.get_rank(group)
        P = self.P
        if n % P or H % P:
            raise ValueError("n and H must be divisible by the group size")
        self.shape = (b, n, H, d)
        device = device if device is not None else torch.device("cuda", torch.cuda.current_device())
        self.ops = ops if ops is not None else CudaOps(device, limit_ns)
        self.ipc = ipc if ipc is not None else CudaIpc()
        h, m = H // P, n // P
        # buffers other ranks store into: allocated through `alloc` (zeroed), so
        # a stand-in can place them where its peers can reach them
        alloc = alloc if alloc is not None else (lambda shape, dt: torch.zeros(shape, dtype=dt, device=device))
        self.recv_head = [alloc((b, n, h, d), dtype) for _ in range(2)]
        self.recv_seq = [alloc((b, m, H, d), dtype) for _ in range(2)]
        self.flags = alloc((4, P), torch.int32)
        local = self.recv_head + self.recv_seq + [self.flags]
        mine = [self.ipc.handle(t) for t in local]
        everyone = [None] * P
        dist.all_gather_object(everyone, mine, group=group)
        self.peer = []        # per rank: addresses of its recv_head[0..1], recv_seq[0..1], flags
        self._opened = []
        for s in range(P):
            if s == self.rank:
                self.peer.append([t.data_ptr() for t in local])
            else:
                addrs = [self.ipc.open(hd, like) for hd, like in zip(everyone[s], local)]
                self._opened += addrs
                self.peer.append(addrs)
        self.epoch = [0, 0]   # last epoch per direction
        self.esize = self.flags.element_size()

    # address of rank s's flag slot [row][col]
    def _flag(self, s: int, row: int, col: int) -> int:
        return self.peer[s][4] + (row * self.P + col) * self.esize

    def _exchange(self, direction: int, x: torch.Tensor):
        P, r = self.P, self.rank
        e = self.epoch[direction] + 1
        copy = e % 2
        data_row, free_row = (DATA_S2H, FREE_S2H) if direction == 0 else (DATA_H2S, FREE_H2S)
        if e >= 2:   # this rank is done with what it received in epoch e - 1: tell its senders
            self.ops.release([self._flag(s, free_row, r) for s in range(P)], e - 1)
        if e >= 3:   # every receiver is done with copy e % 2 (epoch e - 2)
            self.ops.wait(self.flags[free_row], e - 2)
        dst = [self.peer[s][copy if direction == 0 else 2 + copy] for s in range(P)]
        flg = [self._flag(s, data_row, 0) for s in range(P)]
        if direction == 0:
            self.ops.push_s2h(x, dst, flg, r, P, e)
        else:
            self.ops.push_h2s(x, dst, flg, r, P, e)
        self.ops.wait(self.flags[data_row], e)
        self.epoch[direction] = e
        return (self.recv_head if direction == 0 else self.recv_seq)[copy]

    def seq_to_head(self, x_seq: torch.Tensor) -> torch.Tensor:
        """This rank's (b, n/P, H, d) shard -> (b, n, H/P, d), valid until the
        next-but-one call in this direction."""
        b, n, H, d = self.shape
        if tuple(x_seq.shape) != (b, n // self.P, H, d):
            raise ValueError("x_seq has the wrong shape")
        return self._exchange(0, x_seq.contiguous())

    def head_to_seq(self, x_head: torch.Tensor) -> torch.Tensor:
        """(b, n, H/P, d) -> this rank's (b, n/P, H, d), valid until the
        next-but-one call in this direction."""
        b, n, H, d = self.shape
        if tuple(x_head.shape) != (b, n, H // self.P, d):
            raise ValueError("x_head has the wrong shape")
        return self._exchange(1, x_head.contiguous())

    def check(self) -> None:
        """Synchronize and raise if any bounded wait gave up."""
        self.ops.check()

    def close(self) -> None:
        for a in self._opened:
            self.ipc.close(a)
        self._opened = []
