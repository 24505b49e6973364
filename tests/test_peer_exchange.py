"""The multi-process peer-store exchange (ulysses_head_attention_b200.peer) on CPU.

Three gloo ranks on 127.0.0.1 run PeerExchange with its device operations
replaced by numpy stand-ins that keep the kernels' contracts: the push
stores this rank's chunks into every rank's receive buffer and then stores
the epoch into the destination's flag slot; the wait spins (bounded) until
a flag row reaches an epoch; the release stores an epoch into peers' slots.
Receive buffers and flags live in POSIX shared memory, so the stores of one
process land in the others' buffers as peer stores over NVLink would, and
the "IPC handle" is the shared-memory block's name.  Checked: every
exchange in both directions equals the oracle's re-layout of all ranks'
shards, over several epochs (the two buffer copies alternate and the free /
data flag protocol keeps them apart), and a rank that never joins an
exchange makes the others' bounded waits give up instead of hanging.
The CUDA push and wait kernels themselves are checked with emulated ranks
on one GPU (test_gpu_exchange.py).
"""
import datetime
import os
import socket
import sys
import time

import numpy as np
import pytest

from conftest import ROOT


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


class Shm:
    """Shared-memory buffers addressed like device memory: address -> (base, tensor)."""

    def __init__(self):
        self.blocks = []     # (base address, nbytes, torch tensor, SharedMemory)

    def alloc(self, shape, dtype):
        import torch
        from multiprocessing import shared_memory
        nbytes = int(np.prod(shape)) * torch.empty((), dtype=dtype).element_size()
        shm = shared_memory.SharedMemory(create=True, size=nbytes)
        t = torch.frombuffer(shm.buf, dtype=dtype, count=int(np.prod(shape))).view(shape)
        t.zero_()
        shm._uly_own = True
        self.blocks.append((t.data_ptr(), nbytes, t, shm))
        return t

    def attach(self, name, like):
        import torch
        from multiprocessing import shared_memory
        shm = shared_memory.SharedMemory(name=name)
        t = torch.frombuffer(shm.buf, dtype=like.dtype, count=like.numel()).view(like.shape)
        self.blocks.append((t.data_ptr(), t.numel() * t.element_size(), t, shm))
        return t.data_ptr()

    def name_of(self, t):
        for base, nb, tt, shm in self.blocks:
            if base == t.data_ptr():
                return shm.name
        raise KeyError("not a shared buffer")

    def tensor_at(self, addr):
        for base, nb, t, shm in self.blocks:
            if base <= addr < base + nb:
                return t, addr - base
        raise KeyError(hex(addr))

    def int32_at(self, addr):
        t, off = self.tensor_at(addr)
        return t.view(-1).numpy().view(np.uint8)[off:off + 4].view(np.int32)

    def unlink_own(self):
        """Remove the blocks this process created (peers' mappings stay valid until they exit)."""
        for base, nb, t, shm in self.blocks:
            if getattr(shm, "_uly_own", False):
                shm.unlink()


class ShmIpc:
    def __init__(self, mem):
        self.mem = mem

    def handle(self, t):
        return self.mem.name_of(t)

    def open(self, handle, like):
        return self.mem.attach(handle, like)

    def close(self, addr):
        pass


class NumpyOps:
    """The push / wait / release contracts, on host memory."""

    def __init__(self, mem, shape, limit_s=20.0):
        self.mem, self.limit_s = mem, limit_s
        self.b, self.n, self.H, self.d = shape

    def _push(self, x, dsts, flags, r, P, e, to_head):
        b, n, H, d = self.b, self.n, self.H, self.d
        m, h = n // P, H // P
        xs = x.numpy()
        for s in range(P):
            t, off = self.mem.tensor_at(dsts[s])
            assert off == 0
            dst = t.numpy()
            if to_head:
                dst[:, r * m:(r + 1) * m] = xs[:, :, s * h:(s + 1) * h]
            else:
                dst[:, :, r * h:(r + 1) * h] = xs[:, s * m:(s + 1) * m]
            self.mem.int32_at(flags[s] + 4 * r)[0] = e

    def push_s2h(self, x, dsts, flags, r, P, e):
        self._push(x, dsts, flags, r, P, e, True)

    def push_h2s(self, x, dsts, flags, r, P, e):
        self._push(x, dsts, flags, r, P, e, False)

    def wait(self, row, e):
        t0 = time.time()
        while not all(int(np.int32(np.uint32(v) - np.uint32(e))) >= 0 for v in row.numpy().astype(np.int64) & 0xFFFFFFFF):
            if time.time() - t0 > self.limit_s:
                raise TimeoutError("flag wait gave up")
            time.sleep(0.001)

    def release(self, addrs, e):
        for a in addrs:
            self.mem.int32_at(a)[0] = e

    def check(self):
        pass


def _inputs(rank, epoch, shape, P, direction):
    b, n, H, d = shape
    rng = np.random.default_rng(1000 * epoch + 10 * rank + direction)
    if direction == 0:
        return rng.standard_normal((b, n // P, H, d)).astype(np.float32)
    return rng.standard_normal((b, n, H // P, d)).astype(np.float32)


def _rank_main(rank, world, port, root, out, epochs, absent):
    sys.path.insert(0, root)
    import torch
    import torch.distributed as dist
    import oracle
    from ulysses_head_attention_b200 import peer
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    mem = Shm()
    shape = (1, 24, 6, 4)
    P = world
    try:
        ex = peer.PeerExchange(None, *shape, dtype=torch.float32, device="cpu", ops=NumpyOps(mem, shape, 3.0 if absent is not None else 20.0),
                               ipc=ShmIpc(mem), alloc=mem.alloc)
        dist.barrier()
        if rank == absent:   # never joins: the others must give up, not hang
            out.put((rank, "absent"))
            time.sleep(6.0)
            return
        ok = True
        try:
            for e in range(1, epochs + 1):
                xs = _inputs(rank, e, shape, P, 0)
                got = ex.seq_to_head(torch.from_numpy(xs)).numpy().copy()
                all_seq = np.stack([_inputs(s, e, shape, P, 0) for s in range(P)])      # [P][b][m][H][d]
                want = oracle.seq_to_head(all_seq, P)[rank]
                ok = ok and np.array_equal(got, want)
                xh = _inputs(rank, e, shape, P, 1)
                got = ex.head_to_seq(torch.from_numpy(xh)).numpy().copy()
                all_head = np.stack([_inputs(s, e, shape, P, 1) for s in range(P)])     # [P][b][n][h][d]
                want = oracle.head_to_seq(all_head, P)[rank]
                ok = ok and np.array_equal(got, want)
            out.put((rank, ok))
        except TimeoutError:
            out.put((rank, "timeout"))
        dist.barrier()
    finally:
        mem.unlink_own()
        if absent is None:
            dist.destroy_process_group()


def _run(world, epochs, absent=None):
    import torch.multiprocessing as mp
    ctx = mp.get_context("spawn")
    out = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, ROOT, out, epochs, absent)) for r in range(world)]
    for p in procs:
        p.start()
    try:
        got = sorted(out.get(timeout=240) for _ in range(world))
    finally:
        for p in procs:
            p.join(timeout=30)
            if p.is_alive():
                p.kill()
    return got


def test_three_ranks_several_epochs_match_the_oracle():
    got = _run(3, epochs=5)
    assert got == [(0, True), (1, True), (2, True)]


def test_a_rank_that_never_joins_makes_the_waits_give_up():
    got = _run(3, epochs=2, absent=2)
    assert got == [(0, "timeout"), (1, "timeout"), (2, "absent")]
