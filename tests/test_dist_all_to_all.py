"""The multi-process all-to-alls (ulysses_head_attention_b200.distributed) on CPU.

Two and three gloo ranks on 127.0.0.1 run the module's seq_to_head and
head_to_seq with its pack / exchange / unpack order; the CUDA transpose is
replaced by a numpy one with the same contract (dst[j][i] = src[i][j] over
byte runs) and NCCL by gloo's all_to_all_single.  Each rank's result must
equal its slice of the oracle's one-buffer re-layout, bit for bit, and the
way back must return its shard.  The K/V variants for fewer kv heads than
ranks (kv_seq_to_head / kv_head_to_seq) run the same way with numpy
stand-ins for the copy and sum kernels, against the oracle's replicated
re-layout and its summed gradient.  The CUDA transpose itself, and the same
three steps emulated for P ranks on one GPU, are checked in
test_gpu_dist_emulated.py.
"""
import datetime
import os
import socket
import sys

import numpy as np
import pytest

from conftest import ROOT


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def numpy_transpose(src, dst, A, B, run_bytes):
    """dst[j][i][:] = src[i][j][:] over byte runs (the CUDA kernel's contract)."""
    import torch
    s = src.contiguous().view(-1).view(torch.uint8).numpy().reshape(A, B, run_bytes)
    d = np.ascontiguousarray(s.transpose(1, 0, 2))
    dst.view(-1).view(torch.uint8).numpy()[:] = d.reshape(-1)


def numpy_replicate(src, dst, R, T, d):
    """dst[c] = src for c < R (the kv copy kernel's contract, one head)."""
    import torch
    s = src.contiguous().view(-1).view(torch.uint8).numpy()
    dst.view(-1).view(torch.uint8).numpy()[:] = np.tile(s, R)


def numpy_reduce(src, dst, R, T, d):
    """dst = src[0] + src[1] + ... in float32, rounded once (the kv sum kernel's contract)."""
    import torch
    acc = np.zeros(T * d, dtype=np.float32)
    for c in range(R):
        acc += src[c].float().reshape(-1).numpy()
    dst.view(-1).copy_(torch.from_numpy(acc).to(dst.dtype))


def gloo_exchange(recv, send, group):
    import torch.distributed as dist
    dist.all_to_all_single(recv, send, group=group)


def _rank_main(rank, world, port, root, out):
    sys.path.insert(0, root)
    import torch
    import torch.distributed as dist
    import oracle
    from ulysses_head_attention_b200 import distributed as udist
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=30))
    try:
        b, m, H, d = 2, 5, 2 * world, 3
        rng = np.random.default_rng(11)                          # same global tensor on every rank
        glob = rng.integers(-2 ** 15, 2 ** 15, (world, b, m, H, d)).astype(np.int16)
        mine = torch.from_numpy(glob[rank].copy()).view(torch.bfloat16)
        head = udist.seq_to_head(mine, transpose=numpy_transpose, exchange=gloo_exchange)
        want = oracle.seq_to_head(glob, world)[rank]
        ok1 = np.array_equal(head.view(torch.int16).numpy(), want)
        back = udist.head_to_seq(head, transpose=numpy_transpose, exchange=gloo_exchange)
        ok2 = np.array_equal(back.view(torch.int16).numpy(), glob[rank])
        # fp32 as well (run sizes that are not multiples of 16 bytes)
        gf = rng.standard_normal((world, b, m, H, d)).astype(np.float32)
        hf = udist.seq_to_head(torch.from_numpy(gf[rank].copy()), transpose=numpy_transpose, exchange=gloo_exchange)
        ok3 = np.array_equal(hf.numpy(), oracle.seq_to_head(gf, world)[rank])
        dist.barrier()
        out.put((rank, ok1, ok2, ok3))
    except Exception as e:   # report instead of leaving the test to time out
        out.put((rank, False, False, repr(e)))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 3])
def test_all_to_all_round_trip_over_gloo(world):
    import torch.multiprocessing as mp
    ctx = mp.get_context("spawn")
    out = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, ROOT, out)) for r in range(world)]
    for p in procs:
        p.start()
    try:
        res = sorted((out.get(timeout=120) for _ in range(world)), key=lambda r: r[0])
    finally:
        for p in procs:
            p.join(timeout=60)
            if p.is_alive():
                p.kill()
    assert [r[0] for r in res] == list(range(world))
    assert all(r[1] and r[2] and r[3] is True for r in res), res
    assert all(p.exitcode == 0 for p in procs)


def _rank_dies(rank, world, port, root, out):
    sys.path.insert(0, root)
    import time
    import torch
    import torch.distributed as dist
    from ulysses_head_attention_b200 import distributed as udist
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=5))
    if rank == 1:
        out.put((rank, "left before the exchange"))
        out.close()
        out.join_thread()               # the message is out before the process goes
        os._exit(0)                     # a rank that never joins the all-to-all
    t0 = time.time()
    try:
        udist.seq_to_head(torch.zeros((1, 4, 2 * world, 2)), transpose=numpy_transpose, exchange=gloo_exchange)
        out.put((rank, "completed"))
    except Exception as e:               # the survivor must get an error, not hang
        out.put((rank, f"error after {time.time() - t0:.1f}s: {type(e).__name__}"))
    out.close()
    out.join_thread()
    os._exit(0)


def test_a_rank_that_leaves_ends_the_exchange_with_an_error():
    import torch.multiprocessing as mp
    ctx = mp.get_context("spawn")
    out = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_dies, args=(r, 2, port, ROOT, out)) for r in range(2)]
    for p in procs:
        p.start()
    try:
        res = dict(out.get(timeout=120) for _ in range(2))
    finally:
        for p in procs:
            p.join(timeout=60)
            if p.is_alive():
                p.kill()
    assert res[1] == "left before the exchange"
    assert res[0].startswith("error after"), res[0]


def _kv_rank_main(rank, world, H_kv, port, root, out):
    sys.path.insert(0, root)
    import torch
    import torch.distributed as dist
    import oracle
    from ulysses_head_attention_b200 import distributed as udist
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=30))
    try:
        b, m, d = 2, 4, 3
        rng = np.random.default_rng(21 + world)
        # forward: bf16 bits, a bit-exact copy
        glob = rng.integers(-2 ** 15, 2 ** 15, (world, b, m, H_kv, d)).astype(np.int16)
        mine = torch.from_numpy(glob[rank].copy()).view(torch.bfloat16)
        head = udist.kv_seq_to_head(mine, transpose=numpy_transpose, replicate=numpy_replicate,
                                    exchange=gloo_exchange)
        ok1 = np.array_equal(head.view(torch.int16).numpy(), oracle.kv_seq_to_head(glob, world)[rank])
        # backward: integer-valued fp32 gradients, so every summation order is exact
        gh = rng.integers(-1000, 1000, (world, b, m * world, 1, d)).astype(np.float32)
        grad = udist.kv_head_to_seq(torch.from_numpy(gh[rank].copy()), H_kv, transpose=numpy_transpose,
                                    reduce=numpy_reduce, exchange=gloo_exchange)
        want = oracle.kv_head_to_seq_reduce(gh.astype(np.float64), world, H_kv)[rank]
        ok2 = np.array_equal(grad.numpy().astype(np.float64), want)
        dist.barrier()
        out.put((rank, ok1, ok2))
    except Exception as e:   # report instead of leaving the test to time out
        out.put((rank, False, repr(e)))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world,H_kv", [(2, 1), (4, 2), (4, 1)])
def test_kv_all_to_all_with_fewer_kv_heads_than_ranks(world, H_kv):
    import torch.multiprocessing as mp
    ctx = mp.get_context("spawn")
    out = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_kv_rank_main, args=(r, world, H_kv, port, ROOT, out)) for r in range(world)]
    for p in procs:
        p.start()
    try:
        res = sorted((out.get(timeout=120) for _ in range(world)), key=lambda r: r[0])
    finally:
        for p in procs:
            p.join(timeout=60)
            if p.is_alive():
                p.kill()
    assert [r[0] for r in res] == list(range(world))
    assert all(r[1] is True and r[2] is True for r in res), res
    assert all(p.exitcode == 0 for p in procs)
