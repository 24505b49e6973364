"""The all-to-alls of ulysses_head_attention_b200.distributed (seq_to_head /
head_to_seq, and kv_seq_to_head / kv_head_to_seq for fewer kv heads than
ranks), with P ranks emulated by P host threads in one process.

Each thread runs the module's call for its rank;
the exchange stand-in publishes the rank's send buffer, waits for every rank
on a host barrier (bounded), copies chunk r of every rank s into slot s of
its receive buffer, and waits again.  No kernel waits on another: all
waiting is on the host.  On the GPU the pack, copy, sum and unpack steps are
the library's kernels, and the result must equal the one-GPU re-layouts
(ulysses_seq_to_head, ulysses_kv_seq_to_head / ulysses_kv_head_to_seq) bit
for bit, and the oracle.  The same harness runs on the CPU with numpy
stand-ins for the kernels, or with the module's own kernel wrappers over a
shape-checking stand-in of the binding, which checks the harness and the
wrappers' views where no GPU is present.
"""
import threading

import numpy as np
import pytest
import torch

import oracle

BARRIER_TIMEOUT_S = 60


def emulate_ranks(P, fn):
    """Run fn(rank, exchange) for ranks 0..P-1 on P threads; returns the results."""
    sends, recvs = [None] * P, [None] * P
    barrier = threading.Barrier(P)
    results, errors = [None] * P, []

    def make_exchange(r):
        def exchange(recv, send, group):
            sends[r], recvs[r] = send, recv
            if send.is_cuda:
                torch.cuda.synchronize()
            barrier.wait(timeout=BARRIER_TIMEOUT_S)
            for s in range(P):
                recv[s].copy_(sends[s][r])        # chunk r of rank s lands in slot s
            if send.is_cuda:
                torch.cuda.synchronize()
            barrier.wait(timeout=BARRIER_TIMEOUT_S)
        return exchange

    def body(r):
        try:
            results[r] = fn(r, make_exchange(r))
        except BaseException as e:  # noqa: BLE001 -- reported below; the other ranks are released
            errors.append(e)
            barrier.abort()

    threads = [threading.Thread(target=body, args=(r,)) for r in range(P)]
    for t in threads:
        t.start()
    for t in threads:
        t.join(timeout=4 * BARRIER_TIMEOUT_S)
    assert not any(t.is_alive() for t in threads), "an emulated rank did not finish"
    if errors:
        raise errors[0]
    return results


def _numpy_transpose(src, dst, A, B, run_bytes):
    s = src.contiguous().view(-1).view(torch.uint8).numpy().reshape(A, B, run_bytes)
    dst.view(-1).view(torch.uint8).numpy()[:] = np.ascontiguousarray(s.transpose(1, 0, 2)).reshape(-1)


def _numpy_replicate(src, dst, R, T, d):
    dst.view(-1).view(torch.uint8).numpy()[:] = np.tile(src.contiguous().view(-1).view(torch.uint8).numpy(), R)


def _numpy_reduce(src, dst, R, T, d):
    acc = np.zeros(T * d, dtype=np.float32)
    for c in range(R):
        acc += src[c].float().reshape(-1).numpy()
    dst.view(-1).copy_(torch.from_numpy(acc).to(dst.dtype))


def _run(P, H_kv, b, m, d, device, monkeypatch, kernels):
    from ulysses_head_attention_b200 import distributed as udist
    monkeypatch.setattr(udist, "_group_size", lambda group: P)
    rng = np.random.default_rng(P * 10 + H_kv)
    x = rng.integers(-2 ** 15, 2 ** 15, (P, b, m, H_kv, d)).astype(np.int16)        # bf16 bits
    g = rng.integers(-1000, 1000, (P, b, m * P, 1, d)).astype(np.float32)            # exact sums
    xs = torch.from_numpy(x).view(torch.bfloat16).to(device)
    gs = torch.from_numpy(g).to(device)

    def fwd(r, exchange):
        return udist.kv_seq_to_head(xs[r].contiguous(), exchange=exchange, **kernels["fwd"])

    def bwd(r, exchange):
        return udist.kv_head_to_seq(gs[r].contiguous(), H_kv, exchange=exchange, **kernels["bwd"])

    heads = torch.stack(emulate_ranks(P, fwd))
    grads = torch.stack(emulate_ranks(P, bwd))
    assert np.array_equal(heads.view(torch.int16).cpu().numpy(), oracle.kv_seq_to_head(x, P))
    assert np.array_equal(grads.cpu().numpy().astype(np.float64),
                          oracle.kv_head_to_seq_reduce(g.astype(np.float64), P, H_kv))
    return xs, gs, heads, grads


@pytest.mark.parametrize("P,H_kv", [(4, 2), (8, 2), (4, 1)])
def test_harness_with_numpy_kernels(P, H_kv, monkeypatch):
    kernels = {"fwd": dict(transpose=_numpy_transpose, replicate=_numpy_replicate),
               "bwd": dict(transpose=_numpy_transpose, reduce=_numpy_reduce)}
    _run(P, H_kv, 2, 4, 3, torch.device("cpu"), monkeypatch, kernels)


@pytest.mark.gpu
@pytest.mark.parametrize("P,H_kv,b,m", [(4, 2, 1, 256), (8, 2, 2, 64), (16, 8, 1, 128), (4, 1, 1, 512)])
def test_kv_all_to_alls_on_gpu_equal_the_one_gpu_relayouts(cuda_device, P, H_kv, b, m, monkeypatch):
    import ulysses_head_attention_b200 as uly
    d = 128
    xs, gs, heads, grads = _run(P, H_kv, b, m, d, cuda_device, monkeypatch, {"fwd": {}, "bwd": {}})
    one = torch.empty((P, b, m * P, 1, d), dtype=torch.bfloat16, device=cuda_device)
    uly.ulysses_kv_seq_to_head(xs, one)
    assert torch.equal(heads.view(torch.int16), one.view(torch.int16))
    back = torch.empty((P, b, m, H_kv, d), dtype=torch.float32, device=cuda_device)
    uly.ulysses_kv_head_to_seq(gs, back)
    assert torch.equal(grads, back)


def _fake_kv_seq_to_head(x_seq, x_head, stream=None):
    """The binding's contract and shape rule for ulysses_kv_seq_to_head, on host tensors."""
    P, b, m, H, d = x_seq.shape
    assert tuple(x_head.shape) == (P, b, m * P, H // P if H >= P else 1, d) and x_head.dtype == x_seq.dtype
    assert x_seq.is_contiguous() and x_head.is_contiguous() and x_seq.dtype == torch.bfloat16
    x_head.view(torch.int16).numpy()[:] = oracle.kv_seq_to_head(x_seq.view(torch.int16).numpy(), P)


def _fake_kv_head_to_seq(x_head, x_seq, stream=None):
    P, b, m, H, d = x_seq.shape
    assert tuple(x_head.shape) == (P, b, m * P, H // P if H >= P else 1, d) and x_head.dtype == x_seq.dtype
    assert x_seq.is_contiguous() and x_head.is_contiguous()
    out = oracle.kv_head_to_seq_reduce(x_head.double().numpy(), P, H)
    x_seq.copy_(torch.from_numpy(out).to(x_seq.dtype))


def _fake_transpose_runs(src, dst, A, B, run_bytes, stream=None):
    assert src.numel() * src.element_size() == A * B * run_bytes == dst.numel() * dst.element_size()
    _numpy_transpose(src, dst, A, B, run_bytes)


@pytest.mark.parametrize("P,H_kv,b,m", [(4, 2, 1, 8), (8, 2, 2, 4), (16, 8, 1, 4), (4, 1, 1, 8)])
def test_kernel_wrappers_hand_the_binding_valid_shapes(P, H_kv, b, m, monkeypatch):
    """The module's default kernel wrappers, with the binding replaced by host
    stand-ins that enforce its shape rules: the views the wrappers build for
    the kv copy and sum kernels are the ones those calls accept, and the
    results equal the oracle's."""
    from ulysses_head_attention_b200 import distributed as udist
    monkeypatch.setattr(udist, "ulysses_kv_seq_to_head", _fake_kv_seq_to_head)
    monkeypatch.setattr(udist, "ulysses_kv_head_to_seq", _fake_kv_head_to_seq)
    monkeypatch.setattr(udist, "ulysses_transpose_runs", _fake_transpose_runs)
    _run(P, H_kv, b, m, 8, torch.device("cpu"), monkeypatch, {"fwd": {}, "bwd": {}})


def _run_plain(P, H, b, m, d, device, monkeypatch, kernels):
    """seq_to_head / head_to_seq of the module (H divisible by P), emulated ranks."""
    from ulysses_head_attention_b200 import distributed as udist
    monkeypatch.setattr(udist, "_group_size", lambda group: P)
    rng = np.random.default_rng(P * 100 + H)
    x = rng.integers(-2 ** 15, 2 ** 15, (P, b, m, H, d)).astype(np.int16)
    xs = torch.from_numpy(x).view(torch.bfloat16).to(device)
    heads = torch.stack(emulate_ranks(P, lambda r, ex: udist.seq_to_head(xs[r].contiguous(), exchange=ex,
                                                                          **kernels)))
    assert np.array_equal(heads.view(torch.int16).cpu().numpy(), oracle.seq_to_head(x, P))
    back = torch.stack(emulate_ranks(P, lambda r, ex: udist.head_to_seq(heads[r].contiguous(), exchange=ex,
                                                                         **kernels)))
    assert torch.equal(back.view(torch.int16), xs.view(torch.int16))
    return xs, heads


@pytest.mark.parametrize("P,H,b,m", [(2, 4, 2, 4), (4, 8, 1, 8)])
def test_plain_wrappers_hand_the_binding_valid_shapes(P, H, b, m, monkeypatch):
    from ulysses_head_attention_b200 import distributed as udist
    monkeypatch.setattr(udist, "ulysses_transpose_runs", _fake_transpose_runs)
    _run_plain(P, H, b, m, 8, torch.device("cpu"), monkeypatch, {})


@pytest.mark.gpu
@pytest.mark.parametrize("P,H,b,m", [(4, 32, 1, 256), (8, 8, 2, 64)])
def test_plain_all_to_alls_on_gpu_equal_the_one_gpu_relayout(cuda_device, P, H, b, m, monkeypatch):
    import ulysses_head_attention_b200 as uly
    xs, heads = _run_plain(P, H, b, m, 128, cuda_device, monkeypatch, {})
    one = torch.empty((P, b, m * P, H // P, 128), dtype=torch.bfloat16, device=cuda_device)
    uly.ulysses_seq_to_head(xs, one)
    assert torch.equal(heads.view(torch.int16), one.view(torch.int16))
