"""The CUDA pieces of the multi-process all-to-alls, on one GPU.

* ulysses_transpose_runs against numpy for run sizes that take each vector
  width (16, 8, 4, 2 bytes and single bytes) and for misaligned pointers.
* The three steps of ulysses_head_attention_b200.distributed (pack with the
  CUDA transpose, exchange, unpack) emulated for P ranks in one process: the
  exchange is a plain copy of chunk s of rank r into slot r of rank s.  The
  result must equal the one-GPU re-layout (ulysses_seq_to_head) and the
  oracle bit for bit, and the way back must return every shard.
"""
import numpy as np
import pytest
import torch

import oracle
import synthetic
from gpu_util import to_dev_bf16

pytestmark = pytest.mark.gpu


def _uly():
    import ulysses_head_attention_b200 as uly
    return uly


@pytest.mark.parametrize("A,B,run", [(7, 3, 48), (5, 4, 24), (9, 2, 12), (3, 5, 6), (4, 3, 3), (1000, 8, 256),
                                     (2, 2, 70000)])
def test_transpose_runs(cuda_device, A, B, run):
    uly = _uly()
    rng = np.random.default_rng(A * B + run)
    src = rng.integers(0, 256, A * B * run, dtype=np.uint8)
    want = src.reshape(A, B, run).transpose(1, 0, 2).reshape(-1)
    s = torch.from_numpy(src).to(cuda_device)
    d = torch.empty_like(s)
    uly.ulysses_transpose_runs(s, d, A, B, run)
    assert np.array_equal(d.cpu().numpy(), want)
    # misaligned views (one byte in)
    s2 = torch.empty(A * B * run + 1, dtype=torch.uint8, device=cuda_device)
    s2[1:].copy_(s)
    d2 = torch.empty(A * B * run + 1, dtype=torch.uint8, device=cuda_device)
    uly.ulysses_transpose_runs(s2[1:], d2[1:], A, B, run)
    assert np.array_equal(d2[1:].cpu().numpy(), want)


@pytest.mark.parametrize("P,b,n,H,d", [(4, 1, 1024, 8, 128), (2, 2, 512, 4, 64), (8, 1, 256, 32, 128)])
def test_emulated_all_to_all_equals_one_gpu_relayout(cuda_device, P, b, n, H, d):
    uly = _uly()
    m, h = n // P, H // P
    x = synthetic.f32_to_bf16_bits(np.random.default_rng(P + n).standard_normal((P, b, m, H, d), dtype=np.float32))
    xs = to_dev_bf16(x, cuda_device)
    es = 2
    # pack on every rank
    sends = [torch.empty((P, b, m, h, d), dtype=torch.bfloat16, device=cuda_device) for _ in range(P)]
    for r in range(P):
        uly.ulysses_transpose_runs(xs[r].contiguous(), sends[r], b * m, P, h * d * es)
    # exchange: chunk s of rank r goes to slot r of rank s
    recvs = [torch.empty_like(sends[0]) for _ in range(P)]
    for r in range(P):
        for s in range(P):
            recvs[s][r].copy_(sends[r][s])
    # unpack
    outs = [torch.empty((b, n, h, d), dtype=torch.bfloat16, device=cuda_device) for _ in range(P)]
    for r in range(P):
        uly.ulysses_transpose_runs(recvs[r], outs[r], P, b, m * h * d * es)
    got = torch.stack(outs)
    one_gpu = torch.empty((P, b, n, h, d), dtype=torch.bfloat16, device=cuda_device)
    uly.ulysses_seq_to_head(xs, one_gpu)
    assert torch.equal(got.view(torch.int16), one_gpu.view(torch.int16))
    assert np.array_equal(got.view(torch.int16).cpu().numpy().view(np.uint16), oracle.seq_to_head(x, P))
    # and back: (b, P, m h d) -> (P, b, m h d), exchange, (P, b m, h d) -> (b m, P, h d)
    sends2 = [torch.empty((P, b, m, h, d), dtype=torch.bfloat16, device=cuda_device) for _ in range(P)]
    for r in range(P):
        uly.ulysses_transpose_runs(outs[r], sends2[r], b, P, m * h * d * es)
    recvs2 = [torch.empty_like(sends2[0]) for _ in range(P)]
    for r in range(P):
        for s in range(P):
            recvs2[s][r].copy_(sends2[r][s])
    for r in range(P):
        back = torch.empty((b, m, H, d), dtype=torch.bfloat16, device=cuda_device)
        uly.ulysses_transpose_runs(recvs2[r], back, P, b * m, h * d * es)
        assert torch.equal(back.view(torch.int16), xs[r].view(torch.int16))
