"""The fused peer-store all-to-alls (ulysses_seq_to_head_push /
ulysses_head_to_seq_push, ulysses_wait_flags) with P ranks emulated on one GPU.

Every "peer" buffer is a slice of one device tensor, so the stores that
would cross NVLink between GPUs here stay in one GPU's memory; the index
arithmetic, the per-destination completion counting and the flag protocol
are the same.  All P pushes are enqueued on one stream before any wait, so
no kernel ever waits on another launch: every wait finds its flags set.
Checked bit for bit against the one-GPU re-layout (itself bit-exact against
the oracle) and the oracle; a wait on flags nobody sets must give up with
ULY_ERR_TIMEOUT after its limit.
"""
import numpy as np
import pytest
import torch

import oracle
from gpu_util import bits_of, to_dev_bf16

pytestmark = pytest.mark.gpu

ULY_ERR_TIMEOUT = 5


def _rand(shape, dtype, dev, seed):
    g = torch.Generator(device="cpu").manual_seed(seed)
    return torch.randn(shape, generator=g).to(dtype).to(dev)


@pytest.mark.parametrize("P,b,n,H,d,dtype", [
    (4, 1, 4096, 32, 128, torch.bfloat16),     # q-like: 8 heads per rank
    (4, 1, 4096, 8, 128, torch.bfloat16),      # k/v-like: 2 heads per rank
    (8, 2, 2048, 8, 64, torch.bfloat16),       # one 128-byte head per rank, two batch rows
    (4, 1, 1024, 32, 128, torch.float32),      # O / gradients
])
def test_push_round_trip_matches_the_one_gpu_relayout(cuda_device, P, b, n, H, d, dtype):
    import ulysses_head_attention_b200 as uly
    m, h = n // P, H // P
    x_seq = _rand((P, b, m, H, d), dtype, cuda_device, seed=P * 1000 + H)
    want = torch.empty((P, b, n, h, d), dtype=dtype, device=cuda_device)
    uly.ulysses_seq_to_head(x_seq, want)
    heads = torch.full((P, b, n, h, d), float("nan"), dtype=dtype, device=cuda_device)
    flags = torch.zeros((P, P), dtype=torch.int32, device=cuda_device)
    ws = uly.alloc_workspace(4096, cuda_device)
    epoch = 7
    for r in range(P):
        uly.ulysses_seq_to_head_push(x_seq[r], list(heads), list(flags), r, P, epoch, ws)
    st = uly.alloc_workspace(256, cuda_device)
    for s in range(P):
        uly.ulysses_wait_flags(flags[s], epoch, 1_000_000_000, st)
    assert uly.ulysses_workspace_status(st) == 0
    assert (flags == epoch).all()
    assert torch.equal(heads.view(torch.uint8), want.view(torch.uint8))
    if dtype == torch.bfloat16 and b == 1:   # and the oracle's permutation, bit for bit
        ref = oracle.seq_to_head(bits_of(x_seq).reshape(P, 1, m, H, d), P)
        assert np.array_equal(bits_of(heads), ref)

    # the way back, with the next epoch
    back = torch.full_like(x_seq, float("nan"))
    flags2 = torch.zeros((P, P), dtype=torch.int32, device=cuda_device)
    for r in range(P):
        uly.ulysses_head_to_seq_push(heads[r], list(back), list(flags2), r, P, epoch + 1, ws)
    for s in range(P):
        uly.ulysses_wait_flags(flags2[s], epoch + 1, 1_000_000_000, st)
    assert uly.ulysses_workspace_status(st) == 0
    assert torch.equal(back.view(torch.uint8), x_seq.view(torch.uint8))


def test_wait_on_flags_nobody_sets_times_out(cuda_device):
    import ulysses_head_attention_b200 as uly
    flags = torch.zeros(8, dtype=torch.int32, device=cuda_device)
    flags[:5] = 3                    # five of eight peers arrived
    st = uly.alloc_workspace(256, cuda_device)
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    start.record()
    uly.ulysses_wait_flags(flags, 3, 2_000_000, st)   # 2 ms
    end.record()
    torch.cuda.synchronize()
    assert 1.8 <= start.elapsed_time(end) <= 2000.0
    assert uly.ulysses_workspace_status(st) == ULY_ERR_TIMEOUT
    flags[5:] = 3
    uly.ulysses_wait_flags(flags, 3, 2_000_000, st)
    assert uly.ulysses_workspace_status(st) == 0


def test_ipc_handle_of_a_local_allocation(cuda_device):
    """The handle of a device allocation is 64 bytes and stable; opening it
    is for other processes (CUDA refuses it in the exporting process)."""
    import ulysses_head_attention_b200 as uly
    t = torch.empty(1 << 20, dtype=torch.uint8, device=cuda_device)
    h1, h2 = uly.ulysses_ipc_handle(t), uly.ulysses_ipc_handle(t)
    assert len(h1) == 64 and h1 == h2
