"""GPU parity of the seq<->head re-layouts: bit-exact against the oracle."""
import numpy as np
import pytest
import torch

import oracle
import synthetic
from gpu_util import bits_of, to_dev_bf16

pytestmark = pytest.mark.gpu


def _uly():
    import ulysses_head_attention_b200 as uly
    return uly


def run_both(x_seq_bits, P, dev):
    uly = _uly()
    Ps, b, m, H, d = x_seq_bits.shape
    xs = to_dev_bf16(x_seq_bits, dev)
    xh = torch.empty((P, b, m * P, H // P, d), dtype=torch.bfloat16, device=dev)
    uly.ulysses_seq_to_head(xs, xh)
    back = torch.empty_like(xs)
    uly.ulysses_head_to_seq(xh, back)
    torch.cuda.synchronize()
    return bits_of(xh), bits_of(back)


@pytest.mark.parametrize("b,n,H,d,P", [
    (1, 256, 4, 64, 2),        # tiny workload shape
    (1, 1024, 32, 128, 4),
    (1, 1024, 8, 128, 8),      # 256-byte runs
    (2, 96, 12, 64, 4),        # b > 1, 3 heads per rank (non power of two runs)
    (1, 60, 6, 5, 3),          # odd sizes: 10-byte runs, scalar path
    (3, 40, 4, 6, 2),          # 12-byte runs
    (1, 64, 16, 4, 16),        # one head per rank, 8-byte runs
    (1, 48, 2, 1, 1),          # P = 1: identity
])
def test_relayout_small_exact(cuda_device, b, n, H, d, P):
    x = synthetic.custom_inputs(21, b, n, H, H, d, with_do=False)["q"]     # [b][n][H][d]
    x_seq = oracle.shard(x, P)
    got_head, got_back = run_both(x_seq, P, cuda_device)
    assert np.array_equal(got_head, oracle.seq_to_head(x_seq, P))
    assert np.array_equal(got_back, x_seq)


def test_relayout_f32_exact(cuda_device):
    uly = _uly()
    rng = np.random.default_rng(5)
    P, b, n, H, d = 4, 2, 64, 8, 32
    x = rng.standard_normal((b, n, H, d)).astype(np.float32)
    x_seq = oracle.shard(x, P)
    xs = torch.from_numpy(x_seq).to(cuda_device)
    xh = torch.empty((P, b, n, H // P, d), dtype=torch.float32, device=cuda_device)
    uly.ulysses_seq_to_head(xs, xh)
    back = torch.empty_like(xs)
    uly.ulysses_head_to_seq(xh, back)
    assert np.array_equal(xh.cpu().numpy(), oracle.seq_to_head(x_seq, P))
    assert np.array_equal(back.cpu().numpy(), x_seq)


@pytest.mark.parametrize("name", ["llama8b_p4_n32k", "packed_sft_p8_n64k", "roundtrip_p4_n128k"])
def test_relayout_full_size_exact(cuda_device, name):
    """q, k, v of the full workloads, compared element by element."""
    w = synthetic.WORKLOADS[name]
    x = synthetic.make_inputs(w, with_do=False)
    for key in ("q", "k", "v"):
        x_seq = x[key].reshape(w.P, 1, w.n // w.P, x[key].shape[2], w.d)   # b == 1: same bytes
        got_head, got_back = run_both(x_seq, w.P, cuda_device)
        assert np.array_equal(got_head, oracle.seq_to_head(x_seq, w.P)), key
        assert np.array_equal(got_back, x_seq), key


@pytest.mark.large
def test_relayout_long_context_windows(cuda_device):
    """n = 524288: q holds 2^31 elements, so 32-bit offsets would wrap.
    Compared window by window (first, last and random token windows of every
    rank) plus the bit-exact round trip of the whole tensor."""
    uly = _uly()
    w = synthetic.WORKLOADS["long_p8_n512k"]
    P, n = w.P, w.n
    q = synthetic.normal_bf16(synthetic.streams(w.wid)["q"], (w.b, w.n, w.h_q, w.d))
    x_seq = q.reshape(P, 1, n // P, w.h_q, w.d)
    xs = to_dev_bf16(x_seq, cuda_device)
    xh = torch.empty((P, 1, n, w.h_q // P, w.d), dtype=torch.bfloat16, device=cuda_device)
    uly.ulysses_seq_to_head(xs, xh)
    rng = np.random.default_rng(7)
    for r in range(P):
        starts = [0, n - 64] + list(rng.integers(0, n - 64, 6))
        for lo in starts:
            got = bits_of(xh[r, :, lo:lo + 64])
            assert np.array_equal(got, oracle.seq_to_head_window(x_seq, P, r, int(lo), int(lo) + 64)), (r, lo)
    # seq_to_head is checked above and is a bijection, so an exact round trip
    # pins head_to_seq at these sizes too.
    back = torch.empty_like(xs)
    uly.ulysses_head_to_seq(xh, back)
    assert torch.equal(back.view(torch.int16), xs.view(torch.int16))
