"""ulysses_attn_fwd_noalloc: the forward for callers that cannot allocate.

Some callers cannot hand the library a device workspace: their framework's
allocator owns all device memory and forbids raw allocations on the hot path,
or they reserved their memory once at start-up and may not allocate per
request.  For them the forward has a variant whose scratch is a fixed array
inside the library (one per GPU, b*n <= 524288 tokens).  These tests call it
through the C ABI and compare it with the workspace forward, on two calls in
a row with different shapes (the second call reuses the scratch the first one
left behind), and check that sizes beyond the fixed scratch are refused.

Kept in a file that pytest collects last, and independent of the other test
files, so it passes both alone in a fresh process and after them.
"""
import numpy as np
import pytest
import torch

import oracle
import synthetic
from gpu_util import LSE_MAX_ABS, assert_close, to_dev_bf16

pytestmark = pytest.mark.gpu

ULY_ERR_WORKSPACE = 4


def _inputs(seed, P, n, hq, hkv, d, lengths, dev):
    x = synthetic.custom_inputs(seed, 1, n, hq, hkv, d, lengths=lengths, with_do=False)
    heads = [to_dev_bf16(oracle.seq_to_head(oracle.shard(x[k], P), P), dev) for k in ("q", "k", "v")]
    return heads, torch.from_numpy(x["position_ids"]).to(dev)


def test_noalloc_matches_workspace_forward_twice(cuda_device):
    import ulysses_head_attention_b200 as uly
    cases = [  # (seed, P, n, h_q, h_kv, d, lengths): packed first, then a longer single sample
        (301, 2, 640, 4, 2, 128, [[128, 1, 127, 256, 100, 28]]),
        (302, 4, 1000, 8, 4, 128, None),
    ]
    for seed, P, n, hq, hkv, d, lengths in cases:
        (q, k, v), pos = _inputs(seed, P, n, hq, hkv, d, lengths, cuda_device)
        shape = uly.make_shape(1, n, hq, hkv, d, P)
        o_ws = torch.empty((P, 1, n, hq // P, d), dtype=torch.float32, device=cuda_device)
        l_ws = torch.empty((P, 1, hq // P, n), dtype=torch.float32, device=cuda_device)
        ws = uly.alloc_workspace(uly.ulysses_attn_fwd_workspace(shape), cuda_device)
        uly.ulysses_attn_fwd(q, k, v, pos, o_ws, l_ws, ws)
        o_na = torch.full_like(o_ws, float("nan"))
        l_na = torch.full_like(l_ws, float("nan"))
        uly.ulysses_attn_fwd_noalloc(q, k, v, pos, o_na, l_na)
        torch.cuda.synchronize()
        assert uly.ulysses_workspace_status(ws) == 0
        assert uly.ulysses_attn_fwd_noalloc_status() == 0   # the scratch's status word: no timeout
        assert_close(o_na.cpu().numpy(), o_ws.cpu().numpy(), f"noalloc O (n={n})")
        assert np.abs(l_na.cpu().numpy() - l_ws.cpu().numpy()).max() <= LSE_MAX_ABS


def test_noalloc_refuses_sizes_beyond_its_scratch(cuda_device):
    import ulysses_head_attention_b200 as uly
    # b * n = 524288 + 128 tokens: one tile more than the fixed scratch covers.
    # The buffers are real and full-sized, so nothing could run out of bounds
    # even if the check were missing.
    P, n, h, d = 1, (1 << 19) + 128, 1, 64
    q = torch.zeros((P, 1, n, h, d), dtype=torch.bfloat16, device=cuda_device)
    k, v = torch.zeros_like(q), torch.zeros_like(q)
    pos = torch.arange(n, device=cuda_device).view(1, n)
    o = torch.empty((P, 1, n, h, d), dtype=torch.float32, device=cuda_device)
    lse = torch.empty((P, 1, h, n), dtype=torch.float32, device=cuda_device)
    with pytest.raises(uly.UlyssesError) as e:
        uly.ulysses_attn_fwd_noalloc(q, k, v, pos, o, lse)
    assert e.value.status == ULY_ERR_WORKSPACE
