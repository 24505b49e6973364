"""The bounded-wait failure path on a GPU, without a fault.

Every pipeline wait in the attention kernels is bounded in time: when one
runs out, the kernel raises its CTA abort flag and the workspace status word,
lets its copies in flight land, frees TMEM and returns.  On valid input no
wait ever runs out, so ulysses_selftest_wait_timeout runs that sequence on
purpose: one CTA waits on a barrier nothing arrives at.  The test checks
that the call returns within a bounded time, that the status word reads
ULY_ERR_TIMEOUT once and is then cleared, and that the context stays usable:
a normal forward right after it matches the oracle.
"""
import numpy as np
import pytest
import torch

import oracle
import synthetic
from gpu_util import assert_close, assert_lse_close, to_dev_bf16

pytestmark = pytest.mark.gpu

ULY_ERR_TIMEOUT = 5


@pytest.mark.parametrize("limit_ms", [1.0, 100.0])
def test_wait_runs_out_and_the_context_stays_usable(cuda_device, limit_ms):
    import ulysses_head_attention_b200 as uly
    ws = uly.alloc_workspace(4096, cuda_device)
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    start.record()
    uly.ulysses_selftest_wait_timeout(ws, int(limit_ms * 1e6))
    end.record()
    torch.cuda.synchronize()
    ms = start.elapsed_time(end)
    assert limit_ms * 0.9 <= ms <= limit_ms + 2000.0, ms   # gave up after the limit, and did return
    assert uly.ulysses_workspace_status(ws) == ULY_ERR_TIMEOUT
    assert uly.ulysses_workspace_status(ws) == 0            # read once, then cleared

    # a normal forward on the same stream and context
    P, n, hq, hkv, d = 2, 512, 4, 2, 128
    x = synthetic.custom_inputs(61, 1, n, hq, hkv, d, lengths=[[300, 212]], with_do=False)
    heads = [oracle.seq_to_head(oracle.shard(x[k], P), P) for k in ("q", "k", "v")]
    q, k, v = (to_dev_bf16(t, cuda_device) for t in heads)
    pos = torch.from_numpy(x["position_ids"]).to(cuda_device)
    o = torch.empty((P, 1, n, hq // P, d), dtype=torch.float32, device=cuda_device)
    lse = torch.empty((P, 1, hq // P, n), dtype=torch.float32, device=cuda_device)
    shape = uly.make_shape(1, n, hq, hkv, d, P)
    wf = uly.alloc_workspace(uly.ulysses_attn_fwd_workspace(shape), cuda_device)
    uly.ulysses_attn_fwd(q, k, v, pos, o, lse, wf)
    assert uly.ulysses_workspace_status(wf) == 0
    O_ref, L_ref = oracle.ulysses_attn_fwd(*(synthetic.bf16_bits_to_f64(t) for t in heads), x["position_ids"], P)
    assert_close(o.cpu().numpy(), O_ref, "forward after a timed-out wait O")
    assert_lse_close(lse.cpu().numpy(), L_ref, "forward after a timed-out wait LSE")
