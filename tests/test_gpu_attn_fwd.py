"""GPU parity of the attention forward against the fp64 oracle.

Element by element on shapes the oracle finishes in seconds (several tiles,
ragged tails, packed samples, GQA group sizes 1-8, d = 64 and 128, b = 2,
single-rank mode).  Tolerance for fp32-stored O: max-abs <= 1e-2 and
sum|g-r|/sum|r| <= 2e-3; LSE: max-abs <= 1e-3.
"""
import numpy as np
import pytest
import torch

import oracle
import synthetic
from gpu_util import (LSE_MAX_ABS, assert_close, assert_close_bf16_storage, assert_lse_close, to_dev_bf16)

pytestmark = pytest.mark.gpu


def _uly():
    import ulysses_head_attention_b200 as uly
    return uly


def head_layout(bits, P):
    """[b][n][H][d] bf16 bits -> head-sharded [P][b][n][H/P][d] bits (oracle re-layout)."""
    return oracle.seq_to_head(oracle.shard(bits, P), P)


def gpu_fwd(x, P, dev, o_dtype=torch.float32, rank=-1, sentinel=None):
    uly = _uly()
    qh, kh, vh = (head_layout(x[k], P) for k in ("q", "k", "v"))
    q, k, v = (to_dev_bf16(t, dev) for t in (qh, kh, vh))
    pos = torch.from_numpy(x["position_ids"]).to(dev)
    Ps, b, n, hq, d = qh.shape
    o = torch.empty((P, b, n, hq, d), dtype=o_dtype, device=dev)
    lse = torch.empty((P, b, hq, n), dtype=torch.float32, device=dev)
    if sentinel is not None:
        o.fill_(sentinel)
        lse.fill_(sentinel)
    shape = uly.make_shape(b, n, hq * P, kh.shape[3] * P, d, P)
    ws = uly.alloc_workspace(uly.ulysses_attn_fwd_workspace(shape), dev)
    uly.ulysses_attn_fwd(q, k, v, pos, o, lse, ws, rank=rank)
    assert uly.ulysses_workspace_status(ws) == 0
    return o.float().cpu().numpy(), lse.cpu().numpy(), (qh, kh, vh)


def oracle_fwd(heads, pos, P, rank=None):
    qh, kh, vh = (synthetic.bf16_bits_to_f64(t) for t in heads)
    return oracle.ulysses_attn_fwd(qh, kh, vh, pos, P, rank=rank)


CASES = [
    # (id, P, b, n, h_q, h_kv, d, lengths)
    ("tiny_workload", 2, 1, 256, 4, 4, 64, None),
    ("ragged_gqa2", 4, 1, 1000, 8, 4, 128, None),
    ("packed_tile_edges", 2, 1, 640, 4, 2, 128, [[128, 1, 127, 256, 100, 28]]),
    ("batch2_packed", 2, 2, 384, 4, 2, 64, [[384], [200, 184]]),
    ("mha_g1", 1, 1, 300, 2, 2, 128, None),
    ("gqa_g4", 2, 1, 512, 16, 4, 128, [[300, 212]]),
    ("gqa_g8", 1, 1, 520, 8, 1, 64, [[1, 1, 1, 517]]),
    ("many_short", 2, 1, 1024, 4, 2, 128, [[7] * 146 + [2]]),
    ("long_4k", 2, 1, 4096, 4, 2, 128, None),
]


@pytest.mark.parametrize("case", CASES, ids=[c[0] for c in CASES])
def test_fwd_matches_oracle(cuda_device, case):
    _, P, b, n, hq, hkv, d, lengths = case
    x = synthetic.custom_inputs(100 + CASES.index(case), b, n, hq, hkv, d, lengths=lengths, with_do=False)
    O, L, heads = gpu_fwd(x, P, cuda_device)
    O_ref, L_ref = oracle_fwd(heads, x["position_ids"], P)
    assert_close(O, O_ref, f"fwd {case[0]} O")
    assert_lse_close(L, L_ref, f"fwd {case[0]} LSE")


def test_fwd_bf16_output(cuda_device):
    x = synthetic.custom_inputs(31, 1, 768, 8, 2, 128, lengths=[[500, 268]], with_do=False)
    O, L, heads = gpu_fwd(x, 2, cuda_device, o_dtype=torch.bfloat16)
    O_ref, L_ref = oracle_fwd(heads, x["position_ids"], 2)
    assert_close_bf16_storage(O, O_ref, "fwd bf16 storage O")
    assert np.abs(L - L_ref).max() <= LSE_MAX_ABS


def test_fwd_single_rank_leaves_others_untouched(cuda_device):
    P = 4
    x = synthetic.custom_inputs(32, 1, 512, 8, 4, 64, lengths=[[256, 256]], with_do=False)
    for rank in (0, 2, 3):
        O, L, heads = gpu_fwd(x, P, cuda_device, rank=rank, sentinel=7.0)
        O_ref, L_ref = oracle_fwd(heads, x["position_ids"], P, rank=rank)
        assert_close(O[rank], O_ref[rank], f"fwd rank {rank} O")
        assert np.abs(L[rank] - L_ref[rank]).max() <= LSE_MAX_ABS
        others = [s for s in range(P) if s != rank]
        assert (O[others] == 7.0).all() and (L[others] == 7.0).all()


def test_fwd_large_logits_stay_finite(cuda_device):
    """q and k scaled x8 give scores in the hundreds: exercises the lazy O
    rescale and the max subtraction (v stays standard normal, so the usual
    element-wise bounds apply).  LSE is in the hundreds too: its bound is
    relative."""
    x = synthetic.custom_inputs(33, 1, 1024, 4, 2, 128, with_do=False, qk_scale=8.0)
    O, L, heads = gpu_fwd(x, 2, cuda_device)
    O_ref, L_ref = oracle_fwd(heads, x["position_ids"], 2)
    assert np.abs(L_ref).max() > 100.0
    assert_close(O, O_ref, "fwd large logits O")
    assert np.abs(L - L_ref).max() <= 1e-3 * max(1.0, np.abs(L_ref).max())


def test_fwd_is_deterministic(cuda_device):
    x = synthetic.custom_inputs(34, 1, 1024, 8, 2, 128, lengths=[[600, 424]], with_do=False)
    O1, L1, _ = gpu_fwd(x, 2, cuda_device)
    O2, L2, _ = gpu_fwd(x, 2, cuda_device)
    assert np.array_equal(O1, O2) and np.array_equal(L1, L2)
