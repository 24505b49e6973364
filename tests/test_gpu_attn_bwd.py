"""GPU parity of the attention backward against the fp64 oracle.

The GPU forward produces O (fp32) and LSE; the GPU backward then produces
dQ, dK, dV.  The oracle's backward recomputes everything in fp64 from the
same bf16 inputs (its own O, not the GPU's).  Tolerance for fp32-stored
gradients: every element within 1e-2 of the oracle, and
sum|g-r|/sum|r| <= 2e-3; bf16-stored gradients: every element within
1e-2 + 2^-8 |ref| (one more bf16 rounding), sum|g-r|/sum|r| <= 4e-3.
"""
import numpy as np
import pytest
import torch

import oracle
import synthetic
from gpu_util import assert_close, assert_close_bf16_storage, to_dev_bf16

pytestmark = pytest.mark.gpu


def _uly():
    import ulysses_head_attention_b200 as uly
    return uly


def head_layout(bits, P):
    return oracle.seq_to_head(oracle.shard(bits, P), P)


def gpu_fwd_bwd(x, P, dev, g_dtype=torch.float32, o_dtype=torch.float32, rank=-1, sentinel=None, scale=0.0,
                outputs=None):
    uly = _uly()
    heads = [head_layout(x[k], P) for k in ("q", "k", "v", "do")]
    q, k, v, do = (to_dev_bf16(t, dev) for t in heads)
    pos = torch.from_numpy(x["position_ids"]).to(dev)
    Ps, b, n, hq, d = heads[0].shape
    hkv = heads[1].shape[3]
    shape = uly.make_shape(b, n, hq * P, hkv * P, d, P)
    o = torch.zeros((P, b, n, hq, d), dtype=o_dtype, device=dev)
    lse = torch.zeros((P, b, hq, n), dtype=torch.float32, device=dev)
    ws_f = uly.alloc_workspace(uly.ulysses_attn_fwd_workspace(shape), dev)
    uly.ulysses_attn_fwd(q, k, v, pos, o, lse, ws_f, rank=rank, softmax_scale=scale)
    code = 0 if g_dtype == torch.bfloat16 else 1
    ws_b = uly.alloc_workspace(uly.ulysses_attn_bwd_workspace(shape, code), dev)
    dq = torch.empty_like(q, dtype=g_dtype)
    dk = torch.empty_like(k, dtype=g_dtype)
    dv = torch.empty_like(v, dtype=g_dtype)
    if sentinel is not None:
        for t in (dq, dk, dv):
            t.fill_(sentinel)
    uly.ulysses_attn_bwd(q, k, v, o, lse, do, pos, dq, dk, dv, ws_b, rank=rank, softmax_scale=scale)
    assert uly.ulysses_workspace_status(ws_f) == 0
    assert uly.ulysses_workspace_status(ws_b) == 0
    if outputs is not None:   # the forward's results too
        outputs["o"], outputs["lse"] = o.float().cpu().numpy(), lse.cpu().numpy()
    return [t.float().cpu().numpy() for t in (dq, dk, dv)], heads


def oracle_bwd(heads, pos, P, rank=None, scale=None):
    qh, kh, vh, doh = (synthetic.bf16_bits_to_f64(t) for t in heads)
    return oracle.ulysses_attn_bwd(qh, kh, vh, doh, pos, P, scale=scale, rank=rank)


CASES = [
    # (id, P, b, n, h_q, h_kv, d, lengths)
    ("single_256", 2, 1, 256, 4, 2, 128, None),
    ("ragged_gqa2", 4, 1, 1000, 8, 4, 128, None),
    ("packed_tile_edges", 2, 1, 640, 4, 2, 128, [[128, 1, 127, 256, 100, 28]]),
    ("batch2_packed_d64", 2, 2, 384, 4, 2, 64, [[384], [200, 184]]),
    ("gqa_g4", 2, 1, 512, 16, 4, 128, [[300, 212]]),
    ("gqa_g8_d64", 1, 1, 520, 8, 1, 64, [[1, 1, 1, 517]]),
    ("mha_g1_odd", 1, 1, 300, 2, 2, 128, [[77, 223]]),
    ("long_2k", 2, 1, 2048, 4, 2, 128, None),
]


@pytest.mark.parametrize("case", CASES, ids=[c[0] for c in CASES])
def test_bwd_matches_oracle(cuda_device, case):
    name, P, b, n, hq, hkv, d, lengths = case
    x = synthetic.custom_inputs(200 + CASES.index(case), b, n, hq, hkv, d, lengths=lengths)
    (dq, dk, dv), heads = gpu_fwd_bwd(x, P, cuda_device)
    dq_r, dk_r, dv_r = oracle_bwd(heads, x["position_ids"], P)
    for got, ref, nm in ((dq, dq_r, "dQ"), (dk, dk_r, "dK"), (dv, dv_r, "dV")):
        assert_close(got, ref, f"bwd {name} {nm}")


def test_bwd_bf16_storage(cuda_device):
    """bf16 O in, bf16 dQ/dK/dV out (dQ through the fp32 workspace)."""
    x = synthetic.custom_inputs(230, 1, 768, 8, 2, 128, lengths=[[500, 268]])
    (dq, dk, dv), heads = gpu_fwd_bwd(x, 2, cuda_device, g_dtype=torch.bfloat16, o_dtype=torch.bfloat16)
    dq_r, dk_r, dv_r = oracle_bwd(heads, x["position_ids"], 2)
    for got, ref, nm in ((dq, dq_r, "dQ"), (dk, dk_r, "dK"), (dv, dv_r, "dV")):
        assert_close_bf16_storage(got, ref, f"bwd bf16 storage {nm}")


@pytest.mark.parametrize("do_scale", [1e-6, 1e3], ids=["tiny_dO", "large_dO"])
def test_bwd_gradient_magnitudes(cuda_device, do_scale):
    """The backward is linear in dO: gradients of dO scaled by 1e-6 (or 1e3)
    must come out scaled the same way, with the same relative accuracy.  The
    kernels' 16-bit operand copies are scaled by powers of two chosen from
    each tensor's largest magnitude, so neither tiny nor large gradients
    leave their range."""
    x = synthetic.custom_inputs(233, 1, 640, 8, 2, 128, lengths=[[128, 1, 127, 256, 100, 28]], do_scale=do_scale)
    (dq, dk, dv), heads = gpu_fwd_bwd(x, 2, cuda_device)
    dq_r, dk_r, dv_r = oracle_bwd(heads, x["position_ids"], 2)
    for got, ref, nm in ((dq, dq_r, "dQ"), (dk, dk_r, "dK"), (dv, dv_r, "dV")):
        assert_close(got / do_scale, ref / do_scale, f"bwd dO x{do_scale:g} {nm} (divided by the scale)")


@pytest.mark.parametrize("scale", [0.05, 0.2], ids=["scale_0.05", "scale_0.2"])
def test_fwd_bwd_explicit_softmax_scale(cuda_device, scale):
    """softmax_scale given explicitly (the default is 1/sqrt(d) = 0.088 at
    d = 128): the forward's O and LSE and the backward's dQ, dK, dV against
    the oracle run with the same scale, which enters the exponent, the LSE
    and the scale factor of dQ and dK."""
    x = synthetic.custom_inputs(236, 1, 640, 8, 2, 128, lengths=[[128, 1, 127, 256, 100, 28]])
    fwd = {}
    (dq, dk, dv), heads = gpu_fwd_bwd(x, 2, cuda_device, scale=scale, outputs=fwd)
    qh, kh, vh = (synthetic.bf16_bits_to_f64(t) for t in heads[:3])
    O_r, L_r = oracle.ulysses_attn_fwd(qh, kh, vh, x["position_ids"], 2, scale=scale)
    assert_close(fwd["o"], O_r, f"fwd scale {scale} O")
    assert np.abs(fwd["lse"] - L_r).max() <= 1e-3, f"fwd scale {scale} LSE"
    dq_r, dk_r, dv_r = oracle_bwd(heads, x["position_ids"], 2, scale=scale)
    for got, ref, nm in ((dq, dq_r, "dQ"), (dk, dk_r, "dK"), (dv, dv_r, "dV")):
        assert_close(got, ref, f"bwd scale {scale} {nm}")


def test_bwd_large_logits(cuda_device):
    """q and k scaled x8: scores in the hundreds, P nearly one-hot.  dQ is a
    sum of rows of k and dK one of rows of q, so both are 8x larger, and so
    are their absolute errors: their max-abs bound is 8 x 1e-2.  dV (rows of
    dO) keeps 1e-2; mean-relative stays 2e-3 for all three."""
    qk = 8.0
    x = synthetic.custom_inputs(234, 1, 768, 4, 2, 128, lengths=[[500, 268]], qk_scale=qk)
    (dq, dk, dv), heads = gpu_fwd_bwd(x, 2, cuda_device)
    dq_r, dk_r, dv_r = oracle_bwd(heads, x["position_ids"], 2)
    for got, ref, nm, bound in ((dq, dq_r, "dQ", qk * 1e-2), (dk, dk_r, "dK", qk * 1e-2), (dv, dv_r, "dV", 1e-2)):
        assert_close(got, ref, f"bwd large logits {nm}", max_abs=bound)


def test_bwd_single_rank_leaves_others_untouched(cuda_device):
    P = 4
    x = synthetic.custom_inputs(231, 1, 512, 8, 4, 128, lengths=[[256, 256]])
    rank = 1
    (dq, dk, dv), heads = gpu_fwd_bwd(x, P, cuda_device, rank=rank, sentinel=7.0)
    dq_r, dk_r, dv_r = oracle_bwd(heads, x["position_ids"], P, rank=rank)
    for got, ref, nm in ((dq[rank], dq_r[rank], "dQ"), (dk[rank], dk_r[rank], "dK"), (dv[rank], dv_r[rank], "dV")):
        assert_close(got, ref, f"bwd rank {rank} {nm}")
    others = [s for s in range(P) if s != rank]
    for t in (dq, dk, dv):
        assert (t[others] == 7.0).all()


def test_bwd_column_sums(cuda_device):
    """Properties that hold at any size: sum_j dK_j = 0 and
    sum_j dV_j = sum over the group's heads and rows of dO."""
    x = synthetic.custom_inputs(232, 1, 1024, 8, 2, 128, lengths=[[700, 324]])
    P = 2
    (dq, dk, dv), heads = gpu_fwd_bwd(x, P, cuda_device)
    do = synthetic.bf16_bits_to_f64(heads[3])
    G = 4
    for r in range(P):
        s = dk[r, 0].sum(axis=0)
        assert np.abs(s).max() <= 1e-3 * np.abs(dk[r, 0]).sum(axis=0).max()
        for g in range(dv.shape[3]):
            want = do[r, 0, :, g * G:(g + 1) * G].sum(axis=(0, 1))
            assert np.abs(dv[r, 0, :, g].sum(axis=0) - want).max() <= 1e-3 * max(1.0, np.abs(want).max())


def test_bwd_timed_matches_untimed(cuda_device):
    """The event-recording entry point computes exactly what ulysses_attn_bwd
    does, and its five events bracket four kernels in order."""
    uly = _uly()
    P = 2
    x = synthetic.custom_inputs(seed=41, b=1, n=512, h_q=4, h_kv=2, d=128, lengths=[[200, 312]], with_do=True)
    heads = [head_layout(x[k], P) for k in ("q", "k", "v", "do")]
    q, k, v, do = (to_dev_bf16(t, cuda_device) for t in heads)
    pos = torch.from_numpy(x["position_ids"]).to(cuda_device)
    shape = uly.make_shape(1, 512, 4, 2, 128, P)
    o = torch.empty((P, 1, 512, 2, 128), dtype=torch.float32, device=cuda_device)
    lse = torch.empty((P, 1, 2, 512), dtype=torch.float32, device=cuda_device)
    ws_f = uly.alloc_workspace(uly.ulysses_attn_fwd_workspace(shape), cuda_device)
    uly.ulysses_attn_fwd(q, k, v, pos, o, lse, ws_f)
    ws_b = uly.alloc_workspace(uly.ulysses_attn_bwd_workspace(shape, uly.ULY_F32), cuda_device)
    outs = []
    for timed in (False, True):
        g = [torch.empty(t.shape, dtype=torch.float32, device=cuda_device) for t in (q, k, v)]
        if timed:
            evs = [torch.cuda.Event(enable_timing=True) for _ in range(5)]
            uly.ulysses_attn_bwd_timed(q, k, v, o, lse, do, pos, *g, ws_b, evs)
            torch.cuda.synchronize()
            gaps = [evs[i].elapsed_time(evs[i + 1]) for i in range(4)]
            assert all(t >= 0.0 for t in gaps)
            assert gaps[2] > 0.0 and gaps[3] > 0.0
        else:
            uly.ulysses_attn_bwd(q, k, v, o, lse, do, pos, *g, ws_b)
        assert uly.ulysses_workspace_status(ws_b) == 0
        outs.append([t.cpu() for t in g])
    for a, b in zip(*outs):
        assert torch.equal(a, b)
