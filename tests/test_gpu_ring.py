"""GPU parity of the ring-attention building blocks against the fp64 oracle.

* ulysses_attn_fwd_kv_range: O and LSE of every row over one key block
  (fp32 O: max-abs <= 1e-2, sum|g-r|/sum|r| <= 2e-3; LSE max-abs <= 1e-3);
  rows that see no key of the block must come back exactly O = 0,
  LSE = -inf.  Blocks are chosen to start and end inside key tiles, to
  leave whole query tiles empty, and to cover everything.
* ulysses_attn_lse_merge: the merge of a partition of the keys must give the
  full attention (same bounds as the forward tests).
* ulysses_attn_bwd_kv_range, given the merged O and LSE: each block's dQ
  share, and dK / dV that equal the full gradient on the block's keys and
  are exactly zero elsewhere; the shares add up to the full dQ (fp32,
  every element within 1e-2, sum|g-r|/sum|r| <= 2e-3).
"""
import numpy as np
import pytest
import torch

import oracle
import synthetic
from gpu_util import LSE_MAX_ABS, assert_close, to_dev_bf16

pytestmark = pytest.mark.gpu

P, N, HQ, HKV = 2, 1024, 4, 2
LENGTHS = [[300, 500, 224]]


def _uly():
    import ulysses_head_attention_b200 as uly
    return uly


def setup(dev, d=128, seed=31):
    uly = _uly()
    x = synthetic.custom_inputs(seed=seed, b=1, n=N, h_q=HQ, h_kv=HKV, d=d, lengths=LENGTHS)
    heads = {k: oracle.seq_to_head(oracle.shard(x[k], P), P) for k in ("q", "k", "v", "do")}
    t = {k: to_dev_bf16(v, dev) for k, v in heads.items()}
    f64 = {k: synthetic.bf16_bits_to_f64(v) for k, v in heads.items()}
    pos = torch.from_numpy(x["position_ids"]).to(dev)
    shape = uly.make_shape(1, N, HQ, HKV, d, P)
    ws_f = uly.alloc_workspace(uly.ulysses_attn_fwd_workspace(shape), dev)
    ws_b = uly.alloc_workspace(uly.ulysses_attn_bwd_workspace(shape, uly.ULY_F32), dev)
    return x, t, f64, pos, shape, ws_f, ws_b


def fwd_block(t, pos, ws, k_lo, k_hi, dev, d=128):
    uly = _uly()
    o = torch.full((P, 1, N, HQ // P, d), 7.0, device=dev)
    lse = torch.full((P, 1, HQ // P, N), 7.0, device=dev)
    uly.ulysses_attn_fwd_kv_range(t["q"], t["k"], t["v"], pos, o, lse, ws, k_lo, k_hi)
    assert uly.ulysses_workspace_status(ws) == 0
    return o, lse


def check_lse(got, ref):
    inf = np.isneginf(ref)
    assert np.array_equal(np.isneginf(got), inf)
    assert np.abs(got[~inf] - ref[~inf]).max(initial=0.0) <= LSE_MAX_ABS


@pytest.mark.parametrize("k_lo,k_hi", [(0, N), (0, 64), (100, 460), (250, 700), (900, N), (512, 513)])
def test_forward_block_matches_oracle(cuda_device, k_lo, k_hi):
    x, t, f64, pos, _, ws_f, _ = setup(cuda_device)
    o, lse = fwd_block(t, pos, ws_f, k_lo, k_hi, cuda_device)
    O_ref, L_ref = oracle.ulysses_attn_fwd_range(f64["q"], f64["k"], f64["v"], x["position_ids"], P, k_lo, k_hi)
    got_o, got_l = o.cpu().numpy(), lse.cpu().numpy()
    check_lse(got_l, L_ref)
    empty = np.isneginf(L_ref).transpose(0, 1, 3, 2)          # [P][b][n][h]
    assert not got_o[empty].any()
    if (~empty).any():
        assert_close(got_o[~empty], O_ref[~empty], f"O block [{k_lo},{k_hi})")


@pytest.mark.parametrize("cuts", [[0, 300, 700, N], [0, 100, 101, 640, 900, N], [0, N]])
def test_merge_of_blocks_is_full_attention(cuda_device, cuts):
    uly = _uly()
    x, t, f64, pos, _, ws_f, _ = setup(cuda_device, seed=32)
    parts = [fwd_block(t, pos, ws_f, a, b, cuda_device) for a, b in zip(cuts[:-1], cuts[1:])]
    o_parts = torch.stack([p[0] for p in parts]).contiguous()
    l_parts = torch.stack([p[1] for p in parts]).contiguous()
    o = torch.empty_like(parts[0][0])
    lse = torch.empty_like(parts[0][1])
    uly.ulysses_attn_lse_merge(o_parts, l_parts, o, lse, HKV)
    O_ref, L_ref = oracle.ulysses_attn_fwd(f64["q"], f64["k"], f64["v"], x["position_ids"], P)
    assert_close(o.cpu().numpy(), O_ref, "merged O")
    check_lse(lse.cpu().numpy(), L_ref)
    # bf16 output of the merge
    ob = torch.empty(o.shape, dtype=torch.bfloat16, device=cuda_device)
    lb = torch.empty_like(lse)
    uly.ulysses_attn_lse_merge(o_parts, l_parts, ob, lb, HKV)
    assert torch.equal(lb, lse)
    assert np.abs(ob.float().cpu().numpy() - o.cpu().numpy()).max() <= 2.0 ** -8 * np.abs(o.cpu().numpy()).max()


def test_merge_rows_without_keys(cuda_device):
    uly = _uly()
    rng = np.random.default_rng(5)
    B, d = 3, 64
    o_parts = rng.standard_normal((B, P, 1, N, HQ // P, d)).astype(np.float32)
    l_parts = rng.standard_normal((B, P, 1, HQ // P, N)).astype(np.float32)
    l_parts[:, :, :, :, :10] = -np.inf                  # rows no block saw
    l_parts[1, :, :, :, 10:20] = -np.inf                # rows one block missed
    o = torch.empty((P, 1, N, HQ // P, d), device=cuda_device)
    lse = torch.empty((P, 1, HQ // P, N), device=cuda_device)
    uly.ulysses_attn_lse_merge(torch.from_numpy(o_parts).to(cuda_device), torch.from_numpy(l_parts).to(cuda_device),
                               o, lse, HKV)
    O_ref, L_ref = oracle.lse_merge(o_parts.astype(np.float64), l_parts.astype(np.float64))
    check_lse(lse.cpu().numpy(), L_ref)
    assert np.abs(o.cpu().numpy() - O_ref).max() <= 1e-5 * max(1.0, np.abs(O_ref).max())
    assert not o.cpu().numpy()[:, :, :10].any()


@pytest.mark.parametrize("cuts", [[0, 300, 700, N], [0, 100, 101, 640, 900, N]])
def test_backward_blocks_add_up(cuda_device, cuts):
    uly = _uly()
    x, t, f64, pos, shape, ws_f, ws_b = setup(cuda_device, seed=33)
    o = torch.empty((P, 1, N, HQ // P, 128), device=cuda_device)
    lse = torch.empty((P, 1, HQ // P, N), device=cuda_device)
    uly.ulysses_attn_fwd(t["q"], t["k"], t["v"], pos, o, lse, ws_f)
    O_ref, L_ref = oracle.ulysses_attn_fwd(f64["q"], f64["k"], f64["v"], x["position_ids"], P)
    dq_full = oracle.ulysses_attn_bwd(f64["q"], f64["k"], f64["v"], f64["do"], x["position_ids"], P)[0]
    dq_sum = np.zeros_like(dq_full)
    for a, b in zip(cuts[:-1], cuts[1:]):
        g = [torch.full(t[k].shape, 5.0, device=cuda_device) for k in ("q", "k", "v")]
        uly.ulysses_attn_bwd_kv_range(t["q"], t["k"], t["v"], o, lse, t["do"], pos, *g, ws_b, a, b)
        assert uly.ulysses_workspace_status(ws_b) == 0
        refs = oracle.ulysses_attn_bwd_range(f64["q"], f64["k"], f64["v"], f64["do"], O_ref, L_ref,
                                             x["position_ids"], P, a, b)
        got = [x_.cpu().numpy() for x_ in g]
        for nm, gt, rf in zip(("dQ", "dK", "dV"), got, refs):
            assert_close(gt, rf, f"ring bwd {nm} block [{a},{b})")
        for gt in got[1:]:
            assert not gt[:, :, :a].any() and not gt[:, :, b:].any()   # keys outside the block: exactly 0
        dq_sum += got[0]
    assert_close(dq_sum, dq_full, "ring bwd sum of dQ shares")


def test_range_bounds_are_checked(cuda_device):
    uly = _uly()
    x, t, f64, pos, shape, ws_f, _ = setup(cuda_device)
    o = torch.empty((P, 1, N, HQ // P, 128), device=cuda_device)
    lse = torch.empty((P, 1, HQ // P, N), device=cuda_device)
    for lo, hi in ((-1, 10), (10, 10), (0, N + 1), (20, 5)):
        with pytest.raises(uly.UlyssesError):
            uly.ulysses_attn_fwd_kv_range(t["q"], t["k"], t["v"], pos, o, lse, ws_f, lo, hi)
