"""GPU parity of the kv-head replication path (H_kv < P) against the oracle.

* ulysses_kv_seq_to_head: bit-exact copies (and, for H_kv a multiple of P,
  byte-identical to ulysses_seq_to_head).
* ulysses_kv_head_to_seq: the sum of the copies, float32 accumulation in a
  fixed order: within float32 rounding of the fp64 sum for fp32 data, within
  one bf16 rounding for bf16 data.
* The whole layer with H_kv < P (re-layouts, forward, backward, the reducing
  re-layout of dK and dV) against the oracle's layer, with the tolerances of
  the other attention tests: fp32 outputs, every element within 1e-2,
  sum|g-r|/sum|r| <= 2e-3.
"""
import numpy as np
import pytest
import torch

import oracle
import synthetic
from gpu_util import assert_close, to_dev_bf16

pytestmark = pytest.mark.gpu


def _uly():
    import ulysses_head_attention_b200 as uly
    return uly


def bits(t):
    return t.view(torch.int16).cpu().numpy().view(np.uint16)


@pytest.mark.parametrize("P,H,b,n,d", [(8, 2, 2, 1024, 128), (4, 1, 1, 512, 64), (16, 8, 1, 4096, 128),
                                       (6, 3, 1, 96, 64)])
def test_replicate_is_exact(cuda_device, P, H, b, n, d):
    uly = _uly()
    rng = np.random.default_rng(P * 100 + H)
    x = synthetic.f32_to_bf16_bits(rng.standard_normal((P, b, n // P, H, d), dtype=np.float32))
    xs = to_dev_bf16(x, cuda_device)
    xh = torch.empty((P, b, n, 1, d), dtype=torch.bfloat16, device=cuda_device)
    uly.ulysses_kv_seq_to_head(xs, xh)
    assert np.array_equal(bits(xh), oracle.kv_seq_to_head(x, P))
    # fp32 copies too
    xf = torch.from_numpy(rng.standard_normal((P, b, n // P, H, d)).astype(np.float32)).to(cuda_device)
    xhf = torch.empty((P, b, n, 1, d), dtype=torch.float32, device=cuda_device)
    uly.ulysses_kv_seq_to_head(xf, xhf)
    assert np.array_equal(xhf.cpu().numpy(), oracle.kv_seq_to_head(xf.cpu().numpy(), P))


def test_divisible_case_is_the_plain_relayout(cuda_device):
    uly = _uly()
    P, b, n, H, d = 4, 1, 512, 8, 128
    x = to_dev_bf16(synthetic.f32_to_bf16_bits(np.random.default_rng(3).standard_normal(
        (P, b, n // P, H, d), dtype=np.float32)), cuda_device)
    a = torch.empty((P, b, n, H // P, d), dtype=torch.bfloat16, device=cuda_device)
    c = torch.empty_like(a)
    uly.ulysses_kv_seq_to_head(x, a)
    uly.ulysses_seq_to_head(x, c)
    assert torch.equal(a.view(torch.int16), c.view(torch.int16))
    back = torch.empty_like(x)
    uly.ulysses_kv_head_to_seq(a, back)
    assert torch.equal(back.view(torch.int16), x.view(torch.int16))


@pytest.mark.parametrize("P,H,b,n,d", [(8, 2, 2, 1024, 128), (16, 8, 1, 4096, 128), (4, 1, 1, 512, 64),
                                       (6, 3, 1, 96, 64)])
def test_reduce_sums_the_copies(cuda_device, P, H, b, n, d):
    uly = _uly()
    rng = np.random.default_rng(P * 7 + H)
    y = rng.standard_normal((P, b, n, 1, d)).astype(np.float32)
    ref = oracle.kv_head_to_seq_reduce(y.astype(np.float64), P, H)
    absum = oracle.kv_head_to_seq_reduce(np.abs(y).astype(np.float64), P, H)
    out = torch.empty((P, b, n // P, H, d), dtype=torch.float32, device=cuda_device)
    uly.ulysses_kv_head_to_seq(torch.from_numpy(y).to(cuda_device), out)
    got = out.cpu().numpy()
    R = P // H
    assert np.all(np.abs(got - ref) <= R * 2.0 ** -24 * absum + 1e-30)
    # bf16 data: float32 sums of the bf16 values, rounded once (round to nearest even)
    yb = synthetic.f32_to_bf16_bits(y)
    refb = oracle.kv_head_to_seq_reduce(synthetic.bf16_bits_to_f64(yb), P, H)
    outb = torch.empty((P, b, n // P, H, d), dtype=torch.bfloat16, device=cuda_device)
    uly.ulysses_kv_head_to_seq(to_dev_bf16(yb, cuda_device), outb)
    gotb = outb.float().cpu().numpy()
    absb = oracle.kv_head_to_seq_reduce(np.abs(synthetic.bf16_bits_to_f64(yb)), P, H)
    assert np.all(np.abs(gotb - refb) <= 2.0 ** -8 * np.abs(refb) + R * 2.0 ** -24 * absb + 1e-30)
    # deterministic
    out2 = torch.empty_like(out)
    uly.ulysses_kv_head_to_seq(torch.from_numpy(y).to(cuda_device), out2)
    assert torch.equal(out, out2)


@pytest.mark.parametrize("P,hq,hkv,n,lengths", [
    (8, 16, 2, 2048, [[700, 1348]]),
    (4, 8, 1, 1024, [[1024]]),
    (16, 32, 8, 2048, [[512, 1000, 536]]),
])
def test_layer_with_replication_matches_oracle(cuda_device, P, hq, hkv, n, lengths):
    uly = _uly()
    d = 128
    x = synthetic.custom_inputs(seed=60 + P, b=1, n=n, h_q=hq, h_kv=hkv, d=d, lengths=lengths)
    m = n // P
    seq = {k: to_dev_bf16(oracle.shard(x[k], P), cuda_device) for k in ("q", "k", "v", "do")}
    qh = torch.empty((P, 1, n, hq // P, d), dtype=torch.bfloat16, device=cuda_device)
    doh = torch.empty_like(qh)
    kh = torch.empty((P, 1, n, 1, d), dtype=torch.bfloat16, device=cuda_device)
    vh = torch.empty_like(kh)
    uly.ulysses_seq_to_head(seq["q"], qh)
    uly.ulysses_seq_to_head(seq["do"], doh)
    uly.ulysses_kv_seq_to_head(seq["k"], kh)
    uly.ulysses_kv_seq_to_head(seq["v"], vh)
    pos = torch.from_numpy(x["position_ids"]).to(cuda_device)
    shape = uly.make_shape(1, n, hq, hkv, d, P)
    o = torch.empty((P, 1, n, hq // P, d), dtype=torch.float32, device=cuda_device)
    lse = torch.empty((P, 1, hq // P, n), dtype=torch.float32, device=cuda_device)
    ws_f = uly.alloc_workspace(uly.ulysses_attn_fwd_workspace(shape), cuda_device)
    uly.ulysses_attn_fwd(qh, kh, vh, pos, o, lse, ws_f)
    ws_b = uly.alloc_workspace(uly.ulysses_attn_bwd_workspace(shape, uly.ULY_F32), cuda_device)
    dqh = torch.empty(qh.shape, dtype=torch.float32, device=cuda_device)
    dkh = torch.empty(kh.shape, dtype=torch.float32, device=cuda_device)
    dvh = torch.empty(vh.shape, dtype=torch.float32, device=cuda_device)
    uly.ulysses_attn_bwd(qh, kh, vh, o, lse, doh, pos, dqh, dkh, dvh, ws_b)
    assert uly.ulysses_workspace_status(ws_f) == 0 and uly.ulysses_workspace_status(ws_b) == 0
    o_seq = torch.empty((P, 1, m, hq, d), dtype=torch.float32, device=cuda_device)
    uly.ulysses_head_to_seq(o, o_seq)
    g = {}
    for nm, t, H in (("dq", dqh, hq), ("dk", dkh, hkv), ("dv", dvh, hkv)):
        g[nm] = torch.empty((P, 1, m, H, d), dtype=torch.float32, device=cuda_device)
        (uly.ulysses_head_to_seq if nm == "dq" else uly.ulysses_kv_head_to_seq)(t, g[nm])

    f64 = {k: oracle.shard(synthetic.bf16_bits_to_f64(x[k]), P) for k in ("q", "k", "v", "do")}
    O_ref, _ = oracle.ulysses_layer_fwd(f64["q"], f64["k"], f64["v"], x["position_ids"], P)
    refs = oracle.ulysses_layer_bwd(f64["q"], f64["k"], f64["v"], f64["do"], x["position_ids"], P)
    assert_close(o_seq.cpu().numpy(), O_ref, "O")
    for nm, ref in zip(("dq", "dk", "dv"), refs):
        assert_close(g[nm].cpu().numpy(), ref, f"kv replication {nm}")
