"""ulysses_layer_step_host: one layer step from pinned host tensors to host
tensors through the C ABI, with the copies on their own streams.

Its outputs must equal, bit for bit, those of the same calls made one by one
on device tensors (the kernels are deterministic), on three consecutive
steps with different inputs (the device buffers and the ordering events are
reused), and the first step's must match the oracle's layer.
"""
import numpy as np
import pytest
import torch

import oracle
import synthetic
from gpu_util import assert_close

pytestmark = pytest.mark.gpu


def _device_step(uly, x, P, dev):
    b, n = x["position_ids"].shape
    hq, hkv, d = x["q"].shape[2], x["k"].shape[2], x["q"].shape[3]
    m = n // P
    to = lambda a: torch.from_numpy(a.reshape(P, b, m, a.shape[2], d).view(np.int16)).view(torch.bfloat16).to(dev)  # noqa: E731
    q, k, v, do = to(x["q"]), to(x["k"]), to(x["v"]), to(x["do"])
    pos = torch.from_numpy(x["position_ids"]).to(dev)
    hkv_r = hkv // P if hkv >= P else 1
    hh = {nm: torch.empty((P, b, n, t.shape[3] // P if nm in ("q", "do") else hkv_r, d), dtype=torch.bfloat16,
                          device=dev) for nm, t in (("q", q), ("k", k), ("v", v), ("do", do))}
    uly.ulysses_seq_to_head(q, hh["q"])
    uly.ulysses_kv_seq_to_head(k, hh["k"])
    uly.ulysses_kv_seq_to_head(v, hh["v"])
    shape = uly.make_shape(b, n, hq, hkv, d, P)
    o = torch.empty((P, b, n, hq // P, d), device=dev)
    lse = torch.empty((P, b, hq // P, n), device=dev)
    uly.ulysses_attn_fwd(hh["q"], hh["k"], hh["v"], pos, o, lse,
                         uly.alloc_workspace(uly.ulysses_attn_fwd_workspace(shape), dev))
    o_seq = torch.empty((P, b, m, hq, d), device=dev)
    uly.ulysses_head_to_seq(o, o_seq)
    uly.ulysses_seq_to_head(do, hh["do"])
    g = {nm: torch.empty(hh[nm].shape, device=dev) for nm in ("q", "k", "v")}
    uly.ulysses_attn_bwd(hh["q"], hh["k"], hh["v"], o, lse, hh["do"], pos, g["q"], g["k"], g["v"],
                         uly.alloc_workspace(uly.ulysses_attn_bwd_workspace(shape, uly.ULY_F32), dev))
    gs = {"q": torch.empty((P, b, m, hq, d), device=dev), "k": torch.empty((P, b, m, hkv, d), device=dev),
          "v": torch.empty((P, b, m, hkv, d), device=dev)}
    uly.ulysses_head_to_seq(g["q"], gs["q"])
    uly.ulysses_kv_head_to_seq(g["k"], gs["k"])
    uly.ulysses_kv_head_to_seq(g["v"], gs["v"])
    torch.cuda.synchronize()
    return [t.cpu() for t in (o_seq, gs["q"], gs["k"], gs["v"])]


@pytest.mark.parametrize("P,n,hq,hkv,d,lengths", [(4, 1024, 8, 4, 128, [300, 724]), (4, 512, 8, 2, 64, None)])
def test_host_step_equals_the_device_calls(cuda_device, P, n, hq, hkv, d, lengths):
    import ulysses_head_attention_b200 as uly
    b, m = 1, n // P
    step = uly.LayerStepHost(b, n, hq, hkv, d, P, cuda_device)
    for it in range(3):
        x = synthetic.custom_inputs(500 + it + P * hkv, b, n, hq, hkv, d, lengths=None if lengths is None else [lengths])
        pin = lambda a: torch.from_numpy(a.reshape(P, b, m, a.shape[2], d).view(np.int16)).view(torch.bfloat16).pin_memory()  # noqa: E731
        q, k, v, do = pin(x["q"]), pin(x["k"]), pin(x["v"]), pin(x["do"])
        pos = torch.from_numpy(x["position_ids"]).pin_memory()
        outs = [torch.empty((P, b, m, h, d), dtype=torch.float32).pin_memory() for h in (hq, hq, hkv, hkv)]
        step.step(q, k, v, do, pos, *outs)
        step.done_event().synchronize()
        assert step.status() == 0
        want = _device_step(uly, x, P, cuda_device)
        for got, ref, nm in zip(outs, want, ("O", "dQ", "dK", "dV")):
            assert torch.equal(got, ref), f"step {it} {nm}"
        if it == 0:
            qs, ks, vs, dos = (oracle.shard(synthetic.bf16_bits_to_f64(x[t]), P) for t in ("q", "k", "v", "do"))
            O_ref, _ = oracle.ulysses_layer_fwd(qs, ks, vs, x["position_ids"], P)
            assert_close(outs[0].numpy(), O_ref, f"host step (P={P}, n={n}) O")
            dq_r, dk_r, dv_r = oracle.ulysses_layer_bwd(qs, ks, vs, dos, x["position_ids"], P)
            for got, ref, nm in zip(outs[1:], (dq_r, dk_r, dv_r), ("dQ", "dK", "dV")):
                assert_close(got.numpy(), ref, f"host step (P={P}, n={n}) {nm}")
