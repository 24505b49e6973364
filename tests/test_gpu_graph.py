"""A whole layer step (seq->head, forward, head->seq, and the backward with
its re-layouts) issued eagerly twice, then captured once as a CUDA graph and
replayed: every output of every run must be the same bits.

The attention kernels use no atomics and fix every reduction order, so the
library documents its results as bitwise reproducible from call to call; and
no call in a step synchronises with the host or allocates, so a step can be
captured as it runs.  The workspaces' status words must stay clear.
"""
import numpy as np
import pytest
import torch

import synthetic

pytestmark = pytest.mark.gpu


class _Step:
    """Device buffers of one layer step and the calls that fill them."""

    def __init__(self, uly, x, P, dev):
        b, n = x["position_ids"].shape
        hq, hkv, d = x["q"].shape[2], x["k"].shape[2], x["q"].shape[3]
        m = n // P
        self.uly = uly
        to = lambda a: torch.from_numpy(a.reshape(P, b, m, a.shape[2], d).view(np.int16)).view(torch.bfloat16).to(dev)  # noqa: E731
        self.seq = {k: to(x[k]) for k in ("q", "k", "v", "do")}
        self.pos = torch.from_numpy(x["position_ids"]).to(dev)
        hkv_r = hkv // P if hkv >= P else 1
        self.head = {k: torch.empty((P, b, n, hq // P if k in ("q", "do") else hkv_r, d), dtype=torch.bfloat16,
                                    device=dev) for k in ("q", "k", "v", "do")}
        shape = uly.make_shape(b, n, hq, hkv, d, P)
        self.ws_f = uly.alloc_workspace(uly.ulysses_attn_fwd_workspace(shape), dev)
        self.ws_b = uly.alloc_workspace(uly.ulysses_attn_bwd_workspace(shape, uly.ULY_F32), dev)
        self.o = torch.empty((P, b, n, hq // P, d), device=dev)
        self.lse = torch.empty((P, b, hq // P, n), device=dev)
        self.o_seq = torch.empty((P, b, m, hq, d), device=dev)
        self.g = {k: torch.empty(self.head[k].shape, device=dev) for k in ("q", "k", "v")}
        self.g_seq = {"q": torch.empty((P, b, m, hq, d), device=dev), "k": torch.empty((P, b, m, hkv, d), device=dev),
                      "v": torch.empty((P, b, m, hkv, d), device=dev)}

    def run(self):
        u, h, s = self.uly, self.head, self.seq
        u.ulysses_seq_to_head(s["q"], h["q"])
        u.ulysses_kv_seq_to_head(s["k"], h["k"])
        u.ulysses_kv_seq_to_head(s["v"], h["v"])
        u.ulysses_attn_fwd(h["q"], h["k"], h["v"], self.pos, self.o, self.lse, self.ws_f)
        u.ulysses_head_to_seq(self.o, self.o_seq)
        u.ulysses_seq_to_head(s["do"], h["do"])
        u.ulysses_attn_bwd(h["q"], h["k"], h["v"], self.o, self.lse, h["do"], self.pos,
                           self.g["q"], self.g["k"], self.g["v"], self.ws_b)
        u.ulysses_head_to_seq(self.g["q"], self.g_seq["q"])
        u.ulysses_kv_head_to_seq(self.g["k"], self.g_seq["k"])
        u.ulysses_kv_head_to_seq(self.g["v"], self.g_seq["v"])

    def outputs(self):
        torch.cuda.synchronize()
        return [t.cpu().numpy().copy() for t in (self.o_seq, self.lse, self.g_seq["q"], self.g_seq["k"],
                                                 self.g_seq["v"])]

    def clear(self):
        for t in (self.o_seq, self.lse, *self.g_seq.values()):
            t.fill_(float("nan"))


@pytest.mark.parametrize("P,n,hq,hkv,d,lengths", [(4, 1024, 8, 4, 128, [300, 1, 723]), (2, 768, 4, 4, 64, None)])
def test_step_is_bitwise_reproducible_and_replays_as_a_graph(cuda_device, P, n, hq, hkv, d, lengths):
    import ulysses_head_attention_b200 as uly
    x = synthetic.custom_inputs(700 + P + d, 1, n, hq, hkv, d, lengths=None if lengths is None else [lengths])
    st = _Step(uly, x, P, cuda_device)
    st.run()
    first = st.outputs()
    assert all(np.isfinite(a).all() for a in first)
    st.clear()
    st.run()
    second = st.outputs()
    for nm, a, b in zip(("O", "LSE", "dQ", "dK", "dV"), first, second):
        assert np.array_equal(a.view(np.uint32), b.view(np.uint32)), f"{nm} differs between two eager runs"
    # capture on a side stream after a warm-up there, as CUDA graphs require
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        st.run()
    torch.cuda.current_stream().wait_stream(side)
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        st.run()
    for _ in range(2):
        st.clear()
        graph.replay()
        replayed = st.outputs()
        for nm, a, b in zip(("O", "LSE", "dQ", "dK", "dV"), first, replayed):
            assert np.array_equal(a.view(np.uint32), b.view(np.uint32)), f"{nm} differs under graph replay"
    del graph
    assert uly.ulysses_workspace_status(st.ws_f) == 0
    assert uly.ulysses_workspace_status(st.ws_b) == 0
