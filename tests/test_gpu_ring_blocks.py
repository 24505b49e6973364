"""Block attention on the GPU (ulysses_attn_fwd_block / ulysses_attn_bwd_block,
ulysses_accumulate) and the ring driver running on it.

1. The block kernels directly: every (query block, key block) pair of a
   sequence cut into R blocks of 128-multiple rows, merged with
   ulysses_attn_lse_merge and summed with ulysses_accumulate, against the
   oracle's attention of the whole sequence (fp32 outputs; every element
   within 1e-2, sum|g-r|/sum|r| <= 2e-3; LSE within 1e-3), packed samples
   crossing block edges, GQA, a ragged last block.
2. ring.RingAttention with the library's block kernels, R ranks emulated by
   R host threads on one GPU, each on its own stream; the point-to-point
   sends become copies through a mailbox with a host barrier between the
   ranks (no kernel waits on another launch).
3. Block offsets that are not tile multiples are refused.
"""
import threading

import numpy as np
import pytest
import torch

import oracle
import synthetic
from gpu_util import assert_close, assert_lse_close, to_dev_bf16

pytestmark = pytest.mark.gpu


def _problem(n, hq, hkv, d, lengths, seed):
    x = synthetic.custom_inputs(seed, 1, n, hq, hkv, d, lengths=[lengths])
    f = {k: synthetic.bf16_bits_to_f64(x[k]) for k in ("q", "k", "v", "do")}
    O, L = oracle.attention_fwd(f["q"], f["k"], f["v"], x["position_ids"])
    dQ, dK, dV = oracle.attention_bwd(f["q"], f["k"], f["v"], f["do"], x["position_ids"])
    return x, (O, L, dQ, dK, dV)


def _blk(bits, lo, hi, dev):
    """rows [lo, hi) of (1, n, h, d) bf16 bits -> (1, 1, hi - lo, h, d) device tensor."""
    return to_dev_bf16(np.ascontiguousarray(bits[:, lo:hi])[None], dev)


@pytest.mark.parametrize("cuts,hq,hkv,d,lengths", [
    ([0, 256, 512, 768], 4, 2, 128, [300, 1, 250, 217]),
    ([0, 128, 512, 700], 8, 2, 64, [128, 400, 172]),       # uneven blocks, ragged last one
])
def test_block_kernels_cover_the_sequence(cuda_device, cuts, hq, hkv, d, lengths):
    import ulysses_head_attention_b200 as uly
    dev = cuda_device
    n = cuts[-1]
    x, (O, L, dQ, dK, dV) = _problem(n, hq, hkv, d, lengths, seed=71 + hq)
    pos = torch.from_numpy(x["position_ids"]).to(dev)
    shape = uly.make_shape(1, n, hq, hkv, d, 1)
    wf = uly.alloc_workspace(uly.ulysses_attn_fwd_workspace(shape), dev)
    wb = uly.alloc_workspace(uly.ulysses_attn_bwd_workspace(shape, uly.ULY_F32), dev)
    R = len(cuts) - 1
    blocks = [(cuts[i], cuts[i + 1]) for i in range(R)]
    dk_acc = {j: torch.zeros((1, 1, hi - lo, hkv, d), device=dev) for j, (lo, hi) in enumerate(blocks)}
    dv_acc = {j: torch.zeros((1, 1, hi - lo, hkv, d), device=dev) for j, (lo, hi) in enumerate(blocks)}
    for i, (qlo, qhi) in enumerate(blocks):
        q, do = _blk(x["q"], qlo, qhi, dev), _blk(x["do"], qlo, qhi, dev)
        m = qhi - qlo
        parts = i + 1
        o_parts = torch.empty((parts, 1, 1, m, hq, d), device=dev)
        l_parts = torch.empty((parts, 1, 1, hq, m), device=dev)
        for j in range(parts):
            klo, khi = blocks[j]
            uly.ulysses_attn_fwd_block(q, _blk(x["k"], klo, khi, dev), _blk(x["v"], klo, khi, dev), pos,
                                       o_parts[j], l_parts[j], wf, qlo, klo)
        o = torch.empty((1, 1, m, hq, d), device=dev)
        lse = torch.empty((1, 1, hq, m), device=dev)
        uly.ulysses_attn_lse_merge(o_parts, l_parts, o, lse, hkv)
        assert uly.ulysses_workspace_status(wf) == 0
        assert_close(o[0, 0].cpu().numpy(), O[0, qlo:qhi], f"block fwd rows [{qlo},{qhi}) O")
        assert_lse_close(lse[0, 0].cpu().numpy(), L[0, :, qlo:qhi], f"block fwd rows [{qlo},{qhi}) LSE")
        dq = torch.zeros((1, 1, m, hq, d), device=dev)
        sq = torch.empty_like(dq)
        for j in range(parts):
            klo, khi = blocks[j]
            sk = torch.empty_like(dk_acc[j])
            sv = torch.empty_like(dv_acc[j])
            uly.ulysses_attn_bwd_block(q, _blk(x["k"], klo, khi, dev), _blk(x["v"], klo, khi, dev), o, lse, do, pos,
                                       sq, sk, sv, wb, qlo, klo)
            uly.ulysses_accumulate(dq, sq)
            uly.ulysses_accumulate(dk_acc[j], sk)
            uly.ulysses_accumulate(dv_acc[j], sv)
        assert uly.ulysses_workspace_status(wb) == 0
        assert_close(dq[0, 0].cpu().numpy(), dQ[0, qlo:qhi], f"block bwd rows [{qlo},{qhi}) dQ")
    for j, (lo, hi) in enumerate(blocks):
        assert_close(dk_acc[j][0, 0].cpu().numpy(), dK[0, lo:hi], f"block bwd keys [{lo},{hi}) dK")
        assert_close(dv_acc[j][0, 0].cpu().numpy(), dV[0, lo:hi], f"block bwd keys [{lo},{hi}) dV")


class _ThreadComm:
    """The point-to-point shift of R ranks emulated by R host threads: each
    rank's sends go through a mailbox, a barrier separates writing from
    reading.  Every rank finishes its own GPU work before the barrier."""

    def __init__(self, R, mail, barrier, rank):
        self.R, self.mail, self.barrier, self.rank = R, mail, barrier, rank

    def shift(self, sends, recvs, to, frm):
        torch.cuda.current_stream().synchronize()
        self.mail[(self.rank, to)] = [t.clone() for t in sends]
        torch.cuda.current_stream().synchronize()
        self.barrier.wait()
        for dst, src in zip(recvs, self.mail[(frm, self.rank)]):
            dst.copy_(src)
        torch.cuda.current_stream().synchronize()
        self.barrier.wait()
        return []

    def wait(self, reqs):
        pass


def test_ring_driver_with_emulated_ranks(cuda_device, monkeypatch):
    import torch.distributed as dist
    from ulysses_head_attention_b200 import ring
    dev = cuda_device
    R, m, hq, hkv, d = 3, 256, 4, 2, 128
    n = R * m
    x, (O, L, dQ, dK, dV) = _problem(n, hq, hkv, d, [200, 300, 268], seed=91)
    mail, barrier = {}, threading.Barrier(R)
    results, errors = {}, []

    def rank_main(r):
        try:
            torch.cuda.set_device(dev)
            with torch.cuda.stream(torch.cuda.Stream()):
                ra = ring.RingAttention.__new__(ring.RingAttention)
                ra.group, ra.R, ra.r = None, R, r
                ra.ops, ra.comm = ring.LibraryOps(), _ThreadComm(R, mail, barrier, r)
                pos = torch.from_numpy(x["position_ids"]).to(dev)
                t = {k: _blk(x[k], r * m, (r + 1) * m, dev)[0] for k in ("q", "k", "v", "do")}
                o, lse = ra.forward(t["q"], t["k"], t["v"], pos)
                dq, dk, dv = ra.backward(t["q"], t["k"], t["v"], o, lse, t["do"], pos)
                torch.cuda.current_stream().synchronize()
                ra.check()
                results[r] = [a.cpu().numpy() for a in (o, lse, dq, dk, dv)]
        except Exception as e:   # reported below; a failing rank must not leave the others at the barrier
            errors.append((r, repr(e)))
            barrier.abort()

    threads = [threading.Thread(target=rank_main, args=(r,)) for r in range(R)]
    for th in threads:
        th.start()
    for th in threads:
        th.join(timeout=300)
    assert not errors, errors
    for r in range(R):
        sl = slice(r * m, (r + 1) * m)
        o, lse, dq, dk, dv = results[r]
        assert_close(o[0], O[0, sl], f"ring driver rank {r} O")
        assert_lse_close(lse[0], L[0, :, sl], f"ring driver rank {r} LSE")
        assert_close(dq[0], dQ[0, sl], f"ring driver rank {r} dQ")
        assert_close(dk[0], dK[0, sl], f"ring driver rank {r} dK")
        assert_close(dv[0], dV[0, sl], f"ring driver rank {r} dV")


def test_block_offsets_must_be_tile_multiples(cuda_device):
    import ulysses_head_attention_b200 as uly
    dev = cuda_device
    n, hq, hkv, d = 512, 2, 1, 64
    pos = torch.arange(n, device=dev).view(1, n)
    q = torch.zeros((1, 1, 128, hq, d), dtype=torch.bfloat16, device=dev)
    k, v = torch.zeros((1, 1, 128, hkv, d), dtype=torch.bfloat16, device=dev), torch.zeros((1, 1, 128, hkv, d), dtype=torch.bfloat16, device=dev)
    o = torch.empty((1, 1, 128, hq, d), device=dev)
    lse = torch.empty((1, 1, hq, 128), device=dev)
    ws = uly.alloc_workspace(uly.ulysses_attn_fwd_workspace(uly.make_shape(1, n, hq, hkv, d, 1)), dev)
    for qb, kb in ((64, 0), (0, 100), (448, 0), (0, 448)):   # off a tile edge, or past the sequence's end
        with pytest.raises(uly.UlyssesError):
            uly.ulysses_attn_fwd_block(q, k, v, pos, o, lse, ws, qb, kb)
