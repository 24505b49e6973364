"""The multi-process ring attention driver and its Ulysses composition
(ulysses_head_attention_b200.ring) on CPU, over gloo.

The block kernels are replaced by the oracle's key-range attention with the
same contracts (a query block against a key block, both given by their
global row offsets; partial O / LSE merged by the oracle's LSE merge; the
backward's shares from the merged O and LSE), and the accumulation by a host
add; the key/value blocks and the dK / dV accumulators travel between
processes over gloo's point-to-point sends, exactly as the product path
sends them over NCCL.  Checked against the oracle's attention of the whole
sequence, forward and backward, with packed samples that cross block
boundaries:
  * ring attention over 3 ranks;
  * Ulysses inside groups of 2 x ring across 2 groups (4 ranks), with the
    all-to-all of distributed.py (numpy transpose stand-in, gloo exchange).
The block kernels themselves are checked on the GPU (test_gpu_ring_blocks.py).
"""
import datetime
import os
import socket
import sys

import numpy as np
import pytest

from conftest import ROOT


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


class OracleBlockOps:
    """fwd_block / bwd_block / merge / accumulate contracts on host tensors (float64 math)."""

    def __init__(self, n):
        self.n = n

    def _full(self, x5, base):
        """(1, b, rows, h, d) block -> (b, n, h, d) float64 with the block at its rows."""
        x = x5[0].double().numpy()
        out = np.zeros((x.shape[0], self.n) + x.shape[2:])
        out[:, base:base + x.shape[1]] = x
        return out

    def fwd_block(self, q5, k5, v5, pos, q_base, k_base, o, lse):
        import oracle
        import torch
        m, mk = q5.shape[2], k5.shape[2]
        qf, kf, vf = self._full(q5, q_base), self._full(k5, k_base), self._full(v5, k_base)
        ss = oracle.segment_starts(pos.numpy())
        hq, hkv, d = q5.shape[3], k5.shape[3], q5.shape[4]
        G = hq // hkv
        for bb in range(q5.shape[1]):
            for h in range(hq):
                O, L = oracle.attention_fwd_head_range(qf[bb, :, h], kf[bb, :, h // G], vf[bb, :, h // G], ss[bb],
                                                       oracle.default_scale(d), k_base, k_base + mk)
                o[0, bb, :, h] = torch.from_numpy(O[q_base:q_base + m])
                lse[0, bb, h] = torch.from_numpy(L[q_base:q_base + m])

    def bwd_block(self, q5, k5, v5, o5, l5, do5, pos, q_base, k_base, dq, dk, dv):
        import oracle
        import torch
        m, mk = q5.shape[2], k5.shape[2]
        qf, kf, vf, dof, of = (self._full(x, base) for x, base in
                               ((q5, q_base), (k5, k_base), (v5, k_base), (do5, q_base), (o5, q_base)))
        ss = oracle.segment_starts(pos.numpy())
        hq, hkv, d = q5.shape[3], k5.shape[3], q5.shape[4]
        G = hq // hkv
        dk[...] = 0
        dv[...] = 0
        for bb in range(q5.shape[1]):
            for h in range(hq):
                lf = np.full(self.n, np.inf)           # rows outside the query block: P = 0
                lf[q_base:q_base + m] = l5[0, bb, h].double().numpy()
                a, b_, c = oracle.attention_bwd_head_range(qf[bb, :, h], kf[bb, :, h // G], vf[bb, :, h // G],
                                                           dof[bb, :, h], of[bb, :, h], lf, ss[bb],
                                                           oracle.default_scale(d), k_base, k_base + mk)
                dq[0, bb, :, h] = torch.from_numpy(a[q_base:q_base + m])
                dk[0, bb, :, h // G] += torch.from_numpy(b_[k_base:k_base + mk])
                dv[0, bb, :, h // G] += torch.from_numpy(c[k_base:k_base + mk])

    def merge(self, o_parts, lse_parts, o, lse, h_kv):
        import oracle
        import torch
        O, L = oracle.lse_merge(o_parts.double().numpy(), lse_parts.double().numpy())
        o[...] = torch.from_numpy(O)
        lse[...] = torch.from_numpy(L)

    def accumulate(self, dst, src):
        dst += src

    def check(self):
        pass


def _problem(n, hq, hkv, d, lengths, seed=5):
    import synthetic
    x = synthetic.custom_inputs(seed, 1, n, hq, hkv, d, lengths=[lengths])
    f = {k: synthetic.bf16_bits_to_f64(x[k]) for k in ("q", "k", "v", "do")}
    return x, f


def _reference(f, pos):
    import oracle
    O, L = oracle.attention_fwd(f["q"], f["k"], f["v"], pos)
    dQ, dK, dV = oracle.attention_bwd(f["q"], f["k"], f["v"], f["do"], pos)
    return O, L, dQ, dK, dV


def _close(a, b, tol=2e-5):
    a, b = np.asarray(a, np.float64), np.asarray(b, np.float64)
    fin = np.isfinite(b)
    return bool(np.array_equal(np.isfinite(a), fin) and np.abs(a[fin] - b[fin]).max(initial=0.0) <= tol)


def _ring_main(rank, world, port, root, out):
    sys.path.insert(0, root)
    import torch
    import torch.distributed as dist
    from ulysses_head_attention_b200 import ring
    os.environ["MASTER_ADDR"], os.environ["MASTER_PORT"] = "127.0.0.1", str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        n, hq, hkv, d = 3 * 128, 4, 2, 16
        x, f = _problem(n, hq, hkv, d, [100, 200, 84])
        pos = torch.from_numpy(x["position_ids"])
        O, L, dQ, dK, dV = _reference(f, x["position_ids"])
        m = n // world
        sl = slice(rank * m, (rank + 1) * m)
        t = {k: torch.from_numpy(f[k][:, sl]).float() for k in ("q", "k", "v", "do")}
        ra = ring.RingAttention(None, ops=OracleBlockOps(n))
        o, lse = ra.forward(t["q"], t["k"], t["v"], pos)
        dq, dk, dv = ra.backward(t["q"], t["k"], t["v"], o, lse, t["do"], pos)
        ok = {"O": _close(o, O[:, sl]), "LSE": _close(lse, L[:, :, sl]), "dQ": _close(dq, dQ[:, sl]),
              "dK": _close(dk, dK[:, sl]), "dV": _close(dv, dV[:, sl]),
              "k untouched": bool(torch.equal(t["k"], torch.from_numpy(f["k"][:, sl]).float()))}
        out.put((rank, ok))
        dist.barrier()
    finally:
        dist.destroy_process_group()


def _usp_main(rank, world, port, root, out):
    sys.path.insert(0, root)
    import torch
    import torch.distributed as dist
    from ulysses_head_attention_b200 import ring
    from test_dist_all_to_all import gloo_exchange, numpy_transpose
    os.environ["MASTER_ADDR"], os.environ["MASTER_PORT"] = "127.0.0.1", str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        U, R = 2, 2
        ugroups = [dist.new_group([rho * U + u for u in range(U)]) for rho in range(R)]
        rgroups = [dist.new_group([rho * U + u for rho in range(R)]) for u in range(U)]
        rho, u = rank // U, rank % U
        n, hq, hkv, d = 2 * 128, 4, 2, 16
        x, f = _problem(n, hq, hkv, d, [70, 150, 36], seed=9)
        pos = torch.from_numpy(x["position_ids"])
        O, L, dQ, dK, dV = _reference(f, x["position_ids"])
        s = n // (U * R)
        sl = slice(rank * s, (rank + 1) * s)   # rho n/R + u n/(U R)
        t = {k: torch.from_numpy(f[k][:, sl]).float() for k in ("q", "k", "v", "do")}
        usp = ring.UspAttention(ugroups[rho], rgroups[u], ops=OracleBlockOps(n), transpose=numpy_transpose,
                                exchange=gloo_exchange)
        o, lse = usp.forward(t["q"], t["k"], t["v"], pos)
        dq, dk, dv = usp.backward(t["do"], pos)
        hs = slice(u * hq // U, (u + 1) * hq // U)
        blk = slice(rho * n // R, (rho + 1) * n // R)
        ok = {"O": _close(o, O[:, sl]), "LSE": _close(lse, L[:, hs, blk]), "dQ": _close(dq, dQ[:, sl]),
              "dK": _close(dk, dK[:, sl]), "dV": _close(dv, dV[:, sl])}
        out.put((rank, ok))
        dist.barrier()
    finally:
        dist.destroy_process_group()


def _run(target, world):
    import torch.multiprocessing as mp
    ctx = mp.get_context("spawn")
    out = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=target, args=(r, world, port, ROOT, out)) for r in range(world)]
    for p in procs:
        p.start()
    try:
        got = sorted(out.get(timeout=240) for _ in range(world))
    finally:
        for p in procs:
            p.join(timeout=60)
            if p.is_alive():
                p.kill()
    assert all(p.exitcode == 0 for p in procs)
    return got


def test_ring_attention_three_ranks_matches_the_oracle():
    for rank, ok in _run(_ring_main, 3):
        assert all(ok.values()), (rank, ok)


def test_ulysses_times_ring_four_ranks_matches_the_oracle():
    for rank, ok in _run(_usp_main, 4):
        assert all(ok.values()), (rank, ok)
