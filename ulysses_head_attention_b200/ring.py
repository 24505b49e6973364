"""Ring attention over a process group, and its composition with Ulysses (USP).

Accelerate concept guide "Sequence parallelism", "How Ulysses SP differs from
FSDP CP": ring-style context parallelism keeps each rank's sequence block and
passes key/value blocks around the ranks, combining the partial results
(blog "Ulysses Sequence Parallelism: Training with Million-Token Contexts",
"Communication complexity": O(n d) per rank over P - 1 hops, against
Ulysses' O(n d / P)); the guide's hybrid runs Ulysses over the heads inside
a group and the ring across groups, which lifts the head-count limit on the
sequence-parallel degree.

RingAttention, rank r of R, holds query, key and value rows of its sequence
block [r m, (r+1) m), m = n / R (block layout (b, m, heads, d)):

  forward   R steps; at step t it holds the key/value block of rank
            src = r - t (mod R), received from rank r - 1 while the previous
            step computed, and sends it on to rank r + 1.  Blocks with
            src <= r hold keys its queries can see: ulysses_attn_fwd_block
            gives their partial O and LSE, ulysses_attn_lse_merge combines
            them.  Blocks with src > r lie after every local query (causal)
            and are only passed on.
  backward  the key/value blocks travel again, now with their dK and dV
            accumulators (float32): at each step the rank adds the block's
            share from its own queries (ulysses_attn_bwd_block with the
            merged O and LSE) and passes block and accumulators on; after R
            steps the accumulators have visited every rank and one more hop
            takes them home.  dQ sums the key blocks' shares locally
            (ulysses_accumulate).

position_ids are the whole sequence's (b, n): sample starts are global, so
packed samples that cross block boundaries are handled exactly.

UspAttention composes the two: ranks form a U x R grid, global rank
g = rho U + u; the Ulysses group of row rho (U ranks) holds ring block rho,
rank u of it tokens [rho n/R + u n/(R U), + n/(R U)).  The forward is the
Ulysses all-to-all inside the group (distributed.seq_to_head: heads
[u H/U, (u+1) H/U) of all n/R tokens of block rho), ring attention across
the R groups' rank u, and the inverse all-to-all; the backward mirrors it.

``ops`` carries the device operations (fwd_block, bwd_block, merge,
accumulate) and ``comm`` the point-to-point exchange; the defaults call the
library and torch.distributed.  The CPU tests substitute the oracle's
key-range attention and gloo; the product path always uses the defaults.
"""
from __future__ import annotations

import torch

from . import (ulysses_accumulate, ulysses_attn_bwd_block, ulysses_attn_fwd_block, ulysses_attn_lse_merge,
               alloc_workspace, ulysses_attn_bwd_workspace, ulysses_attn_fwd_workspace, ulysses_workspace_status,
               make_shape, ULY_F32)


class LibraryOps:
    """The block kernels of the library; tensors in block layout (1, b, rows, heads, d)."""

    def __init__(self):
        self.ws = {}

    def _ws(self, kind, shape, device):
        key = (kind, shape.b, shape.n, shape.h_q, shape.h_kv, shape.d)
        if key not in self.ws:
            size = ulysses_attn_fwd_workspace(shape) if kind == "f" else ulysses_attn_bwd_workspace(shape, ULY_F32)
            self.ws[key] = alloc_workspace(size, device)
        return self.ws[key]

    def fwd_block(self, q, k, v, pos, q_base, k_base, o, lse):
        b, n = pos.shape
        shape = make_shape(b, n, q.shape[3], k.shape[3], q.shape[4], 1)
        ulysses_attn_fwd_block(q, k, v, pos, o, lse, self._ws("f", shape, q.device), q_base, k_base)

    def bwd_block(self, q, k, v, o, lse, do, pos, q_base, k_base, dq, dk, dv):
        b, n = pos.shape
        shape = make_shape(b, n, q.shape[3], k.shape[3], q.shape[4], 1)
        ulysses_attn_bwd_block(q, k, v, o, lse, do, pos, dq, dk, dv, self._ws("b", shape, q.device), q_base, k_base)

    def merge(self, o_parts, lse_parts, o, lse, h_kv):
        ulysses_attn_lse_merge(o_parts, lse_parts, o, lse, h_kv)

    def accumulate(self, dst, src):
        ulysses_accumulate(dst, src)

    def check(self):
        for ws in self.ws.values():
            if ulysses_workspace_status(ws) != 0:
                raise TimeoutError("a ring block kernel gave up waiting on its own pipeline")


class TorchComm:
    """Point-to-point exchange over a torch.distributed group (NCCL between GPUs)."""

    def __init__(self, group):
        import torch.distributed as dist
        self.dist, self.group = dist, group
        self.ranks = dist.get_process_group_ranks(group) if group is not None else list(range(dist.get_world_size()))

    def shift(self, sends, recvs, to, frm):
        """Start sending `sends` to group rank `to` and receiving `recvs` from
        group rank `frm`; returns the requests to wait on."""
        ops = [self.dist.P2POp(self.dist.isend, t, self.ranks[to], group=self.group) for t in sends]
        ops += [self.dist.P2POp(self.dist.irecv, t, self.ranks[frm], group=self.group) for t in recvs]
        return self.dist.batch_isend_irecv(ops)

    @staticmethod
    def wait(reqs):
        for rq in reqs:
            rq.wait()


class RingAttention:
    """Causal attention of this rank's sequence block against the whole
    sequence, with key/value blocks passed around the group."""

    def __init__(self, group=None, ops=None, comm=None):
        import torch.distributed as dist
        self.group = group
        self.R = dist.get_world_size(group)
        self.r = dist.get_rank(group)
        self.ops = ops if ops is not None else LibraryOps()
        self.comm = comm if comm is not None else TorchComm(group)

    def _blocks(self, m):
        R, r = self.R, self.r
        for t in range(R):
            yield t, (r - t) % R

    def forward(self, q, k, v, position_ids):
        """q (b, m, h_q, d), k / v (b, m, h_kv, d) bf16 of this rank's block;
        returns O (b, m, h_q, d) float32 and LSE (b, h_q, m) float32."""
        R, r = self.R, self.r
        b, m, hq, d = q.shape
        hkv = k.shape[2]
        if position_ids.shape[1] != m * R:
            raise ValueError("position_ids must cover the whole sequence (R blocks of m tokens)")
        q5 = q.unsqueeze(0)
        parts = r + 1                                # blocks 0..r hold visible keys
        o_parts = torch.empty((parts, 1, b, m, hq, d), dtype=torch.float32, device=q.device)
        l_parts = torch.empty((parts, 1, b, hq, m), dtype=torch.float32, device=q.device)
        # receive buffers alternate; the caller's k and v are only ever sent
        bufs = [(torch.empty_like(k), torch.empty_like(v)) for _ in range(2)]
        cur = (k.contiguous(), v.contiguous())
        filled = 0
        for t, src in self._blocks(m):
            nxt = bufs[t % 2]
            reqs = self.comm.shift(cur, nxt, (r + 1) % R, (r - 1) % R) if t + 1 < R else []
            if src <= r:
                self.ops.fwd_block(q5, cur[0].unsqueeze(0), cur[1].unsqueeze(0), position_ids, r * m, src * m,
                                   o_parts[filled], l_parts[filled])
                filled += 1
            self.comm.wait(reqs)
            cur = nxt
        o = torch.empty((1, b, m, hq, d), dtype=torch.float32, device=q.device)
        lse = torch.empty((1, b, hq, m), dtype=torch.float32, device=q.device)
        self.ops.merge(o_parts, l_parts, o, lse, hkv)
        return o[0], lse[0]

    def backward(self, q, k, v, o, lse, do, position_ids):
        """Gradients of this rank's block: dQ (b, m, h_q, d), dK and dV
        (b, m, h_kv, d), float32.  o / lse are this rank's merged forward
        results, do (b, m, h_q, d) bf16."""
        R, r = self.R, self.r
        b, m, hq, d = q.shape
        hkv = k.shape[2]
        f32 = torch.float32
        q5, o5, l5, do5 = q.unsqueeze(0), o.unsqueeze(0), lse.unsqueeze(0), do.unsqueeze(0)
        dq = torch.empty((1, b, m, hq, d), dtype=f32, device=q.device)
        share_q = torch.empty_like(dq)
        share_k = torch.empty((1, b, m, hkv, d), dtype=f32, device=q.device)
        share_v = torch.empty_like(share_k)
        # the travelling block: k, v and their gradient accumulators; receive
        # buffers alternate, the caller's k and v are only ever sent
        cur = [k.contiguous(), v.contiguous(), torch.empty((b, m, hkv, d), dtype=f32, device=q.device),
               torch.empty((b, m, hkv, d), dtype=f32, device=q.device)]
        bufs = [[torch.empty_like(x) for x in cur] for _ in range(2)]
        for t, src in self._blocks(m):
            nxt = bufs[t % 2]
            # k and v move on while this step computes; the accumulators follow
            # once they hold this step's share
            reqs = self.comm.shift(cur[:2], nxt[:2], (r + 1) % R, (r - 1) % R) if t + 1 < R else []
            if src <= r:
                if t == 0:   # the diagonal block: its shares start dQ and this block's accumulators
                    self.ops.bwd_block(q5, cur[0].unsqueeze(0), cur[1].unsqueeze(0), o5, l5, do5, position_ids,
                                       r * m, src * m, dq, cur[2].unsqueeze(0), cur[3].unsqueeze(0))
                else:
                    self.ops.bwd_block(q5, cur[0].unsqueeze(0), cur[1].unsqueeze(0), o5, l5, do5, position_ids,
                                       r * m, src * m, share_q, share_k, share_v)
                    self.ops.accumulate(dq, share_q)
                    self.ops.accumulate(cur[2].unsqueeze(0), share_k)
                    self.ops.accumulate(cur[3].unsqueeze(0), share_v)
            # pass the accumulators on (after R - 1 hops this one takes them home)
            self.comm.wait(self.comm.shift(cur[2:], nxt[2:], (r + 1) % R, (r - 1) % R))
            self.comm.wait(reqs)
            cur = nxt
        return dq[0], cur[2], cur[3]

    def check(self):
        self.ops.check()


class UspAttention:
    """Ulysses inside groups of U ranks, ring attention across the R groups."""

    def __init__(self, ulysses_group, ring_group, ops=None, comm=None, transpose=None, exchange=None):
        from . import distributed
        self.dist = distributed
        self.ug = ulysses_group
        self.ring = RingAttention(ring_group, ops, comm)
        self.kw = {}
        if transpose is not None:
            self.kw["transpose"] = transpose
        if exchange is not None:
            self.kw["exchange"] = exchange

    def forward(self, q_seq, k_seq, v_seq, position_ids):
        """This rank's token shard (b, n/(U R), H, d) of q, k, v (H_kv for k, v)
        -> O (b, n/(U R), H_q, d) float32 and the head-sharded LSE (b, H_q/U, n/R)."""
        d = self.dist
        qh = d.seq_to_head(q_seq, self.ug, **self.kw)
        kh = d.seq_to_head(k_seq, self.ug, **self.kw)
        vh = d.seq_to_head(v_seq, self.ug, **self.kw)
        o, lse = self.ring.forward(qh, kh, vh, position_ids)
        self.saved = (qh, kh, vh, o, lse)
        return d.head_to_seq(o, self.ug, **self.kw), lse

    def backward(self, do_seq, position_ids):
        """Gradients of this rank's token shard: dQ, dK, dV float32."""
        d = self.dist
        qh, kh, vh, o, lse = self.saved
        doh = d.seq_to_head(do_seq, self.ug, **self.kw)
        dq, dk, dv = self.ring.backward(qh, kh, vh, o, lse, doh, position_ids)
        return (d.head_to_seq(dq, self.ug, **self.kw), d.head_to_seq(dk, self.ug, **self.kw),
                d.head_to_seq(dv, self.ug, **self.kw))
