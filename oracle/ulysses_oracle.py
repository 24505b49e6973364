"""Plain float64 CPU oracle of Ulysses sequence parallelism's hot path.

TEST INFRASTRUCTURE ONLY (see the package docstring for who may call it).

What is computed, step by step, and where the pages define it:

  1. Sequence sharding -- [BLOG] "How Ulysses works", step 1: with P ranks,
     rank i holds tokens [i*n/P, (i+1)*n/P) with every head.
  2. seq->head re-layout (the first all-to-all) -- [BLOG] step 3 and the
     [TF-ALST] figure: afterwards every rank holds all n positions for its
     H/P heads.
  3. Local attention per head -- [BLOG] step 4 ("standard attention", i.e.
     softmax(scale * q k^T) v), with causality and sample boundaries taken
     from position_ids ([BLOG], position_ids paragraph under "Loss
     aggregation"; [ACC-SP] "ALST/Ulysses SP backend configuration":
     concatenated samples must not attend to one another).
  4. head->seq re-layout (the second all-to-all) -- [BLOG] step 5.
  5. Backward: the gradient of the attention with respect to q, k, v
     (training through the layer, [ACC-SP] custom training loop); the
     gradient of a re-layout is the inverse re-layout.
  6. Attention over one block of keys, and the LSE merge of such blocks --
     [ACC-SP] "How Ulysses SP differs from FSDP CP" and [BLOG] on ring
     attention: the sequence is sharded, KV blocks travel between ranks, and
     each rank combines the partial results of the blocks it saw.  A block's
     partial result is (O_b, LSE_b) over the visible keys of the block; the
     merge is LSE = log sum_b exp(LSE_b), O = sum_b exp(LSE_b - LSE) O_b.
     The backward of a block, given the merged O and LSE, is that block's
     share of dQ and the full dK, dV of its keys.
  7. Weighted loss aggregation across the SP ranks -- [ACC-SP] custom
     training loop (each rank's loss weighted by its count of labels other
     than -100; ranks without such labels skipped; divided by
     max(total count, 1)) and [BLOG] "Loss aggregation".

Readings taken where the pages are silent (each pinned by a test):
  * softmax scale = 1/sqrt(d) unless given ("standard attention");
  * a new sample starts at t == 0 and wherever position_ids[t] == 0; inside a
    sample, causality is by token index: key j is visible to query i iff
    j <= i and both lie in the same sample;
  * GQA: query head h reads kv head h // G (G = H_q / H_kv); ranks split both
    H_q and H_kv contiguously, so a rank's query heads map onto its own kv
    heads;
  * after the first all-to-all, rank j's chunk lands at positions
    [j*n/P, (j+1)*n/P), and a rank's heads keep ascending global order;
  * LSE is the natural-log log-sum-exp of the scaled scores, per row.
  * H_kv < P (GQA with fewer kv heads than ranks; the pages are silent): when
    P is a multiple of H_kv, every rank r receives a copy of the one kv head
    its query heads read, g(r) = r * H_kv // P; the gradient of that copy is
    the sum over the ranks that hold it.
  * loss aggregation: the gradient returned is the derivative of the
    aggregated loss with respect to each rank's loss (good_r / max(G, 1) for
    a rank with good tokens, 0 for one without); how a framework then scales
    gradients across ranks is outside the path.

Arrays: unsharded tensors are [b][n][H][d]; seq-sharded [P][b][n/P][H][d];
head-sharded [P][b][n][H/P][d]; LSE of head-sharded attention [P][b][H_q/P][n].
All arithmetic is float64.
"""
from __future__ import annotations

import math
from typing import Optional, Sequence, Tuple

import numpy as np

__all__ = [
    "check_shape", "valid_sp_sizes",
    "shard", "unshard", "seq_to_head", "head_to_seq", "seq_to_head_window", "head_to_seq_window",
    "kv_rank_head", "kv_seq_to_head", "kv_head_to_seq_reduce",
    "segment_ids", "segment_starts", "segment_ends", "allowed_matrix",
    "attention_brute_head", "attention_bwd_brute_head",
    "attention_fwd_head", "attention_bwd_head",
    "attention_fwd_rows", "attention_bwd_rows",
    "attention_fwd", "attention_bwd",
    "ulysses_attn_fwd", "ulysses_attn_bwd",
    "ulysses_layer_fwd", "ulysses_layer_bwd",
    "default_scale",
    "sp_good_tokens", "sp_loss_aggregate",
    "attention_fwd_head_range", "attention_bwd_head_range", "lse_merge",
    "ulysses_attn_fwd_range", "ulysses_attn_bwd_range",
]


# --------------------------------------------------------------------------
# Shape rules
# --------------------------------------------------------------------------

def check_shape(b: int, n: int, h_q: int, h_kv: int, d: int, P: int) -> None:
    """Raise ValueError unless the sizes satisfy the pages' divisibility rules.

    [TF-ALST] "Configuration": the head count must be divisible by sp_size, and
    sequences are padded to a multiple of sp_size.  With GQA both head counts
    must divide (reading above), and H_q must be a multiple of H_kv.
    """
    if P < 1:
        raise ValueError("P must be >= 1")
    if b < 1 or n < 1 or d < 1 or h_q < 1 or h_kv < 1:
        raise ValueError("sizes must be positive")
    if n % P:
        raise ValueError("sequence length must be a multiple of P")
    if h_q % P or h_kv % P:
        raise ValueError("query and kv head counts must be divisible by P")
    if h_q % h_kv:
        raise ValueError("H_q must be a multiple of H_kv")


def valid_sp_sizes(H: int) -> list:
    """All sp sizes P for which an H-head model can run ([TF-ALST] "Configuration")."""
    return [P for P in range(1, H + 1) if H % P == 0]


# --------------------------------------------------------------------------
# Sharding and the two re-layouts
# --------------------------------------------------------------------------

def shard(x: np.ndarray, P: int) -> np.ndarray:
    """[b][n][H][d] -> [P][b][n/P][H][d]; rank i holds tokens [i*n/P,(i+1)*n/P).

    [BLOG] "How Ulysses works", step 1.
    """
    b, n, H, d = x.shape
    if n % P:
        raise ValueError("n must be a multiple of P")
    m = n // P
    return np.stack([x[:, i * m:(i + 1) * m] for i in range(P)])


def unshard(xs: np.ndarray) -> np.ndarray:
    """Inverse of shard: concatenate the ranks' chunks along the sequence."""
    return np.concatenate(list(xs), axis=1)


def seq_to_head(x_seq: np.ndarray, P: int) -> np.ndarray:
    """The first all-to-all as a permutation of one buffer.

    x_head[r][bb][t][j] = x_seq[t // (n/P)][bb][t % (n/P)][r*h + j],  h = H/P.
    Rank r ends up with all n positions of its heads [r*h, (r+1)*h), the
    positions in rank order ([BLOG] "How Ulysses works", step 3; [TF-ALST]
    figure, "all N tokens, heads 0..H/2").  Written with explicit index
    arrays, element by element, not as a reshape.
    """
    Ps, b, m, H, d = x_seq.shape
    if Ps != P or H % P:
        raise ValueError("bad shape for P")
    n, h = m * P, H // P
    r = np.arange(P)[:, None, None]
    t = np.arange(n)[None, :, None]
    j = np.arange(h)[None, None, :]
    src_rank = np.broadcast_to(t // m, (P, n, h))
    src_tok = np.broadcast_to(t % m, (P, n, h))
    src_head = np.broadcast_to(r * h + j, (P, n, h))
    gathered = x_seq[src_rank, :, src_tok, src_head]          # (P, n, h, b, d)
    return np.ascontiguousarray(gathered.transpose(0, 3, 1, 2, 4))


def head_to_seq(x_head: np.ndarray, P: int) -> np.ndarray:
    """The second all-to-all: back to seq-sharded ([BLOG] step 5).

    x_seq[s][bb][u][g] = x_head[g // h][bb][s*(n/P) + u][g % h].
    """
    Ps, b, n, h, d = x_head.shape
    if Ps != P or n % P:
        raise ValueError("bad shape for P")
    m, H = n // P, h * P
    s = np.arange(P)[:, None, None]
    u = np.arange(m)[None, :, None]
    g = np.arange(H)[None, None, :]
    src_rank = np.broadcast_to(g // h, (P, m, H))
    src_tok = np.broadcast_to(s * m + u, (P, m, H))
    src_head = np.broadcast_to(g % h, (P, m, H))
    gathered = x_head[src_rank, :, src_tok, src_head]          # (P, m, H, b, d)
    return np.ascontiguousarray(gathered.transpose(0, 3, 1, 2, 4))


def kv_rank_head(P: int, H_kv: int, r: int) -> int:
    """The kv head rank r's query heads read when H_kv < P (P a multiple of
    H_kv): rank r holds query heads [r*H_q/P, (r+1)*H_q/P), all inside group
    r*H_kv//P of the GQA grouping h -> h // (H_q/H_kv)."""
    return (r * H_kv) // P


def kv_seq_to_head(x_seq: np.ndarray, P: int) -> np.ndarray:
    """K/V re-layout for the attention.  H_kv a multiple of P: seq_to_head.
    H_kv < P with P a multiple of H_kv: rank r receives all n positions of
    its one kv head (reading above): x_head[r][bb][t][0] =
    x_seq[t // (n/P)][bb][t % (n/P)][kv_rank_head(P, H_kv, r)]."""
    Ps, b, m, H, d = x_seq.shape
    if Ps != P:
        raise ValueError("bad shape for P")
    if H % P == 0:
        return seq_to_head(x_seq, P)
    if P % H:
        raise ValueError("H_kv must divide P or be divisible by it")
    n = m * P
    out = np.empty((P, b, n, 1, d), dtype=x_seq.dtype)
    for r in range(P):
        g = kv_rank_head(P, H, r)
        for t in range(0, n, m):
            out[r, :, t:t + m, 0] = x_seq[t // m, :, :, g]
    return out


def kv_head_to_seq_reduce(x_head: np.ndarray, P: int, H_kv: int) -> np.ndarray:
    """Gradient of kv_seq_to_head.  H_kv a multiple of P: head_to_seq.
    Otherwise x_seq[s][bb][u][g] = sum over ranks r with kv_rank_head(r) == g
    of x_head[r][bb][s*(n/P) + u][0]."""
    if H_kv % P == 0:
        return head_to_seq(x_head, P)
    Ps, b, n, one, d = x_head.shape
    if Ps != P or one != 1 or P % H_kv or n % P:
        raise ValueError("bad shape for P, H_kv")
    m = n // P
    out = np.zeros((P, b, m, H_kv, d), dtype=np.float64)
    for r in range(P):
        g = kv_rank_head(P, H_kv, r)
        for s_ in range(P):
            out[s_, :, :, g] += x_head[r, :, s_ * m:(s_ + 1) * m, 0]
    return out


def seq_to_head_window(x_seq: np.ndarray, P: int, r: int, t_lo: int, t_hi: int) -> np.ndarray:
    """Tokens [t_lo, t_hi) of rank r's head-sharded buffer, [b][T][H/P][d].

    The same index formula as seq_to_head, evaluated only for those rows, so
    multi-GiB buffers can be checked window by window.
    """
    Ps, b, m, H, d = x_seq.shape
    h = H // P
    t = np.arange(t_lo, t_hi)[:, None]
    j = np.arange(h)[None, :]
    shape = (t_hi - t_lo, h)
    g = x_seq[np.broadcast_to(t // m, shape), :, np.broadcast_to(t % m, shape), np.broadcast_to(r * h + j, shape)]
    return np.ascontiguousarray(g.transpose(2, 0, 1, 3))


def head_to_seq_window(x_head: np.ndarray, P: int, s: int, u_lo: int, u_hi: int) -> np.ndarray:
    """Tokens [u_lo, u_hi) of rank s's seq-sharded buffer, [b][U][H][d]."""
    Ps, b, n, h, d = x_head.shape
    m, H = n // P, h * P
    u = np.arange(u_lo, u_hi)[:, None]
    g = np.arange(H)[None, :]
    shape = (u_hi - u_lo, H)
    x = x_head[np.broadcast_to(g // h, shape), :, np.broadcast_to(s * m + u, shape), np.broadcast_to(g % h, shape)]
    return np.ascontiguousarray(x.transpose(2, 0, 1, 3))


# --------------------------------------------------------------------------
# Segments from position_ids
# --------------------------------------------------------------------------

def _starts_flag(position_ids: np.ndarray) -> np.ndarray:
    pos = np.asarray(position_ids)
    flag = pos == 0
    flag[..., 0] = True
    return flag


def segment_ids(position_ids: np.ndarray) -> np.ndarray:
    """Sample index of every token: number of sample starts at or before it."""
    return np.cumsum(_starts_flag(position_ids), axis=-1) - 1


def segment_starts(position_ids: np.ndarray) -> np.ndarray:
    """First token of the sample that holds each token."""
    flag = _starts_flag(position_ids)
    n = flag.shape[-1]
    idx = np.where(flag, np.arange(n), 0)
    return np.maximum.accumulate(idx, axis=-1)


def segment_ends(position_ids: np.ndarray) -> np.ndarray:
    """One past the last token of the sample that holds each token."""
    flag = _starts_flag(position_ids)
    n = flag.shape[-1]
    nxt = np.where(flag, np.arange(n), n)
    # next start strictly after t: shift left by one, then suffix minimum
    shifted = np.concatenate([nxt[..., 1:], np.full(nxt.shape[:-1] + (1,), n)], axis=-1)
    return np.minimum.accumulate(shifted[..., ::-1], axis=-1)[..., ::-1]


def allowed_matrix(pos_row: np.ndarray) -> np.ndarray:
    """n x n visibility: allowed[i, j] iff same sample and j <= i (brute force only)."""
    seg = segment_ids(pos_row)
    n = seg.shape[0]
    i = np.arange(n)
    return (seg[None, :] == seg[:, None]) & (i[None, :] <= i[:, None])


def default_scale(d: int) -> float:
    return 1.0 / math.sqrt(d)


# --------------------------------------------------------------------------
# Attention on one head: brute force (the definition, tiny n only)
# --------------------------------------------------------------------------

def attention_brute_head(q, k, v, pos_row, scale) -> Tuple[np.ndarray, np.ndarray]:
    """O = softmax(scale * q k^T restricted to visible keys) v, and the row LSE.

    Builds the full n x n score matrix: the literal definition, for n <= ~2048.
    """
    S = scale * (q @ k.T)
    S = np.where(allowed_matrix(pos_row), S, -np.inf)
    m = S.max(axis=1, keepdims=True)
    E = np.exp(S - m)
    l = E.sum(axis=1, keepdims=True)
    Pm = E / l
    return Pm @ v, m[:, 0] + np.log(l[:, 0])


def attention_bwd_brute_head(q, k, v, dO, pos_row, scale):
    """Gradients of sum(dO * O) w.r.t. q, k, v by the full-matrix chain rule.

    Uses the textbook softmax Jacobian, dS_ij = P_ij (dP_ij - sum_k P_ik dP_ik),
    not the D = <dO, O> shortcut, so the two formulations check each other.
    """
    S = scale * (q @ k.T)
    S = np.where(allowed_matrix(pos_row), S, -np.inf)
    m = S.max(axis=1, keepdims=True)
    E = np.exp(S - m)
    Pm = E / E.sum(axis=1, keepdims=True)
    dV = Pm.T @ dO
    dP = dO @ v.T
    dS = Pm * (dP - (Pm * dP).sum(axis=1, keepdims=True))
    return scale * (dS @ k), scale * (dS.T @ q), dV


# --------------------------------------------------------------------------
# Attention on one head: blocked (large n; never builds n x n)
# --------------------------------------------------------------------------

def _slab(q, k, seg_start, scale, i0, i1):
    """Scores of query rows [i0, i1) against their visible key range, masked."""
    lo = int(seg_start[i0])
    S = scale * (q[i0:i1] @ k[lo:i1].T)
    jj = np.arange(lo, i1)[None, :]
    ii = np.arange(i0, i1)[:, None]
    ok = (jj >= seg_start[i0:i1, None]) & (jj <= ii)
    return lo, np.where(ok, S, -np.inf)


def attention_fwd_head(q, k, v, seg_start, scale, block: int = 256,
                       row_lo: int = 0, row_hi: Optional[int] = None):
    """Blocked exact forward for rows [row_lo, row_hi) of one head.

    Each block of query rows is scored against keys from the block's first
    sample start to its last row (all keys any of its rows can see), with an
    exact two-pass softmax (row max, then exp and sum) in float64.
    """
    q = np.ascontiguousarray(q); k = np.ascontiguousarray(k); v = np.ascontiguousarray(v)
    n = q.shape[0]
    row_hi = n if row_hi is None else row_hi
    O = np.zeros((row_hi - row_lo, v.shape[1]))
    lse = np.zeros(row_hi - row_lo)
    for i0 in range(row_lo, row_hi, block):
        i1 = min(row_hi, i0 + block)
        lo, S = _slab(q, k, seg_start, scale, i0, i1)
        m = S.max(axis=1)
        E = np.exp(S - m[:, None])
        l = E.sum(axis=1)
        O[i0 - row_lo:i1 - row_lo] = (E @ v[lo:i1]) / l[:, None]
        lse[i0 - row_lo:i1 - row_lo] = m + np.log(l)
    return O, lse


def attention_bwd_head(q, k, v, dO, seg_start, scale, block: int = 256,
                       row_lo: int = 0, row_hi: Optional[int] = None):
    """Blocked exact backward: contributions of query rows [row_lo, row_hi).

    Returns dQ for those rows and dK, dV over all n keys holding only those
    rows' contributions (exact for every key whose visible rows all lie in
    the range, e.g. the whole sequence when the range is [0, n)).
    Per block: recompute P from the scores, D_i = <dO_i, O_i>,
    dS = P * (dO v^T - D), dQ = scale dS k, dK += scale dS^T q, dV += P^T dO.
    """
    q = np.ascontiguousarray(q); k = np.ascontiguousarray(k)
    v = np.ascontiguousarray(v); dO = np.ascontiguousarray(dO)
    n = q.shape[0]
    row_hi = n if row_hi is None else row_hi
    dQ = np.zeros((row_hi - row_lo, q.shape[1]))
    dK = np.zeros_like(k, dtype=np.float64)
    dV = np.zeros_like(v, dtype=np.float64)
    for i0 in range(row_lo, row_hi, block):
        i1 = min(row_hi, i0 + block)
        lo, S = _slab(q, k, seg_start, scale, i0, i1)
        m = S.max(axis=1)
        E = np.exp(S - m[:, None])
        Pm = E / E.sum(axis=1)[:, None]
        O = Pm @ v[lo:i1]
        D = (dO[i0:i1] * O).sum(axis=1)
        dP = dO[i0:i1] @ v[lo:i1].T
        dS = Pm * (dP - D[:, None])
        dQ[i0 - row_lo:i1 - row_lo] = scale * (dS @ k[lo:i1])
        dK[lo:i1] += scale * (dS.T @ q[i0:i1])
        dV[lo:i1] += Pm.T @ dO[i0:i1]
    return dQ, dK, dV


def attention_fwd_rows(q, k, v, seg_start, scale, rows: Sequence[int], key_chunk: int = 16384):
    """Exact forward for an arbitrary set of query rows of one head.

    Two passes over key chunks: the row max first, then exp, sum and the
    weighted sum of v.  Cost is |rows| x (longest visible prefix).
    """
    rows = np.asarray(rows, dtype=np.int64)
    qs = q[rows]
    ss = seg_start[rows]
    lo, hi = int(ss.min()), int(rows.max()) + 1
    m = np.full(len(rows), -np.inf)
    for c0 in range(lo, hi, key_chunk):
        c1 = min(hi, c0 + key_chunk)
        S = scale * (qs @ k[c0:c1].T)
        jj = np.arange(c0, c1)[None, :]
        S = np.where((jj >= ss[:, None]) & (jj <= rows[:, None]), S, -np.inf)
        m = np.maximum(m, S.max(axis=1))
    l = np.zeros(len(rows))
    acc = np.zeros((len(rows), v.shape[1]))
    for c0 in range(lo, hi, key_chunk):
        c1 = min(hi, c0 + key_chunk)
        S = scale * (qs @ k[c0:c1].T)
        jj = np.arange(c0, c1)[None, :]
        S = np.where((jj >= ss[:, None]) & (jj <= rows[:, None]), S, -np.inf)
        E = np.exp(S - m[:, None])
        l += E.sum(axis=1)
        acc += E @ v[c0:c1]
    return acc / l[:, None], m + np.log(l)


def attention_bwd_rows(q, k, v, dO, seg_start, scale, rows: Sequence[int], key_chunk: int = 16384):
    """Exact dQ for an arbitrary set of query rows of one head."""
    rows = np.asarray(rows, dtype=np.int64)
    O, lse = attention_fwd_rows(q, k, v, seg_start, scale, rows, key_chunk)
    qs, dOs = q[rows], dO[rows]
    ss = seg_start[rows]
    D = (dOs * O).sum(axis=1)
    lo, hi = int(ss.min()), int(rows.max()) + 1
    dQ = np.zeros_like(qs, dtype=np.float64)
    for c0 in range(lo, hi, key_chunk):
        c1 = min(hi, c0 + key_chunk)
        S = scale * (qs @ k[c0:c1].T)
        jj = np.arange(c0, c1)[None, :]
        ok = (jj >= ss[:, None]) & (jj <= rows[:, None])
        Pm = np.where(ok, np.exp(np.where(ok, S, 0.0) - lse[:, None]), 0.0)
        dP = dOs @ v[c0:c1].T
        dQ += scale * ((Pm * (dP - D[:, None])) @ k[c0:c1])
    return dQ


# --------------------------------------------------------------------------
# All heads (unsharded), GQA
# --------------------------------------------------------------------------

def attention_fwd(q, k, v, position_ids, scale: Optional[float] = None, brute: bool = False):
    """Unsharded causal attention over [b][n][H][d]; returns O and LSE [b][H_q][n]."""
    b, n, h_q, d = q.shape
    h_kv = k.shape[2]
    G = h_q // h_kv
    scale = default_scale(d) if scale is None else scale
    O = np.zeros((b, n, h_q, v.shape[3]))
    lse = np.zeros((b, h_q, n))
    ss = segment_starts(position_ids)
    for bb in range(b):
        for h in range(h_q):
            g = h // G
            if brute:
                o, l = attention_brute_head(q[bb, :, h], k[bb, :, g], v[bb, :, g], position_ids[bb], scale)
            else:
                o, l = attention_fwd_head(q[bb, :, h], k[bb, :, g], v[bb, :, g], ss[bb], scale)
            O[bb, :, h], lse[bb, h] = o, l
    return O, lse


def attention_bwd(q, k, v, dO, position_ids, scale: Optional[float] = None, brute: bool = False):
    """Unsharded backward; dK, dV of a kv head sum over its group of query heads."""
    b, n, h_q, d = q.shape
    h_kv = k.shape[2]
    G = h_q // h_kv
    scale = default_scale(d) if scale is None else scale
    dQ = np.zeros(q.shape)
    dK = np.zeros(k.shape)
    dV = np.zeros(v.shape)
    ss = segment_starts(position_ids)
    for bb in range(b):
        for h in range(h_q):
            g = h // G
            if brute:
                a, bk, c = attention_bwd_brute_head(q[bb, :, h], k[bb, :, g], v[bb, :, g],
                                                    dO[bb, :, h], position_ids[bb], scale)
            else:
                a, bk, c = attention_bwd_head(q[bb, :, h], k[bb, :, g], v[bb, :, g],
                                              dO[bb, :, h], ss[bb], scale)
            dQ[bb, :, h] = a
            dK[bb, :, g] += bk
            dV[bb, :, g] += c
    return dQ, dK, dV


# --------------------------------------------------------------------------
# Per-rank attention on head-sharded buffers, and the whole layer
# --------------------------------------------------------------------------

def _ranks(P: int, rank: Optional[int]):
    return range(P) if rank is None or rank < 0 else [rank]


def ulysses_attn_fwd(q_head, k_head, v_head, position_ids, P: int,
                     scale: Optional[float] = None, rank: Optional[int] = None):
    """Local attention of every rank (or one) on its head slice ([BLOG] step 4).

    q_head [P][b][n][H_q/P][d], k_head/v_head [P][b][n][H_kv/P][d].
    Returns O_head (same layout as q_head; zeros for ranks not computed) and
    LSE [P][b][H_q/P][n].
    """
    Ps, b, n, hq, d = q_head.shape
    hkv = k_head.shape[3]
    G = hq // hkv
    scale = default_scale(d) if scale is None else scale
    ss = segment_starts(position_ids)
    O = np.zeros(q_head.shape[:4] + (v_head.shape[4],))
    lse = np.zeros((P, b, hq, n))
    for r in _ranks(P, rank):
        for bb in range(b):
            for j in range(hq):
                o, l = attention_fwd_head(q_head[r, bb, :, j], k_head[r, bb, :, j // G],
                                          v_head[r, bb, :, j // G], ss[bb], scale)
                O[r, bb, :, j], lse[r, bb, j] = o, l
    return O, lse


def ulysses_attn_bwd(q_head, k_head, v_head, do_head, position_ids, P: int,
                     scale: Optional[float] = None, rank: Optional[int] = None):
    """Per-rank backward on head-sharded buffers: dQ, dK, dV in head layout."""
    Ps, b, n, hq, d = q_head.shape
    hkv = k_head.shape[3]
    G = hq // hkv
    scale = default_scale(d) if scale is None else scale
    ss = segment_starts(position_ids)
    dQ = np.zeros(q_head.shape)
    dK = np.zeros(k_head.shape)
    dV = np.zeros(v_head.shape)
    for r in _ranks(P, rank):
        for bb in range(b):
            for j in range(hq):
                g = j // G
                a, bk, c = attention_bwd_head(q_head[r, bb, :, j], k_head[r, bb, :, g],
                                              v_head[r, bb, :, g], do_head[r, bb, :, j],
                                              ss[bb], scale)
                dQ[r, bb, :, j] = a
                dK[r, bb, :, g] += bk
                dV[r, bb, :, g] += c
    return dQ, dK, dV


def ulysses_layer_fwd(q_seq, k_seq, v_seq, position_ids, P: int, scale: Optional[float] = None):
    """seq-sharded q, k, v -> seq_to_head -> local attention -> head_to_seq."""
    O_head, lse = ulysses_attn_fwd(seq_to_head(q_seq, P), kv_seq_to_head(k_seq, P),
                                   kv_seq_to_head(v_seq, P), position_ids, P, scale)
    return head_to_seq(O_head, P), lse


def ulysses_layer_bwd(q_seq, k_seq, v_seq, do_seq, position_ids, P: int,
                      scale: Optional[float] = None):
    """Backward of the layer: re-layout dO, local attention backward, re-layout back."""
    H_kv = k_seq.shape[3]
    dQ, dK, dV = ulysses_attn_bwd(seq_to_head(q_seq, P), kv_seq_to_head(k_seq, P),
                                  kv_seq_to_head(v_seq, P), seq_to_head(do_seq, P),
                                  position_ids, P, scale)
    return head_to_seq(dQ, P), kv_head_to_seq_reduce(dK, P, H_kv), kv_head_to_seq_reduce(dV, P, H_kv)


# --------------------------------------------------------------------------
# Attention over one key block, and the merge of blocks (ring attention)
# --------------------------------------------------------------------------

def attention_fwd_head_range(q, k, v, seg_start, scale, k_lo: int, k_hi: int, block: int = 256):
    """Attention of every query row over the keys j in [k_lo, k_hi) it may
    see (same sample, j <= i).  Rows with no such key: O = 0, LSE = -inf."""
    n = q.shape[0]
    O = np.zeros((n, v.shape[1]))
    lse = np.full(n, -np.inf)
    for i0 in range(0, n, block):
        i1 = min(n, i0 + block)
        rows = np.arange(i0, i1)
        lo = np.maximum(seg_start[i0:i1], k_lo)
        hi = np.minimum(rows + 1, k_hi)
        j0, j1 = int(lo.min()), int(hi.max())
        if j1 <= j0:
            continue
        cols = np.arange(j0, j1)
        vis = (cols[None, :] >= lo[:, None]) & (cols[None, :] < hi[:, None])
        has = vis.any(axis=1)
        S = np.where(vis, scale * (q[i0:i1] @ k[j0:j1].T), -np.inf)
        m = np.where(has, S.max(axis=1), 0.0)
        E = np.where(vis, np.exp(S - m[:, None]), 0.0)
        l = E.sum(axis=1)
        Ob, Lb = O[i0:i1], lse[i0:i1]
        Ob[has] = (E[has] @ v[j0:j1]) / l[has, None]
        Lb[has] = m[has] + np.log(l[has])
    return O, lse


def attention_bwd_head_range(q, k, v, dO, O, lse, seg_start, scale, k_lo: int, k_hi: int, block: int = 256):
    """One key block's share of the attention gradients, given the merged
    (full) O and LSE of every row: P_ij = exp(scale q_i.k_j - LSE_i) over the
    block's visible keys, D_i = dO_i . O_i, dS = P (dO v^T - D).
    Returns dQ (this block's share), dK and dV (complete for the block's
    keys, zero for the others)."""
    n = q.shape[0]
    dQ, dK, dV = np.zeros_like(q), np.zeros_like(k), np.zeros_like(v)
    D = np.sum(dO * O, axis=1)
    for i0 in range(0, n, block):
        i1 = min(n, i0 + block)
        rows = np.arange(i0, i1)
        lo = np.maximum(seg_start[i0:i1], k_lo)
        hi = np.minimum(rows + 1, k_hi)
        j0, j1 = int(lo.min()), int(hi.max())
        if j1 <= j0:
            continue
        cols = np.arange(j0, j1)
        vis = (cols[None, :] >= lo[:, None]) & (cols[None, :] < hi[:, None])
        S = scale * (q[i0:i1] @ k[j0:j1].T)
        Pm = np.where(vis, np.exp(np.where(vis, S, 0.0) - lse[i0:i1, None]), 0.0)
        dP = dO[i0:i1] @ v[j0:j1].T
        dS = Pm * (dP - D[i0:i1, None])
        dQ[i0:i1] += scale * (dS @ k[j0:j1])
        dK[j0:j1] += scale * (dS.T @ q[i0:i1])
        dV[j0:j1] += Pm.T @ dO[i0:i1]
    return dQ, dK, dV


def lse_merge(o_parts: np.ndarray, lse_parts: np.ndarray) -> Tuple[np.ndarray, np.ndarray]:
    """Merge partial results of B key blocks (head layout):
    o_parts [B][P][b][n][h][d], lse_parts [B][P][b][h][n] ->
    LSE = log sum_b exp(LSE_b); O = sum_b exp(LSE_b - LSE) O_b.
    Rows where every LSE_b is -inf: O = 0, LSE = -inf."""
    B = o_parts.shape[0]
    m = np.max(lse_parts, axis=0)                       # [P][b][h][n]
    fin = np.isfinite(m)
    msafe = np.where(fin, m, 0.0)
    total = np.zeros_like(m)
    for bk in range(B):
        total += np.where(np.isfinite(lse_parts[bk]), np.exp(lse_parts[bk] - msafe), 0.0)
    lse = np.where(fin, msafe + np.log(np.where(fin, total, 1.0)), -np.inf)
    O = np.zeros(o_parts.shape[1:])
    for bk in range(B):
        w = np.where(fin & np.isfinite(lse_parts[bk]), np.exp(lse_parts[bk] - np.where(fin, lse, 0.0)), 0.0)
        O += np.transpose(w, (0, 1, 3, 2))[..., None] * o_parts[bk]   # [P][b][n][h][1]
    return O, lse


def ulysses_attn_fwd_range(q_head, k_head, v_head, position_ids, P: int, k_lo: int, k_hi: int,
                           scale: Optional[float] = None, rank: Optional[int] = None):
    """ulysses_attn_fwd restricted to keys [k_lo, k_hi) (one ring block)."""
    Ps, b, n, hq, d = q_head.shape
    G = hq // k_head.shape[3]
    scale = default_scale(d) if scale is None else scale
    ss = segment_starts(position_ids)
    O = np.zeros(q_head.shape[:4] + (v_head.shape[4],))
    lse = np.full((P, b, hq, n), -np.inf)
    for r in _ranks(P, rank):
        for bb in range(b):
            for j in range(hq):
                O[r, bb, :, j], lse[r, bb, j] = attention_fwd_head_range(
                    q_head[r, bb, :, j], k_head[r, bb, :, j // G], v_head[r, bb, :, j // G], ss[bb], scale, k_lo, k_hi)
    return O, lse


def ulysses_attn_bwd_range(q_head, k_head, v_head, do_head, o_head, lse, position_ids, P: int, k_lo: int,
                           k_hi: int, scale: Optional[float] = None, rank: Optional[int] = None):
    """One key block's share of the per-rank backward (head layout)."""
    Ps, b, n, hq, d = q_head.shape
    G = hq // k_head.shape[3]
    scale = default_scale(d) if scale is None else scale
    ss = segment_starts(position_ids)
    dQ, dK, dV = np.zeros(q_head.shape), np.zeros(k_head.shape), np.zeros(v_head.shape)
    for r in _ranks(P, rank):
        for bb in range(b):
            for j in range(hq):
                g = j // G
                a, bk, c = attention_bwd_head_range(q_head[r, bb, :, j], k_head[r, bb, :, g], v_head[r, bb, :, g],
                                                    do_head[r, bb, :, j], o_head[r, bb, :, j], lse[r, bb, j],
                                                    ss[bb], scale, k_lo, k_hi)
                dQ[r, bb, :, j] = a
                dK[r, bb, :, g] += bk
                dV[r, bb, :, g] += c
    return dQ, dK, dV


# --------------------------------------------------------------------------
# Weighted SP loss aggregation
# --------------------------------------------------------------------------
def sp_good_tokens(shift_labels: np.ndarray, ignore_index: int = -100) -> np.ndarray:
    """Per-rank count of labels that take part in the loss ([ACC-SP] custom
    training loop: tokens labelled -100 are excluded).  shift_labels is
    seq-sharded, [P][b][n/P] (int); returns int64[P]."""
    lab = np.asarray(shift_labels)
    P = lab.shape[0]
    counts = np.zeros(P, dtype=np.int64)
    for r in range(P):
        counts[r] = int(np.count_nonzero(lab[r] != ignore_index))
    return counts


def sp_loss_aggregate(losses: np.ndarray, shift_labels: np.ndarray,
                      ignore_index: int = -100) -> Tuple[float, np.ndarray, np.ndarray]:
    """Weighted aggregation of the P per-rank losses ([ACC-SP] custom training
    loop; [BLOG] "Loss aggregation").

    total = sum over ranks r with good_r > 0 of loss_r * good_r (ranks
    without good tokens are skipped, so a NaN loss there cannot leak in);
    G = sum_r good_r; loss = total / max(G, 1).
    Returns (loss, good[P], dloss/dloss_r[P])."""
    losses = np.asarray(losses, dtype=np.float64)
    good = sp_good_tokens(shift_labels, ignore_index)
    P = losses.shape[0]
    total = 0.0
    for r in range(P):
        if good[r] > 0:
            total += losses[r] * float(good[r])
    denom = float(max(int(good.sum()), 1))
    loss = total / denom
    grad = np.zeros(P, dtype=np.float64)
    for r in range(P):
        if good[r] > 0:
            grad[r] = float(good[r]) / denom
    return loss, good, grad
