"""Pins of the oracle's attention forward/backward (CPU only).

Each test checks the oracle against something other than itself: the
full-matrix definition, torch's fp64 SDPA (a library routine), closed forms,
finite differences, or layout/segment facts the pages state.
"""
import math

import numpy as np
import pytest
import torch

import oracle
import synthetic
from conftest import read_golden


def f64(bits):
    return synthetic.bf16_bits_to_f64(bits)


def case(seed, b, n, hq, hkv, d, lengths=None, scale=1.0):
    x = synthetic.custom_inputs(seed, b, n, hq, hkv, d, lengths=lengths, scale=scale)
    return f64(x["q"]), f64(x["k"]), f64(x["v"]), f64(x["do"]), x["position_ids"]


def rel(a, b):
    return np.abs(a - b).max() / max(np.abs(b).max(), 1e-300)


# ---------------------------------------------------------------- segments

def brute_segment_tables(pos):
    n = len(pos)
    starts, ends = [], []
    for t in range(n):
        s = t
        while s > 0 and pos[s] != 0:
            s -= 1
        e = t + 1
        while e < n and pos[e] != 0:
            e += 1
        starts.append(s)
        ends.append(e)
    return np.array(starts), np.array(ends)


@pytest.mark.parametrize("pos", [
    [0, 1, 2, 3, 4, 5],
    [0, 1, 2, 0, 1, 0, 0, 1, 2, 3],
    [5, 6, 7, 0, 1],           # row not starting at 0: token 0 still starts a sample
    [0, 0, 0, 0],
    [0],
])
def test_segment_tables(pos):
    pos = np.array(pos, dtype=np.int64)
    s, e = brute_segment_tables(pos)
    assert np.array_equal(oracle.segment_starts(pos), s)
    assert np.array_equal(oracle.segment_ends(pos), e)
    seg = oracle.segment_ids(pos)
    for t in range(len(pos)):
        assert (seg == seg[t]).sum() == e[t] - s[t]
    # sample indices count from 0 at token 0, one up at every later start
    assert seg[0] == 0
    assert np.array_equal(np.diff(seg), (pos[1:] == 0).astype(seg.dtype))


def test_packed_visibility_golden():
    rows = read_golden("packed_sample_visibility.txt")
    pos = np.array([int(x) for x in rows[0][1:]])
    A = oracle.allowed_matrix(pos)
    for r in rows[1:]:
        i = int(r[1])
        want = sorted(int(x) for x in r[3:])
        assert np.nonzero(A[i])[0].tolist() == want


# ---------------------------------------------------------------- forward

@pytest.mark.parametrize("n,lengths", [
    (300, None), (257, [[100, 57, 100]]), (512, [[1, 1, 200, 255, 55]]), (64, [[64]]),
])
def test_blocked_equals_brute(n, lengths):
    q, k, v, do, pos = case(1, 1, n, 4, 2, 16, lengths)
    O1, L1 = oracle.attention_fwd(q, k, v, pos, brute=True)
    for block in (64, 256):
        ss = oracle.segment_starts(pos)[0]
        for h in range(4):
            o, l = oracle.attention_fwd_head(q[0, :, h], k[0, :, h // 2], v[0, :, h // 2], ss,
                                             1 / 4, block=block)
            assert rel(o, O1[0, :, h]) < 1e-12
            assert rel(l, L1[0, h]) < 1e-12


def test_matches_torch_sdpa_single_sample():
    """A single sample is textbook causal softmax attention."""
    q, k, v, do, pos = case(2, 2, 200, 4, 4, 32)
    O, L = oracle.attention_fwd(q, k, v, pos)
    t = lambda x: torch.from_numpy(x).permute(0, 2, 1, 3)
    ref = torch.nn.functional.scaled_dot_product_attention(t(q), t(k), t(v), is_causal=True)
    assert rel(O, ref.permute(0, 2, 1, 3).numpy()) < 1e-12


def test_matches_torch_sdpa_per_packed_sample():
    lengths = [[70, 1, 129, 56]]
    q, k, v, do, pos = case(3, 1, 256, 2, 2, 16, lengths)
    O, L = oracle.attention_fwd(q, k, v, pos)
    s = 0
    t = lambda x: torch.from_numpy(x).permute(0, 2, 1, 3)
    for Ls in lengths[0]:
        sl = slice(s, s + Ls)
        ref = torch.nn.functional.scaled_dot_product_attention(
            t(q[:, sl]), t(k[:, sl]), t(v[:, sl]), is_causal=True)
        assert rel(O[:, sl], ref.permute(0, 2, 1, 3).numpy()) < 1e-12
        s += Ls


def test_lse_matches_logsumexp():
    from scipy.special import logsumexp
    q, k, v, do, pos = case(4, 1, 128, 2, 1, 8, [[50, 78]])
    O, L = oracle.attention_fwd(q, k, v, pos)
    A = oracle.allowed_matrix(pos[0])
    for h in range(2):
        S = (q[0, :, h] @ k[0, :, 0].T) / math.sqrt(8)
        for i in range(128):
            assert abs(L[0, h, i] - logsumexp(S[i][A[i]])) < 1e-12


def test_single_token_returns_v0():
    q, k, v, do, pos = case(5, 1, 1, 2, 2, 8)
    O, L = oracle.attention_fwd(q, k, v, pos)
    assert np.array_equal(O[0, 0], v[0, 0])
    for h in range(2):
        assert abs(L[0, h, 0] - q[0, 0, h] @ k[0, 0, h] / math.sqrt(8)) < 1e-14


def test_uniform_keys_closed_form():
    """Equal keys -> uniform weights: O_i = mean of visible v, LSE_i = s_i + ln(count)."""
    lengths = [[40, 60, 28]]
    q, k, v, do, pos = case(6, 1, 128, 2, 1, 16, lengths)
    k[:] = k[0, 0]
    O, L = oracle.attention_fwd(q, k, v, pos)
    ss = oracle.segment_starts(pos)[0]
    for h in range(2):
        for i in range(128):
            want = v[0, ss[i]:i + 1, 0].mean(axis=0)
            assert np.abs(O[0, i, h] - want).max() < 1e-12
            s = q[0, i, h] @ k[0, 0, 0] / 4.0
            assert abs(L[0, h, i] - (s + math.log(i + 1 - ss[i]))) < 1e-12


def test_constant_v_gives_v():
    q, k, v, do, pos = case(7, 1, 96, 2, 2, 8, [[33, 63]])
    v[:] = v[0, 0]
    O, _ = oracle.attention_fwd(q, k, v, pos)
    assert np.abs(O - v[0, 0]).max() < 1e-12


def test_gqa_equals_mha_on_repeated_kv():
    q, k, v, do, pos = case(8, 1, 160, 8, 2, 16, [[100, 60]])
    G = 4
    kr, vr = np.repeat(k, G, axis=2), np.repeat(v, G, axis=2)
    O1, L1 = oracle.attention_fwd(q, k, v, pos)
    O2, L2 = oracle.attention_fwd(q, kr, vr, pos)
    assert np.array_equal(O1, O2) and np.array_equal(L1, L2)
    dq1, dk1, dv1 = oracle.attention_bwd(q, k, v, do, pos)
    dq2, dk2, dv2 = oracle.attention_bwd(q, kr, vr, do, pos)
    assert np.array_equal(dq1, dq2)
    assert rel(dk1, dk2.reshape(1, 160, 2, G, 16).sum(axis=3)) < 1e-12
    assert rel(dv1, dv2.reshape(1, 160, 2, G, 16).sum(axis=3)) < 1e-12


def test_packed_equals_separate_and_negative_control():
    """A packed row equals its samples run one by one; ignoring the
    boundaries (the whole row as one sample) gives a different answer."""
    lengths = [[90, 1, 37, 128]]
    n = 256
    q, k, v, do, pos = case(9, 1, n, 4, 2, 16, lengths)
    O, L = oracle.attention_fwd(q, k, v, pos)
    dq, dk, dv = oracle.attention_bwd(q, k, v, do, pos)
    s = 0
    for Ls in lengths[0]:
        sl = slice(s, s + Ls)
        one = np.arange(Ls)[None]
        o, l = oracle.attention_fwd(q[:, sl], k[:, sl], v[:, sl], one)
        a, bk, c = oracle.attention_bwd(q[:, sl], k[:, sl], v[:, sl], do[:, sl], one)
        assert rel(O[:, sl], o) < 1e-12 and rel(L[:, :, sl], l) < 1e-12
        assert rel(dq[:, sl], a) < 1e-12 and rel(dk[:, sl], bk) < 1e-12 and rel(dv[:, sl], c) < 1e-12
        s += Ls
    O_one, _ = oracle.attention_fwd(q, k, v, np.arange(n)[None])
    assert np.abs(O_one[:, 90:] - O[:, 90:]).max() > 1e-2
    assert np.array_equal(O_one[:, :90], O[:, :90])


@pytest.mark.parametrize("hq,hkv,P_list", [(8, 8, [1, 2, 4, 8]), (8, 4, [1, 2, 4]), (16, 4, [1, 2, 4])])
def test_ulysses_equals_unsharded(hq, hkv, P_list):
    """Heads are independent ("How Ulysses works"), so the layer equals plain
    attention for every P dividing both head counts -- bitwise."""
    n = 64
    q, k, v, do, pos = case(10, 1, n, hq, hkv, 8, [[20, 44]])
    O_ref, L_ref = oracle.attention_fwd(q, k, v, pos)
    dq_ref, dk_ref, dv_ref = oracle.attention_bwd(q, k, v, do, pos)
    for P in P_list:
        sh = lambda x: oracle.shard(x, P)
        O_seq, lse = oracle.ulysses_layer_fwd(sh(q), sh(k), sh(v), pos, P)
        assert np.array_equal(oracle.unshard(O_seq), O_ref)
        # lse [P][b][hq/P][n] -> global head order
        assert np.array_equal(lse.transpose(1, 0, 2, 3).reshape(1, hq, n), L_ref)
        dq, dk, dv = oracle.ulysses_layer_bwd(sh(q), sh(k), sh(v), sh(do), pos, P)
        assert np.array_equal(oracle.unshard(dq), dq_ref)
        assert np.array_equal(oracle.unshard(dk), dk_ref)
        assert np.array_equal(oracle.unshard(dv), dv_ref)


def test_single_rank_mode_matches_all_ranks():
    q, k, v, do, pos = case(11, 1, 64, 8, 4, 8)
    P = 4
    qh, kh, vh = (oracle.seq_to_head(oracle.shard(x, P), P) for x in (q, k, v))
    O_all, L_all = oracle.ulysses_attn_fwd(qh, kh, vh, pos, P)
    for r in range(P):
        O_r, L_r = oracle.ulysses_attn_fwd(qh, kh, vh, pos, P, rank=r)
        assert np.array_equal(O_r[r], O_all[r]) and np.array_equal(L_r[r], L_all[r])


def test_rows_functions_match_blocked():
    lengths = [[300, 2, 210]]
    q, k, v, do, pos = case(12, 1, 512, 2, 1, 16, lengths)
    ss = oracle.segment_starts(pos)[0]
    rows = [0, 1, 299, 300, 301, 302, 400, 511]
    o_full, l_full = oracle.attention_fwd_head(q[0, :, 1], k[0, :, 0], v[0, :, 0], ss, 0.25)
    o, l = oracle.attention_fwd_rows(q[0, :, 1], k[0, :, 0], v[0, :, 0], ss, 0.25, rows, key_chunk=100)
    assert rel(o, o_full[rows]) < 1e-12 and rel(l, l_full[rows]) < 1e-12
    dq_full, _, _ = oracle.attention_bwd_head(q[0, :, 1], k[0, :, 0], v[0, :, 0], do[0, :, 1], ss, 0.25)
    dq = oracle.attention_bwd_rows(q[0, :, 1], k[0, :, 0], v[0, :, 0], do[0, :, 1], ss, 0.25, rows,
                                   key_chunk=77)
    assert rel(dq, dq_full[rows]) < 1e-12


def test_row_window_backward_is_exact_for_late_keys():
    n = 384
    q, k, v, do, pos = case(13, 1, n, 1, 1, 16)
    ss = oracle.segment_starts(pos)[0]
    a, bk, c = oracle.attention_bwd_head(q[0, :, 0], k[0, :, 0], v[0, :, 0], do[0, :, 0], ss, 0.25)
    a2, bk2, c2 = oracle.attention_bwd_head(q[0, :, 0], k[0, :, 0], v[0, :, 0], do[0, :, 0], ss, 0.25,
                                            row_lo=300)
    assert rel(bk2[300:], bk[300:]) < 1e-12 and rel(c2[300:], c[300:]) < 1e-12
    assert rel(a2, a[300:]) < 1e-12


# ---------------------------------------------------------------- backward

def test_backward_blocked_equals_brute_jacobian():
    lengths = [[100, 3, 153]]
    q, k, v, do, pos = case(14, 1, 256, 4, 2, 16, lengths)
    g1 = oracle.attention_bwd(q, k, v, do, pos, brute=True)
    g2 = oracle.attention_bwd(q, k, v, do, pos)
    for a, b in zip(g1, g2):
        assert rel(b, a) < 1e-11


def test_backward_finite_differences():
    """Central differences of L = sum(dO * O) in fp64 on a tiny packed case."""
    rng = np.random.default_rng(0)
    n, hq, hkv, d = 12, 2, 1, 4
    q = rng.standard_normal((1, n, hq, d)); k = rng.standard_normal((1, n, hkv, d))
    v = rng.standard_normal((1, n, hkv, d)); do = rng.standard_normal((1, n, hq, d))
    pos = np.array([[0, 1, 2, 3, 4, 0, 1, 2, 0, 1, 2, 3]])
    dq, dk, dv = oracle.attention_bwd(q, k, v, do, pos, brute=True)

    def loss(q_, k_, v_):
        O, _ = oracle.attention_fwd(q_, k_, v_, pos, brute=True)
        return float((O * do).sum())

    eps = 1e-6
    for name, X, G in (("q", q, dq), ("k", k, dk), ("v", v, dv)):
        num = np.zeros_like(X)
        for idx in np.ndindex(X.shape):
            Xp, Xm = X.copy(), X.copy()
            Xp[idx] += eps
            Xm[idx] -= eps
            args_p = {"q": q, "k": k, "v": v}; args_m = dict(args_p)
            args_p[name], args_m[name] = Xp, Xm
            num[idx] = (loss(**{kk + "_": vv for kk, vv in args_p.items()})
                        - loss(**{kk + "_": vv for kk, vv in args_m.items()})) / (2 * eps)
        assert np.abs(num - G).max() <= 1e-6 * max(1.0, np.abs(G).max()), name


def test_backward_column_sums():
    """sum_j dK_j = 0 (rows of dS sum to zero) and sum_j dV_j = sum over the
    group's query heads and rows of dO (rows of P sum to one)."""
    lengths = [[150, 106]]
    q, k, v, do, pos = case(15, 1, 256, 4, 2, 16, lengths)
    dq, dk, dv = oracle.attention_bwd(q, k, v, do, pos)
    for g in range(2):
        assert np.abs(dk[0, :, g].sum(axis=0)).max() < 1e-12 * np.abs(dk).sum()
        want = do[0, :, 2 * g:2 * g + 2].sum(axis=(0, 1))
        assert np.abs(dv[0, :, g].sum(axis=0) - want).max() < 1e-11
