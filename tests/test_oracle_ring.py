"""Pins of the oracle's key-block attention and LSE merge (ring attention).

Checked against: a per-row loop over the explicit list of visible keys in
the block (softmax written out, no blocking, no masking arrays); the full
attention (one block covering every key); the merge of a partition of the
keys, which must give the full attention back; and, for the backward, the
full gradients (pinned elsewhere by brute force and finite differences):
the blocks' dQ shares add up to dQ, and each block's dK, dV are the full
rows of its keys and zero elsewhere.
"""
import math

import numpy as np
import pytest

import oracle


def inputs(seed, n=160, d=8):
    rng = np.random.default_rng(seed)
    q, k, v, do = (rng.standard_normal((n, d)) for _ in range(4))
    pos = np.concatenate([np.arange(50), np.arange(70), np.arange(40)])
    return q, k, v, do, pos, oracle.segment_starts(pos)


@pytest.mark.parametrize("k_lo,k_hi", [(0, 160), (30, 90), (55, 56), (150, 160), (0, 1)])
def test_block_matches_per_row_definition(k_lo, k_hi):
    q, k, v, _, pos, ss = inputs(1)
    scale = 0.37
    O, lse = oracle.attention_fwd_head_range(q, k, v, ss, scale, k_lo, k_hi, block=64)
    seg = oracle.segment_ids(pos)
    for i in range(len(q)):
        keys = [j for j in range(k_lo, k_hi) if j <= i and seg[j] == seg[i]]
        if not keys:
            assert lse[i] == -math.inf and not O[i].any()
            continue
        s = [scale * float(q[i] @ k[j]) for j in keys]
        mx = max(s)
        w = [math.exp(x - mx) for x in s]
        tot = sum(w)
        o = sum(wi * v[j] for wi, j in zip(w, keys)) / tot
        assert np.allclose(O[i], o, rtol=0, atol=1e-12)
        assert lse[i] == pytest.approx(mx + math.log(tot), abs=1e-12)


def test_one_block_over_all_keys_is_full_attention():
    q, k, v, do, pos, ss = inputs(2)
    O_full, L_full = oracle.attention_brute_head(q, k, v, pos, 0.5)
    O, L = oracle.attention_fwd_head_range(q, k, v, ss, 0.5, 0, len(q))
    assert np.allclose(O, O_full, atol=1e-12) and np.allclose(L, L_full, atol=1e-12)


@pytest.mark.parametrize("cuts", [[0, 160], [0, 64, 128, 160], [0, 1, 50, 51, 119, 160], [0, 40, 80, 120, 160]])
def test_merge_of_a_partition_is_full_attention(cuts):
    q, k, v, do, pos, ss = inputs(3)
    scale = 0.4
    parts = [oracle.attention_fwd_head_range(q, k, v, ss, scale, a, b) for a, b in zip(cuts[:-1], cuts[1:])]
    # head layout with P = b = h = 1
    o_parts = np.stack([p[0] for p in parts])[:, None, None, :, None, :]
    l_parts = np.stack([p[1] for p in parts])[:, None, None, None, :]
    O, L = oracle.lse_merge(o_parts, l_parts)
    O_full, L_full = oracle.attention_brute_head(q, k, v, pos, scale)
    assert np.allclose(O[0, 0, :, 0], O_full, atol=1e-12)
    assert np.allclose(L[0, 0, 0], L_full, atol=1e-12)


def test_merge_of_empty_rows_and_order_independence():
    rng = np.random.default_rng(4)
    o = rng.standard_normal((3, 1, 1, 5, 1, 2))
    l = rng.standard_normal((3, 1, 1, 1, 5))
    l[:, 0, 0, 0, 2] = -np.inf                          # row 2: no block saw a key
    l[1, 0, 0, 0, 3] = -np.inf                          # row 3: one block empty
    O, L = oracle.lse_merge(o, l)
    assert L[0, 0, 0, 2] == -np.inf and not O[0, 0, 2].any()
    O2, L2 = oracle.lse_merge(o[::-1], l[::-1])
    assert np.allclose(O, O2, atol=1e-14) and np.allclose(L[np.isfinite(L)], L2[np.isfinite(L2)])
    # row 3 equals the merge of blocks 0 and 2 only
    O3, L3 = oracle.lse_merge(o[[0, 2]], l[[0, 2]])
    assert np.allclose(O[0, 0, 3], O3[0, 0, 3]) and L[0, 0, 0, 3] == pytest.approx(L3[0, 0, 0, 3])


@pytest.mark.parametrize("cuts", [[0, 160], [0, 64, 128, 160], [0, 1, 50, 51, 119, 160]])
def test_block_backward_shares_add_up(cuts):
    q, k, v, do, pos, ss = inputs(5)
    scale = 0.3
    O, L = oracle.attention_fwd_head(q, k, v, ss, scale)
    dq_ref, dk_ref, dv_ref = oracle.attention_bwd_brute_head(q, k, v, do, pos, scale)
    dq = np.zeros_like(q)
    for a, b in zip(cuts[:-1], cuts[1:]):
        gq, gk, gv = oracle.attention_bwd_head_range(q, k, v, do, O, L, ss, scale, a, b)
        dq += gq
        assert np.allclose(gk[a:b], dk_ref[a:b], atol=1e-11) and not gk[:a].any() and not gk[b:].any()
        assert np.allclose(gv[a:b], dv_ref[a:b], atol=1e-11) and not gv[:a].any() and not gv[b:].any()
    assert np.allclose(dq, dq_ref, atol=1e-11)


@pytest.mark.parametrize("base", [0.0, 1000.0, -1000.0, 700.0])
def test_merge_closed_form_at_extreme_lse(base):
    """Two blocks with LSE base and base + ln 3 weigh their outputs 1/4 and
    3/4, and the merged LSE is base + ln 4, however large |base| is (the
    merge must not form exp(LSE) itself)."""
    o = np.zeros((2, 1, 1, 1, 1, 2))
    o[0, ..., 0] = 1.0
    o[1, ..., 1] = 1.0
    l = np.array([base, base + math.log(3.0)]).reshape(2, 1, 1, 1, 1)
    O, L = oracle.lse_merge(o, l)
    # base + ln 3 is stored to the ulp of |base| (1.1e-13 at 1000), which the
    # weights inherit
    assert np.allclose(O[0, 0, 0, 0], [0.25, 0.75], rtol=0, atol=1e-12)
    assert L[0, 0, 0, 0] == pytest.approx(base + math.log(4.0), abs=1e-12)


def test_merge_of_blocks_far_apart_keeps_the_dominant_one():
    """LSEs 800 and -800: the second block's weight exp(-1600) is 0 in any
    float format, so the merge returns the first block unchanged."""
    o = np.stack([np.full((1, 1, 1, 1, 3), 2.0), np.full((1, 1, 1, 1, 3), -5.0)])
    l = np.array([800.0, -800.0]).reshape(2, 1, 1, 1, 1)
    O, L = oracle.lse_merge(o, l)
    assert np.array_equal(O[0, 0, 0, 0], [2.0, 2.0, 2.0]) and L[0, 0, 0, 0] == 800.0
