"""Pins of the oracle's kv-head replication (H_kv < P).

The pages are silent on GQA with fewer kv heads than ranks; the reading is
that every rank gets a copy of the one kv head its query heads read, and that
copy's gradient is the sum over the ranks holding it.  Checked against:
the plain re-layouts where H_kv is a multiple of P (the rule must reduce to
them); the adjoint identity <R x, y> = <x, R^T y> that makes the sum the
gradient of the copy; and the whole layer against unsharded attention,
forward and backward, which is what the replication exists to reproduce.
"""
import numpy as np
import pytest

import oracle


def rnd(rng, *shape):
    return rng.standard_normal(shape)


def test_reduces_to_plain_relayout_when_heads_divide():
    rng = np.random.default_rng(1)
    P, b, m, H, d = 4, 2, 3, 8, 5
    x = rnd(rng, P, b, m, H, d)
    assert np.array_equal(oracle.kv_seq_to_head(x, P), oracle.seq_to_head(x, P))
    y = rnd(rng, P, b, m * P, H // P, d)
    assert np.array_equal(oracle.kv_head_to_seq_reduce(y, P, H), oracle.head_to_seq(y, P))


@pytest.mark.parametrize("P,H", [(4, 2), (8, 2), (8, 1), (6, 3)])
def test_replicas_are_exact_copies(P, H):
    rng = np.random.default_rng(P * 10 + H)
    b, m, d = 2, 3, 4
    x = rnd(rng, P, b, m, H, d)
    out = oracle.kv_seq_to_head(x, P)
    assert out.shape == (P, b, m * P, 1, d)
    unsharded = oracle.unshard(x)                       # [b][n][H][d]
    for r in range(P):
        g = oracle.kv_rank_head(P, H, r)
        assert np.array_equal(out[r, :, :, 0], unsharded[:, :, g])
    # every kv head is held by exactly P / H ranks
    holders = [oracle.kv_rank_head(P, H, r) for r in range(P)]
    assert all(holders.count(g) == P // H for g in range(H))


@pytest.mark.parametrize("P,H", [(4, 2), (8, 2), (6, 3)])
def test_reduce_is_the_adjoint_of_the_copy(P, H):
    rng = np.random.default_rng(100 + P + H)
    b, m, d = 2, 5, 3
    x = rnd(rng, P, b, m, H, d)
    y = rnd(rng, P, b, m * P, 1, d)
    lhs = float(np.sum(oracle.kv_seq_to_head(x, P) * y))
    rhs = float(np.sum(x * oracle.kv_head_to_seq_reduce(y, P, H)))
    assert lhs == pytest.approx(rhs, rel=1e-12)


def test_rank_groups_match_gqa_grouping():
    # rank r's query heads [r*H_q/P, (r+1)*H_q/P) all read kv head kv_rank_head(r)
    for H_q, H_kv, P in ((32, 8, 16), (32, 8, 32), (8, 2, 8), (12, 3, 6)):
        G, hq = H_q // H_kv, H_q // P
        for r in range(P):
            assert {h // G for h in range(r * hq, (r + 1) * hq)} == {oracle.kv_rank_head(P, H_kv, r)}


@pytest.mark.parametrize("P,H_q,H_kv", [(8, 8, 2), (4, 8, 1)])
def test_layer_with_replication_equals_unsharded_attention(P, H_q, H_kv):
    rng = np.random.default_rng(7 + P)
    b, n, d = 1, 48, 8
    q, k, v, do = rnd(rng, b, n, H_q, d), rnd(rng, b, n, H_kv, d), rnd(rng, b, n, H_kv, d), rnd(rng, b, n, H_q, d)
    pos = np.concatenate([np.arange(20), np.arange(28)])[None, :]
    O_ref, _ = oracle.attention_fwd(q, k, v, pos)
    dq_ref, dk_ref, dv_ref = oracle.attention_bwd(q, k, v, do, pos)
    sh = [oracle.shard(t, P) for t in (q, k, v, do)]
    O, _ = oracle.ulysses_layer_fwd(sh[0], sh[1], sh[2], pos, P)
    assert np.allclose(oracle.unshard(O), O_ref, rtol=0, atol=1e-12)
    dq, dk, dv = oracle.ulysses_layer_bwd(*sh, pos, P)
    assert np.allclose(oracle.unshard(dq), dq_ref, rtol=0, atol=1e-12)
    assert np.allclose(oracle.unshard(dk), dk_ref, rtol=0, atol=1e-12)
    assert np.allclose(oracle.unshard(dv), dv_ref, rtol=0, atol=1e-12)
