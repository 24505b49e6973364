"""Pins of the oracle's weighted SP loss aggregation.

Checked against: the hand-worked cases in tests/golden/sp_loss_aggregation.txt;
the identity the weighting exists for (aggregating per-rank means of
per-token losses gives the mean over every valid token of the sequence);
central finite differences for the gradient; the single-rank case.
"""
import math

import numpy as np
import pytest

import oracle
from conftest import read_golden


def golden_cases():
    cases, cur = [], None
    for row in read_golden("sp_loss_aggregation.txt"):
        key = row[0]
        if key == "case":
            cur = {"name": row[1], "labels": []}
            cases.append(cur)
        elif key == "losses":
            cur["losses"] = np.array([float(v) for v in row[1:]])
        elif key == "labels":
            cur["labels"].append([int(v) for v in row[3:]])
        elif key == "good":
            cur["good"] = np.array([int(v) for v in row[1:]])
        elif key == "loss":
            cur["loss"] = float(row[1])
        elif key == "grad":
            cur["grad"] = np.array([float(v) for v in row[1:]])
    return cases


@pytest.mark.parametrize("case", golden_cases(), ids=lambda c: c["name"])
def test_golden_cases(case):
    labels = np.array(case["labels"], dtype=np.int64)[:, None, :]   # [P][b=1][n/P]
    loss, good, grad = oracle.sp_loss_aggregate(case["losses"], labels)
    assert np.array_equal(good, case["good"])
    assert not math.isnan(loss)
    assert loss == pytest.approx(case["loss"], abs=1e-15)
    assert np.allclose(grad, case["grad"], rtol=0, atol=1e-15)


def test_equals_mean_over_all_valid_tokens():
    rng = np.random.default_rng(7)
    P, b, m = 4, 2, 64
    labels = rng.integers(0, 1000, (P, b, m))
    labels[rng.random((P, b, m)) < 0.4] = -100
    labels[2] = -100                                   # one rank holds only masked tokens
    tok_loss = rng.random((P, b, m)) * 5.0
    per_rank = np.array([tok_loss[r][labels[r] != -100].mean() if (labels[r] != -100).any() else np.nan
                         for r in range(P)])
    loss, good, _ = oracle.sp_loss_aggregate(per_rank, labels)
    assert good[2] == 0
    assert loss == pytest.approx(tok_loss[labels != -100].mean(), rel=1e-13)


def test_gradient_matches_finite_differences():
    rng = np.random.default_rng(8)
    P = 5
    labels = rng.integers(0, 50, (P, 1, 32))
    labels[rng.random(labels.shape) < 0.5] = -100
    labels[1] = -100
    losses = rng.random(P) * 3.0
    _, good, grad = oracle.sp_loss_aggregate(losses, labels)
    h = 1e-6
    for r in range(P):
        up, dn = losses.copy(), losses.copy()
        up[r] += h
        dn[r] -= h
        fd = (oracle.sp_loss_aggregate(up, labels)[0] - oracle.sp_loss_aggregate(dn, labels)[0]) / (2 * h)
        assert grad[r] == pytest.approx(fd, abs=1e-8)
    assert grad[1] == 0.0
    assert grad.sum() == pytest.approx(1.0)


def test_single_rank_is_its_own_loss():
    labels = np.array([[[3, -100, 4]]])
    loss, good, grad = oracle.sp_loss_aggregate(np.array([2.5]), labels)
    assert (loss, int(good[0]), grad[0]) == (2.5, 2, 1.0)


def test_ignore_index_is_the_only_excluded_label():
    """Only labels equal to the ignore index are left out: with ignore_index
    = -1, the -100 labels count and the -1 labels do not."""
    labels = np.array([[[-1, -100, 7]], [[-1, -1, -1]]])
    loss, good, grad = oracle.sp_loss_aggregate(np.array([3.0, float("nan")]), labels, ignore_index=-1)
    assert good.tolist() == [2, 0]
    assert (loss, grad.tolist()) == (3.0, [1.0, 0.0])
