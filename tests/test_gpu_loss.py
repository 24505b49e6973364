"""GPU parity of the weighted SP loss aggregation against the fp64 oracle.

Good-token counts are integers and must match exactly.  The aggregate and
its gradient are summed in double on the GPU and rounded to float once, so
they must match the oracle to float rounding (relative 2^-23, plus 1e-30).
"""
import math

import numpy as np
import pytest
import torch

import oracle
import synthetic
from test_oracle_loss import golden_cases

pytestmark = pytest.mark.gpu

REL = 2.0 ** -23


def shard_labels(labels, P):
    """[b][n] -> seq-sharded [P][b][n/P] (rank r holds tokens [r n/P, (r+1) n/P))."""
    b, n = labels.shape
    return np.ascontiguousarray(labels.reshape(b, P, n // P).transpose(1, 0, 2))


def run(losses, labels_sharded, dev, ignore_index=-100):
    import ulysses_head_attention_b200 as uly
    P = labels_sharded.shape[0]
    t_loss = torch.from_numpy(np.asarray(losses, dtype=np.float32)).to(dev)
    t_lab = torch.from_numpy(labels_sharded).to(dev)
    out = torch.full((1,), -7.0, device=dev)
    good = torch.full((P,), -7, dtype=torch.int64, device=dev)
    dl = torch.full((P,), -7.0, device=dev)
    uly.ulysses_sp_loss_aggregate(t_loss, t_lab, out, good, dl, ignore_index=ignore_index)
    torch.cuda.synchronize()
    return float(out.item()), good.cpu().numpy(), dl.cpu().numpy()


def check(losses, labels_sharded, dev):
    loss, good, dl = run(losses, labels_sharded, dev)
    # the oracle sees exactly the float32 losses the GPU sees
    r_loss, r_good, r_dl = oracle.sp_loss_aggregate(np.asarray(losses, dtype=np.float32).astype(np.float64),
                                                    labels_sharded)
    assert np.array_equal(good, r_good)
    assert not math.isnan(loss)
    assert abs(loss - r_loss) <= REL * abs(r_loss) + 1e-30
    assert np.all(np.abs(dl - r_dl) <= REL * np.abs(r_dl) + 1e-30)
    return loss, good, dl


@pytest.mark.parametrize("case", golden_cases(), ids=lambda c: c["name"])
def test_golden_cases_on_gpu(cuda_device, case):
    labels = np.array(case["labels"], dtype=np.int64)[:, None, :]
    loss, good, dl = check(case["losses"], labels, cuda_device)
    assert np.array_equal(good, case["good"])
    assert loss == pytest.approx(case["loss"], rel=REL)
    assert np.allclose(dl, case["grad"], rtol=REL, atol=0)


@pytest.mark.parametrize("name", ["llama8b_p4_n32k", "packed_sft_p8_n64k", "long_p8_n512k"])
def test_workload_sizes(cuda_device, name):
    w = synthetic.WORKLOADS[name]
    labels = synthetic.sft_shift_labels(w.wid, synthetic.sample_lengths(w))
    check(synthetic.rank_losses(w.wid, w.P), shard_labels(labels, w.P), cuda_device)


def test_batch_rows_and_a_rank_without_valid_labels(cuda_device):
    P, b, n = 8, 3, 4096
    labels = synthetic.sft_shift_labels(5, [[1000, 3096], [4096], [17, 4079]])
    labels[:, n // P: 2 * n // P] = -100                # rank 1 holds only masked labels
    sh = shard_labels(labels, P)
    losses = synthetic.rank_losses(5, P)
    losses[1] = np.nan                                  # its loss is NaN and must not leak in
    loss, good, dl = check(losses, sh, cuda_device)
    assert good[1] == 0 and dl[1] == 0.0


def test_every_rank_empty_gives_zero(cuda_device):
    sh = np.full((4, 1, 64), -100, dtype=np.int64)
    loss, good, dl = run(np.full(4, np.nan), sh, cuda_device)
    assert loss == 0.0 and not good.any() and not dl.any()


@pytest.mark.parametrize("P,b,n", [(1, 1, 1), (1, 2, 5000), (1024, 1, 2048), (3, 1, 3 * 4099)])
def test_edge_sizes(cuda_device, P, b, n):
    lengths = [[n] for _ in range(b)]
    labels = synthetic.sft_shift_labels(P + b + n, lengths, prompt_lo=0.0, prompt_hi=0.5)
    check(synthetic.rank_losses(P, P), shard_labels(labels, P), cuda_device)


def test_other_ignore_index(cuda_device):
    labels = np.array([[[0, 0, 5]], [[5, 5, 5]]], dtype=np.int64)
    loss, good, _ = run(np.array([1.0, 3.0]), labels, cuda_device, ignore_index=0)
    assert list(good) == [1, 3] and loss == pytest.approx((1 * 1 + 3 * 3) / 4, rel=REL)


def test_deterministic(cuda_device):
    w = synthetic.WORKLOADS["packed_sft_p8_n64k"]
    sh = shard_labels(synthetic.sft_shift_labels(9, synthetic.sample_lengths(w)), w.P)
    losses = synthetic.rank_losses(9, w.P)
    a = run(losses, sh, cuda_device)
    b = run(losses, sh, cuda_device)
    assert a[0] == b[0] and np.array_equal(a[1], b[1]) and np.array_equal(a[2], b[2])
