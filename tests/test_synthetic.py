"""The seeded input generator: determinism, rounding, packed-sample recipe."""
import numpy as np
import torch

import synthetic


def test_bf16_rounding_matches_torch():
    rng = np.random.default_rng(1)
    x = np.concatenate([rng.standard_normal(100000).astype(np.float32),
                        np.array([1.0 + 2 ** -8, 1.0 + 3 * 2 ** -8, -0.0, 0.0, 65504.0], np.float32)])
    want = torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(synthetic.f32_to_bf16_bits(x), want)
    back = synthetic.bf16_bits_to_f32(want)
    assert np.array_equal(back, torch.from_numpy(x).to(torch.bfloat16).float().numpy())


def test_streams_are_deterministic_and_chunk_invariant():
    a = synthetic.normal_bf16(synthetic.streams(3)["q"], (5, 1000))
    b = synthetic.normal_bf16(synthetic.streams(3)["q"], (5, 1000), chunk_elems=333)
    c = synthetic.normal_bf16(synthetic.streams(3)["k"], (5, 1000))
    assert np.array_equal(a, b)
    assert not np.array_equal(a, c)


def test_packed_lengths_recipe():
    w = synthetic.WORKLOADS["packed_sft_p8_n64k"]
    (ls,) = synthetic.sample_lengths(w)
    assert sum(ls) == w.n
    assert all(w.len_lo <= L <= w.len_hi for L in ls[:-1])
    assert 1 <= ls[-1] <= w.len_hi
    pos = synthetic.position_ids_from_lengths(ls)
    starts = np.nonzero(pos == 0)[0]
    assert np.array_equal(starts, np.cumsum([0] + ls[:-1]))


def test_workload_table_obeys_divisibility():
    for w in synthetic.WORKLOADS.values():
        assert w.n % w.P == 0 and w.h_q % w.P == 0 and w.h_q % w.h_kv == 0
        # kv heads: divisible by P, or (kv-head replication) a divisor of P
        assert w.h_kv % w.P == 0 or (w.h_kv < w.P and w.P % w.h_kv == 0)
