"""Pins of the oracle's sharding and re-layouts (CPU only)."""
import numpy as np
import pytest

import oracle
from conftest import read_golden


def iota(shape):
    return np.arange(int(np.prod(shape)), dtype=np.int64).reshape(shape)


SHAPES = [(1, 8, 4, 3, 2), (2, 12, 6, 2, 3), (1, 32, 32, 4, 4), (3, 6, 4, 2, 1), (1, 16, 8, 8, 8)]


@pytest.mark.parametrize("b,n,H,d,P", SHAPES)
def test_round_trip_is_identity(b, n, H, d, P):
    x_seq = oracle.shard(iota((b, n, H, d)), P)
    assert np.array_equal(oracle.head_to_seq(oracle.seq_to_head(x_seq, P), P), x_seq)
    y_head = iota((P, b, n, H // P, d))
    assert np.array_equal(oracle.seq_to_head(oracle.head_to_seq(y_head, P), P), y_head)


def test_p1_is_identity():
    x = iota((2, 10, 3, 5))
    xs = oracle.shard(x, 1)
    assert np.array_equal(oracle.seq_to_head(xs, 1)[0], x)
    assert np.array_equal(oracle.head_to_seq(xs, 1)[0], x)


@pytest.mark.parametrize("b,n,H,d,P", SHAPES)
def test_matches_reshape_formulation(b, n, H, d, P):
    """An independent formulation: view [P][b][n/P][P][H/P][d], swap the rank axes."""
    x_seq = oracle.shard(iota((b, n, H, d)), P)
    h, m = H // P, n // P
    alt = x_seq.reshape(P, b, m, P, h, d).transpose(3, 1, 0, 2, 4, 5).reshape(P, b, n, h, d)
    assert np.array_equal(oracle.seq_to_head(x_seq, P), alt)


@pytest.mark.parametrize("b,n,H,d,P", SHAPES)
def test_every_element_written_once(b, n, H, d, P):
    x_seq = oracle.shard(iota((b, n, H, d)), P)
    out = oracle.seq_to_head(x_seq, P)
    counts = np.bincount(out.ravel(), minlength=x_seq.size)
    assert counts.min() == 1 and counts.max() == 1


def test_shard_is_contiguous_token_ranges():
    """Rank i holds tokens [i*n/P, (i+1)*n/P) ("How Ulysses works", step 1)."""
    b, n, H, d, P = 1, 12, 2, 1, 3
    tok = np.broadcast_to(np.arange(n)[None, :, None, None], (b, n, H, d))
    xs = oracle.shard(tok, P)
    for i in range(P):
        assert set(np.unique(xs[i])) == set(range(i * n // P, (i + 1) * n // P))
    assert np.array_equal(oracle.unshard(xs), tok)


def test_figure_two_gpu_layout():
    rows = read_golden("figure_p2_layout.txt")
    hdr = {r[0]: int(r[1]) for r in rows if len(r) == 2}
    N, H, P = hdr["N"], hdr["H"], hdr["P"]
    x = np.zeros((1, N, H, 1), dtype=np.int64)
    for t in range(N):
        for h in range(H):
            x[0, t, h, 0] = 100 * t + h
    xs = oracle.shard(x, P)
    xh = oracle.seq_to_head(xs, P)
    back = oracle.head_to_seq(xh, P)

    def decode(tokens):
        return [100 * int(s.split(".")[0]) + int(s.split(".")[1]) for s in tokens]

    for r in rows:
        if r[0] in ("seq_sharded", "head_sharded"):
            gpu = int(r[1][3:])
            want = decode(r[2:])
            got = (xs if r[0] == "seq_sharded" else xh)[gpu].ravel().tolist()
            assert got == want, (r[0], gpu)
            if r[0] == "seq_sharded":
                assert back[gpu].ravel().tolist() == want


@pytest.mark.parametrize("P", [1, 2, 4, 8])
def test_communication_volume(P):
    """"Communication complexity": per GPU the all-to-all moves O(n*d/P).

    Exactly, each rank keeps 1/P of its shard and sends the rest, so it
    sends (P-1)/P * n*H*d/P elements -- the message sizes of a real
    all-to-all among P GPUs.
    """
    b, n, H, d = 1, 64, 8, 4
    src_rank = np.broadcast_to((np.arange(n) // (n // P))[None, :, None, None], (b, n, H, d))
    xs = oracle.shard(src_rank, P)
    xh = oracle.seq_to_head(xs, P)
    for r in range(P):
        sent = sum(int((xh[s] == r).sum()) for s in range(P) if s != r)
        assert sent == (P - 1) * n * H * d // (P * P)


def test_sp_sizes_for_32_heads():
    rows = read_golden("sp_sizes_32_heads.txt")
    H = int(rows[0][1])
    want = [int(x) for x in rows[1][1:]]
    assert oracle.valid_sp_sizes(H) == want
    for P in range(1, 40):
        ok = P in want
        try:
            oracle.check_shape(1, 64 * P, H, H, 64, P)
            accepted = True
        except ValueError:
            accepted = False
        assert accepted == ok


@pytest.mark.parametrize("args", [
    (1, 100, 32, 8, 128, 8),    # n not a multiple of P (padding rule)
    (1, 64, 32, 8, 128, 16),    # H_kv not divisible by P
    (1, 64, 12, 8, 128, 4),     # H_q not a multiple of H_kv
    (1, 64, 32, 8, 128, 0),     # P < 1
])
def test_check_shape_rejects(args):
    with pytest.raises(ValueError):
        oracle.check_shape(*args)


@pytest.mark.parametrize("b,n,H,d,P", SHAPES)
def test_windows_match_full(b, n, H, d, P):
    x_seq = oracle.shard(iota((b, n, H, d)), P)
    x_head = oracle.seq_to_head(x_seq, P)
    for r in range(P):
        for lo, hi in ((0, n), (1, n - 1), (n // 2, n // 2 + 1)):
            assert np.array_equal(oracle.seq_to_head_window(x_seq, P, r, lo, hi), x_head[r][:, lo:hi])
    m = n // P
    for s in range(P):
        for lo, hi in ((0, m), (m - 1, m)):
            assert np.array_equal(oracle.head_to_seq_window(x_head, P, s, lo, hi), x_seq[s][:, lo:hi])
