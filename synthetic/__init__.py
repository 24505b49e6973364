"""Seeded synthetic inputs for the Ulysses hot path.

This module only draws random numbers and packs them; it holds none of the
method's arithmetic (no sharding, no re-layout, no attention).  Both the CPU
oracle tests and the GPU harness take their inputs from here, so the two sides
see the same bits.

Recipe (stated once, used everywhere):
  * bit generator: numpy PCG64 seeded with SeedSequence(20261202 + workload_id),
    spawned into independent child streams, one per tensor (q, k, v, dO) plus
    one for packed-sample lengths;
  * values: standard-normal float32 draws rounded to bfloat16 with
    round-to-nearest-even, kept as uint16 bit patterns (numpy has no bf16);
  * packed samples: lengths drawn uniformly from [lo, hi] until their sum
    reaches n, the last one truncated to fit; position_ids restart at 0 at
    every sample start (the layout the Accelerate sequence-parallelism guide
    describes for concatenated samples, "ALST/Ulysses SP backend
    configuration", sp_attn_implementation bullet).

Tensors are generated unsharded as [b][n][H][d]; for b == 1 that is
byte-identical to the seq-sharded layout [P][b][n/P][H][d].
"""
from __future__ import annotations

import dataclasses
from typing import Dict, List, Optional

import numpy as np

SEED_BASE = 20261202
STREAMS = ("q", "k", "v", "do", "lengths")


@dataclasses.dataclass(frozen=True)
class Workload:
    """Shape and structure of one synthetic workload (full, unsharded sizes)."""
    wid: int             # seeds SeedSequence(SEED_BASE + wid)
    name: str
    P: int               # virtual sequence-parallel ranks
    b: int
    n: int
    h_q: int
    h_kv: int
    d: int
    packed: bool = False         # several samples per row, position_ids restart at 0
    len_lo: int = 1024
    len_hi: int = 16384
    backward: bool = True
    rank_by_rank: bool = False   # run each virtual rank's head slice in turn

    @property
    def group(self) -> int:
        return self.h_q // self.h_kv


# The workloads, named by what they are.
WORKLOADS: Dict[str, Workload] = {
    w.name: w for w in (
        Workload(1, "tiny_p2_n256", P=2, b=1, n=256, h_q=4, h_kv=4, d=64, backward=False),
        Workload(2, "llama8b_p4_n32k", P=4, b=1, n=32768, h_q=32, h_kv=8, d=128),
        Workload(3, "packed_sft_p8_n64k", P=8, b=1, n=65536, h_q=32, h_kv=8, d=128, packed=True),
        Workload(4, "long_p8_n512k", P=8, b=1, n=524288, h_q=32, h_kv=8, d=128,
                 backward=False, rank_by_rank=True),
        Workload(5, "roundtrip_p4_n128k", P=4, b=1, n=131072, h_q=32, h_kv=8, d=128),
        # more ranks than kv heads: each rank holds a copy of one kv head
        Workload(6, "llama8b_p16_n32k_kvrep", P=16, b=1, n=32768, h_q=32, h_kv=8, d=128),
    )
}


def streams(wid: int) -> Dict[str, np.random.Generator]:
    """Independent PCG64 generators for one workload id."""
    children = np.random.SeedSequence(SEED_BASE + wid).spawn(len(STREAMS))
    return {name: np.random.Generator(np.random.PCG64(c)) for name, c in zip(STREAMS, children)}


def f32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round float32 to bfloat16 (round to nearest, ties to even); return uint16 bits."""
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32)
    bias = ((u >> 16) & np.uint32(1)) + np.uint32(0x7FFF)
    return ((u + bias) >> 16).astype(np.uint16)


def bf16_bits_to_f32(bits: np.ndarray) -> np.ndarray:
    """Widen bfloat16 bit patterns to float32 exactly."""
    return (np.ascontiguousarray(bits, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32)


def bf16_bits_to_f64(bits: np.ndarray) -> np.ndarray:
    """Widen bfloat16 bit patterns to float64 exactly."""
    return bf16_bits_to_f32(bits).astype(np.float64)


def normal_bf16(rng: np.random.Generator, shape, chunk_elems: int = 1 << 26) -> np.ndarray:
    """Standard-normal draws rounded to bf16, as uint16 bits of the given shape.

    Drawn in chunks so multi-GiB tensors never need a full float32 copy; the
    stream of values is the same for any chunk size (tested).
    """
    total = int(np.prod(shape))
    out = np.empty(total, dtype=np.uint16)
    pos = 0
    while pos < total:
        m = min(chunk_elems, total - pos)
        out[pos:pos + m] = f32_to_bf16_bits(rng.standard_normal(m, dtype=np.float32))
        pos += m
    return out.reshape(shape)


def packed_lengths(rng: np.random.Generator, n: int, lo: int, hi: int) -> List[int]:
    """Sample lengths uniform in [lo, hi] until they cover n; truncate the last."""
    lengths: List[int] = []
    total = 0
    while total < n:
        L = int(rng.integers(lo, hi + 1))
        L = min(L, n - total)
        lengths.append(L)
        total += L
    return lengths


def position_ids_from_lengths(lengths: List[int]) -> np.ndarray:
    """Concatenate arange(L) for each sample (int64)."""
    return np.concatenate([np.arange(L, dtype=np.int64) for L in lengths])


def sample_lengths(w: Workload) -> List[List[int]]:
    """Per batch row, the sample lengths of the workload."""
    rng = streams(w.wid)["lengths"]
    if not w.packed:
        return [[w.n] for _ in range(w.b)]
    return [packed_lengths(rng, w.n, w.len_lo, w.len_hi) for _ in range(w.b)]


def make_inputs(w: Workload, with_do: Optional[bool] = None) -> Dict[str, np.ndarray]:
    """All inputs of a workload as bf16 bits ([b][n][H][d]) plus position_ids ([b][n])."""
    if with_do is None:
        with_do = w.backward
    g = streams(w.wid)
    lengths = sample_lengths(w)
    out = {
        "q": normal_bf16(g["q"], (w.b, w.n, w.h_q, w.d)),
        "k": normal_bf16(g["k"], (w.b, w.n, w.h_kv, w.d)),
        "v": normal_bf16(g["v"], (w.b, w.n, w.h_kv, w.d)),
        "position_ids": np.stack([position_ids_from_lengths(ls) for ls in lengths]),
        "lengths": lengths,
    }
    if with_do:
        out["do"] = normal_bf16(g["do"], (w.b, w.n, w.h_q, w.d))
    return out


def custom_inputs(seed: int, b: int, n: int, h_q: int, h_kv: int, d: int,
                  lengths: Optional[List[List[int]]] = None, with_do: bool = True,
                  scale: float = 1.0, qk_scale: float = 1.0, do_scale: float = 1.0) -> Dict[str, np.ndarray]:
    """Inputs of an arbitrary small shape (for edge-case tests).

    ``lengths`` gives each batch row's sample lengths (default: one sample);
    ``scale`` multiplies the normal draws before bf16 rounding, and
    ``qk_scale`` multiplies those of q and k once more (large logits with
    ordinary values), ``do_scale`` those of dO (gradient magnitudes).
    """
    g = streams(10_000 + seed)
    if lengths is None:
        lengths = [[n] for _ in range(b)]
    for ls in lengths:
        assert sum(ls) == n, "sample lengths must cover the row"

    def draw(rng, shape, extra=1.0):
        x = rng.standard_normal(int(np.prod(shape)), dtype=np.float32) * np.float32(scale) * np.float32(extra)
        return f32_to_bf16_bits(x).reshape(shape)

    out = {
        "q": draw(g["q"], (b, n, h_q, d), qk_scale),
        "k": draw(g["k"], (b, n, h_kv, d), qk_scale),
        "v": draw(g["v"], (b, n, h_kv, d)),
        "position_ids": np.stack([position_ids_from_lengths(ls) for ls in lengths]),
        "lengths": lengths,
    }
    if with_do:
        out["do"] = draw(g["do"], (b, n, h_q, d), do_scale)
    return out


def sft_shift_labels(seed: int, lengths: List[List[int]], vocab: int = 128256,
                     prompt_lo: float = 0.1, prompt_hi: float = 0.6) -> np.ndarray:
    """shift_labels of packed SFT samples, int64 [b][n].

    Per sample of length L: a prompt fraction f ~ U[prompt_lo, prompt_hi];
    the first floor(f * L) positions and the sample's last position (it has
    no next token) are -100, the rest are token ids ~ U[0, vocab).  Seeded
    with SeedSequence(20261202 + 20000 + seed)."""
    rng = np.random.default_rng(np.random.SeedSequence(SEED_BASE + 20_000 + seed))
    rows = []
    for ls in lengths:
        parts = []
        for L in ls:
            lab = rng.integers(0, vocab, L, dtype=np.int64)
            cut = int(np.floor(rng.uniform(prompt_lo, prompt_hi) * L))
            lab[:cut] = -100
            lab[L - 1] = -100
            parts.append(lab)
        rows.append(np.concatenate(parts))
    return np.stack(rows)


def rank_losses(seed: int, P: int) -> np.ndarray:
    """P per-rank losses, float32 ~ U[0.5, 4)."""
    rng = np.random.default_rng(np.random.SeedSequence(SEED_BASE + 30_000 + seed))
    return rng.uniform(0.5, 4.0, P).astype(np.float32)
