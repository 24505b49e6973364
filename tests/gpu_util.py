"""Shared helpers for the GPU parity tests (data movement and error metrics only)."""
import numpy as np
import torch


def to_dev_bf16(bits: np.ndarray, device) -> torch.Tensor:
    """uint16 bf16 bit patterns -> bfloat16 CUDA tensor (same bits)."""
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).to(device)


def bits_of(t: torch.Tensor) -> np.ndarray:
    """bfloat16 tensor -> uint16 bit patterns on the host."""
    return t.contiguous().view(torch.int16).cpu().numpy().view(np.uint16)


def shard_b1(x: np.ndarray, P: int) -> np.ndarray:
    """[1][n][H][d] -> [P][1][n/P][H][d]; for b == 1 this is a pure reshape (same bytes)."""
    b, n, H, d = x.shape
    assert b == 1
    return x.reshape(P, 1, n // P, H, d)


def errors(got: np.ndarray, ref: np.ndarray):
    """(max-abs, mean-relative = sum|g-r| / sum|r|)."""
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    diff = np.abs(got - ref)
    return float(diff.max()), float(diff.sum() / max(np.abs(ref).sum(), 1e-300))


# Tolerances for bf16-in / fp32-accumulate attention outputs stored as fp32,
# element by element: every |g - r| <= MAX_ABS, and sum|g-r| / sum|r| <= MEAN_REL.
MAX_ABS = 1e-2
MEAN_REL = 2e-3
# Outputs stored as bf16 carry one more rounding, of up to 2^-9 of each
# value (half a bf16 unit in the last place; 1.6e-2 for a value in [4, 8)):
# every element within 1e-2 + 2^-8 |ref|, and sum|g-r|/sum|r| <= 4e-3.
MAX_ABS_BF16 = 1e-2
REL_BF16 = 2.0 ** -8
MEAN_REL_BF16 = 4e-3
# LSE is an fp32 log-sum-exp of the same scores.
LSE_MAX_ABS = 1e-3

# (what, max-abs, mean-rel, bound on max-abs, bound on mean-rel) of every
# comparison made in this process, printed at the end of the pytest run.
RECORDS = []


def assert_close(got, ref, what, max_abs=MAX_ABS, mean_rel=MEAN_REL):
    ma, mr = errors(got, ref)
    RECORDS.append((what, ma, mr, max_abs, mean_rel))
    assert np.isfinite(np.asarray(got, dtype=np.float64)).all(), f"{what}: non-finite values"
    assert ma <= max_abs and mr <= mean_rel, f"{what}: max-abs {ma:.3e} (<= {max_abs}), mean-rel {mr:.3e} (<= {mean_rel})"
    return ma, mr


def assert_close_bf16_storage(got, ref, what, max_abs=MAX_ABS_BF16, rel=REL_BF16, mean_rel=MEAN_REL_BF16):
    """Element by element: |g - r| <= max_abs + rel * |r| (bf16-stored outputs)."""
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    excess = float((np.abs(got - ref) - rel * np.abs(ref)).max())
    _, mr = errors(got, ref)
    RECORDS.append((what + " (max of |g-r| - 2^-8 |r|)", excess, mr, max_abs, mean_rel))
    assert np.isfinite(got).all(), f"{what}: non-finite values"
    assert excess <= max_abs and mr <= mean_rel, \
        f"{what}: max(|g-r| - {rel:g}|r|) {excess:.3e} (<= {max_abs}), mean-rel {mr:.3e} (<= {mean_rel})"
    return excess, mr


def assert_lse_close(got, ref, what, max_abs=LSE_MAX_ABS):
    ma = float(np.abs(np.asarray(got, dtype=np.float64) - np.asarray(ref, dtype=np.float64)).max(initial=0.0))
    RECORDS.append((what, ma, float("nan"), max_abs, float("nan")))
    assert ma <= max_abs, f"{what}: max-abs {ma:.3e} (<= {max_abs})"
    return ma
