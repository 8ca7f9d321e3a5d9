"""The two-part E4M3 split of bf16 Q values is exact where the attention kernel relies on it.

The attention kernel computes S = Q K^T on FP8 tensor cores without rounding Q: each Q row is
scaled by a power of two 2^s that brings its largest magnitude into [128, 256), and every
scaled value q' is written as q1 + q2 with q1 = E4M3(q') and q2 = E4M3(q' - q1), both rounded
to nearest even.  An 8-bit bf16 significand is a 4-bit E4M3 significand plus a remainder of
at most 8 units of its last place, so the split is exact for every q' >= 2^-2 (the remainder
stays a multiple of 2^-9, the E4M3 subnormal quantum); below that the error is at most
2^-10.  This checks the claim on every bf16 value of the scaled range, with E4M3 rounding
taken from ml_dtypes (not from the kernel or the oracle).
"""
import ml_dtypes
import numpy as np


def _all_bf16_in(lo: float, hi: float) -> np.ndarray:
    bits = np.arange(0, 0x8000, dtype=np.uint32)  # every non-negative bf16 pattern
    vals = (bits << 16).view(np.float32)
    keep = np.isfinite(vals) & (vals >= lo) & (vals < hi)
    v = vals[keep]
    return np.concatenate([v, -v])


def _split(q: np.ndarray):
    q1 = q.astype(ml_dtypes.float8_e4m3fn).astype(np.float32)
    r = (q - q1).astype(np.float32)  # exact in fp32: q and q1 agree in all high bits
    q2 = r.astype(ml_dtypes.float8_e4m3fn).astype(np.float32)
    return q1, q2


def test_split_is_exact_above_quarter():
    q = _all_bf16_in(0.25, 256.0)
    q1, q2 = _split(q)
    assert np.all(np.isfinite(q1)) and np.all(np.isfinite(q2))
    assert np.array_equal((q1.astype(np.float64) + q2.astype(np.float64)), q.astype(np.float64))


def test_split_error_bound_below_quarter():
    q = _all_bf16_in(2.0 ** -30, 0.25)
    q1, q2 = _split(q)
    err = np.abs(q1.astype(np.float64) + q2.astype(np.float64) - q.astype(np.float64))
    assert err.max() <= 2.0 ** -10


def test_scale_exponent_brings_row_max_into_range():
    # s = 134 - E(max) for the largest bf16 exponent field E of the row
    rng = np.random.default_rng(3)
    for _ in range(2000):
        row = rng.standard_normal(128).astype(np.float32) * np.float32(2.0 ** rng.integers(-60, 60))
        row = row.astype(ml_dtypes.bfloat16).astype(np.float32)
        e = int(((row.view(np.uint32) >> 23) & 0xFF).max())
        s = min(max(134 - e, -126), 126)
        m = np.abs(row).max() * np.float32(2.0 ** s)
        assert 128.0 <= m < 256.0
