"""The two-part f16 form of P used by the products O += P_hi V + P_lo V: hi = P rounded to f16,
lo = (P - hi) rounded to f16, P - hi being exact in f32.  These tests pin the error bound the
design relies on (round to nearest, as the hardware conversion does) over the whole range the
lazy max allows, P in [0, 256]."""
import numpy as np


def _split(p32):
    hi = p32.astype(np.float16)
    d = p32 - hi.astype(np.float32)              # exact: hi is p to 11 bits
    lo = d.astype(np.float16)
    return hi, lo


def test_difference_is_exact_in_f32():
    rng = np.random.default_rng(1)
    p = (rng.random(200000) * 256.0).astype(np.float32)
    hi = p.astype(np.float16)
    d32 = p - hi.astype(np.float32)
    d64 = p.astype(np.float64) - hi.astype(np.float64)
    assert np.array_equal(d32.astype(np.float64), d64)


def test_error_bound_over_the_range():
    rng = np.random.default_rng(2)
    # log-uniform over [2^-40, 256] plus uniform over [0, 256]
    p = np.concatenate([np.exp2(rng.uniform(-40.0, 8.0, 300000)), rng.random(300000) * 256.0])
    p = p.astype(np.float32)
    hi, lo = _split(p)
    err = np.abs(p.astype(np.float64) - hi.astype(np.float64) - lo.astype(np.float64))
    bound = np.maximum(np.exp2(-22.0) * p.astype(np.float64), np.exp2(-25.0))
    assert np.all(err <= bound)


def test_about_22_bits_where_both_parts_are_normal():
    rng = np.random.default_rng(3)
    p = np.exp2(rng.uniform(-3.0, 8.0, 200000)).astype(np.float32)
    hi, lo = _split(p)
    rel = np.abs(p.astype(np.float64) - hi.astype(np.float64) - lo.astype(np.float64)) / p
    assert rel.max() <= np.exp2(-21.0)
    assert np.median(rel) < np.exp2(-23.0)


def test_one_f16_part_alone_is_far_coarser():
    rng = np.random.default_rng(4)
    p = np.exp2(rng.uniform(-3.0, 8.0, 100000)).astype(np.float32)
    hi, _ = _split(p)
    rel = np.abs(p.astype(np.float64) - hi.astype(np.float64)) / p
    assert rel.max() > np.exp2(-12.5)     # the single part keeps 11 bits only
