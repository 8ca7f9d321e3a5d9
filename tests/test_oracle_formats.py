"""Pins of the oracle's number formats against independent definitions.

FP8 E4M3 KV is used throughout the method ("PageWeaver: KV-Guided Query Unions for Sparse
Attention", Abstract).  Q and O are bf16.  Each oracle routine is checked here against
library implementations (ml_dtypes, torch) and exact rational arithmetic, never against
itself.
"""
import json
import os
from fractions import Fraction

import ml_dtypes
import numpy as np
import pytest
import torch

from oracle import oracle

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def test_e4m3_all_codes_match_two_libraries():
    codes = np.arange(256, dtype=np.uint8)
    ours = oracle.e4m3_to_f64(codes)
    via_ml = codes.view(ml_dtypes.float8_e4m3fn).astype(np.float64)
    via_torch = torch.from_numpy(codes).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    assert np.array_equal(ours, via_ml, equal_nan=True)
    assert np.array_equal(ours, via_torch, equal_nan=True)


def test_e4m3_golden_codes():
    # Values fixed by the E4M3 bit layout (bias 7, 3 mantissa bits, S.1111.111 = NaN).
    with open(os.path.join(GOLDEN, "e4m3_codes.json")) as f:
        g = json.load(f)
    for item in g["codes"]:
        v = oracle.e4m3_to_f64(np.array([item["code"]], np.uint8))[0]
        if item["value"] == "nan":
            assert np.isnan(v)
        else:
            assert v == float(Fraction(item["value"])), item


def test_bf16_to_f64_matches_ml_dtypes():
    rng = np.random.default_rng(1)
    bits = rng.integers(0, 1 << 16, size=4096, dtype=np.uint32).astype(np.uint16)
    bits = np.concatenate([bits, np.array([0, 0x8000, 0x0001, 0x7F7F, 0xFF7F, 0x3F80, 0x7F80],
                                          np.uint16)])
    ours = oracle.bf16_to_f64(bits)
    ref = bits.view(ml_dtypes.bfloat16).astype(np.float64)
    assert np.array_equal(ours, ref, equal_nan=True)


def _nearest_even_bf16(x: float) -> float:
    """Exact RNE to 8 significant bits with Fraction arithmetic (finite, in bf16 range)."""
    fx = Fraction(x)
    if fx == 0:
        return 0.0
    sign = -1 if fx < 0 else 1
    a = abs(fx)
    e = 0
    while a >= 2:
        a /= 2
        e += 1
    while a < 1:
        a *= 2
        e -= 1
    q = Fraction(2) ** max(e - 7, -133)
    n = abs(fx) / q
    fl = n.numerator // n.denominator
    rem = n - fl
    if rem > Fraction(1, 2) or (rem == Fraction(1, 2) and fl % 2 == 1):
        fl += 1
    return float(sign * fl * q)


def test_f64_to_bf16_exact_rounding():
    rng = np.random.default_rng(2)
    x = rng.standard_normal(3000) * np.exp(rng.uniform(-80, 80, 3000))
    ours = oracle.f64_to_bf16(x).view(ml_dtypes.bfloat16).astype(np.float64)
    ref = np.array([_nearest_even_bf16(v) for v in x])
    assert np.array_equal(ours, ref)


def test_f64_to_bf16_agrees_with_library_on_binary32_inputs():
    # For binary32-exact inputs the library's single rounding is the correct one.
    rng = np.random.default_rng(3)
    x = (rng.standard_normal(20000) * np.exp(rng.uniform(-40, 40, 20000))).astype(np.float32)
    ours = oracle.f64_to_bf16(x.astype(np.float64))
    ref = x.astype(ml_dtypes.bfloat16).view(np.uint16)
    assert np.array_equal(ours, ref)


def test_f64_to_bf16_golden_ties_and_edges():
    with open(os.path.join(GOLDEN, "bf16_rounding.json")) as f:
        g = json.load(f)
    for item in g["cases"]:
        x = float(Fraction(item["x"])) if item["x"] not in ("inf", "-inf") else float(item["x"])
        got = int(oracle.f64_to_bf16(np.array([x]))[0])
        assert got == int(item["bits"], 16), item
