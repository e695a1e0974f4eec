"""Pins for the oracle's number-format helpers: binary16 rounding and exact sums.

The oracle builds binary16 from the format definition; these tests pin it against numpy's own
float64 -> float16 conversion (a library routine that rounds directly, ties to even) and against
exact rational arithmetic.
"""
from fractions import Fraction

import numpy as np
import pytest

import oracle as O


def test_f16_table_known_values():
    t = O.f16_table()
    assert t[0x0000] == 0.0
    assert t[0x0001] == 2.0 ** -24            # smallest subnormal
    assert t[0x03FF] == 1023 * 2.0 ** -24     # largest subnormal
    assert t[0x0400] == 2.0 ** -14            # smallest normal
    assert t[0x3C00] == 1.0
    assert t[0x3555] == 0.333251953125
    assert t[0x7BFF] == 65504.0
    assert np.all(np.diff(t) > 0)


def test_f16_bits_to_f64_all_patterns_match_numpy():
    bits = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    ours = O.f16_bits_to_f64(bits)
    ref = bits.view(np.float16).astype(np.float64)
    same = (ours == ref) | (np.isnan(ours) & np.isnan(ref))
    assert same.all()


def _numpy_round(d):
    with np.errstate(over="ignore"):
        return np.asarray(d, np.float64).astype(np.float16).view(np.uint16)


def test_f64_to_f16_random_wide_range_matches_numpy():
    rng = np.random.default_rng(1234)
    d = rng.standard_normal(400_000) * np.exp2(rng.integers(-40, 20, 400_000).astype(np.float64))
    assert np.array_equal(O.f64_to_f16_bits(d), _numpy_round(d))


def test_f64_to_f16_midpoints_and_neighbours():
    t = O.f16_table()
    mids = (t[:-1] + t[1:]) / 2.0               # exact in fp64
    cases = np.concatenate([
        mids, np.nextafter(mids, 0), np.nextafter(mids, np.inf), t,
        [65504.0, 65519.99, 65520.0, 65536.0, 1e6, 2.0 ** -25, np.nextafter(2.0 ** -25, 1),
         2.0 ** -26, 0.0, 1e-300],
    ])
    cases = np.concatenate([cases, -cases])
    assert np.array_equal(O.f64_to_f16_bits(cases), _numpy_round(cases))


def test_f64_to_f16_ties_go_to_even_pattern():
    # 1 + 2^-11 lies halfway between 1.0 (0x3C00, even) and 1 + 2^-10 (0x3C01, odd)
    assert O.f64_to_f16_bits(1.0 + 2.0 ** -11) == 0x3C00
    # 1 + 3*2^-11 lies halfway between 0x3C01 (odd) and 0x3C02 (even)
    assert O.f64_to_f16_bits(1.0 + 3 * 2.0 ** -11) == 0x3C02
    assert O.f64_to_f16_bits(65520.0) == 0x7C00
    assert O.f64_to_f16_bits(0.1) == 0x2E66
    assert O.f64_to_f16_bits(0.7) == 0x399A


def _exact(values):
    return float(sum((Fraction(float(abs(v))) for v in values), Fraction(0)))


def test_exact_abs_sum_beats_naive_order():
    v = [1.0, 2.0 ** -53, 2.0 ** -53]
    naive = 0.0
    for x in v:
        naive += x
    assert naive == 1.0                        # sequential fp64 loses both tiny terms
    assert O.exact_abs_sum(v) == 1.0 + 2.0 ** -52 == _exact(v)


@pytest.mark.parametrize("seed", [0, 1, 2])
def test_exact_abs_sum_matches_fractions(seed):
    rng = np.random.default_rng(seed)
    n = 3000
    w = (rng.standard_normal(n) * np.exp2(rng.integers(-60, 30, n))).astype(np.float32)
    assert O.exact_abs_sum(w) == _exact(w.astype(np.float64))
    w16 = (rng.standard_normal(n) * 0.02).astype(np.float16)
    assert O.exact_abs_sum(w16) == _exact(w16.astype(np.float64))


def test_exact_abs_sum_is_order_independent():
    rng = np.random.default_rng(7)
    w = (rng.standard_normal(5000) * np.exp2(rng.integers(-30, 10, 5000))).astype(np.float32)
    s0 = O.exact_abs_sum(w)
    for _ in range(5):
        assert O.exact_abs_sum(rng.permutation(w)) == s0
