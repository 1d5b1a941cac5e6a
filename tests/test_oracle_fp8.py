"""Pins of the oracle's row-wise E4M3 weight quantiser (CPU only).

The pages name FP8 expert weights ("LatentMoE Explained": an expert is about
22 MB in FP8) but print no recipe; the oracle's recipe is stated in its C
source.  These pins hold it to the E4M3 format's definition: every finite
E4M3 value round-trips, midpoints round to the even mantissa, scales are the
smallest powers of two that bring the row maximum into range, and the error
stays within half a unit in the last place.
"""
import numpy as np

import oracle


def _e4m3_values():
    """All positive finite E4M3 values, from the format's definition."""
    vals = [m / 8 * 2.0 ** -6 for m in range(1, 8)]                     # subnormals
    for e in range(1, 16):
        for m in range(8):
            if e == 15 and m == 7:
                continue                                                 # NaN code
            vals.append(2.0 ** (e - 7) * (1 + m / 8))
    return np.array(sorted(vals))


def test_every_finite_value_round_trips():
    v = _e4m3_values()
    assert len(v) == 126 and v[-1] == 448.0 and v[0] == 2.0 ** -9
    row = np.concatenate([v, -v])[None, :]       # amax 448 -> scale 1
    q, s = oracle.fp8_rows(row)
    assert s[0] == 1.0
    np.testing.assert_array_equal(q, row)


def test_midpoints_round_to_even_mantissa():
    v = _e4m3_values()
    lo, hi = v[:-1], v[1:]
    mid = (lo + hi) / 2
    row = np.concatenate([mid, [448.0]])[None, :]
    q, _ = oracle.fp8_rows(row)
    q = q[0, :-1]
    # the even neighbour: its mantissa index (value / spacing) is even
    def mant_even(x):
        e = np.maximum(np.floor(np.log2(x)), -6)
        return (np.round(x / 2.0 ** (e - 3)) % 2) == 0
    expect = np.where(mant_even(lo), lo, hi)
    np.testing.assert_array_equal(q, expect)


def test_scale_is_the_smallest_power_of_two_in_range():
    rng = np.random.default_rng(0)
    w = rng.standard_normal((64, 96)) * np.exp(rng.uniform(-12, 8, size=(64, 1)))
    w[3] = 0.0
    q, s = oracle.fp8_rows(w)
    amax = np.abs(w).max(axis=1)
    assert s[3] == 1.0 and not np.any(q[3])
    nz = amax > 0
    e = np.log2(s[nz])
    np.testing.assert_array_equal(e, np.round(e))                  # powers of two
    assert np.all(amax[nz] <= 448 * s[nz]) and np.all(amax[nz] > 224 * s[nz])


def test_error_within_half_an_ulp():
    rng = np.random.default_rng(1)
    w = rng.standard_normal((32, 200)) * 0.02
    q, s = oracle.fp8_rows(w)
    x = np.abs(w) / s[:, None]
    ulp = 2.0 ** (np.maximum(np.floor(np.log2(np.maximum(x, 2.0 ** -9))), -6) - 3)
    assert np.all(np.abs(q - w) <= 0.5 * ulp * s[:, None] * (1 + 1e-12))
    # order is kept (rounding is monotonic)
    o = np.argsort(w[0])
    assert np.all(np.diff(q[0][o]) >= 0)


def test_saturation_and_bf16_inputs():
    q, s = oracle.fp8_rows(np.array([[448.0, 460.0, -459.0]]))
    assert s[0] == 2.0
    np.testing.assert_array_equal(q, [[448.0, 448.0, -448.0]])
    # bf16 bit patterns are widened exactly before quantising
    bits = (np.array([1.0, 0.5, -3.0], dtype=np.float32).view(np.uint32) >> 16).astype(np.uint16)
    q, s = oracle.fp8_rows(bits[None, :])
    np.testing.assert_array_equal(q, [[1.0, 0.5, -3.0]])


# ---- the pins above must catch plausible mistakes in the quantiser
import os
import subprocess

import pytest

SRC = os.path.join(os.path.dirname(oracle.__file__), "lmoe_oracle.c")
MUTATIONS = {
    "ties_away_from_zero": ("const double frac = n - k;\n    if (frac > 0.5 || (frac == 0.5 && fmod(k, 2.0) != 0.0)) k += 1.0;",
                            "const double frac = n - k;\n    if (frac >= 0.5) k += 1.0;"),
    "scale_one_step_too_large": ("while (e > -200 && ldexp(448.0, e - 1) >= amax) --e;",
                                 "while (e > -200 && ldexp(448.0, e - 1) >= amax) --e;\n    ++e;"),
    "no_subnormals": ("if (ex < -6) ex = -6;", "if (ex < -6) return 0.0;"),
    "two_mantissa_bits": ("const double q = ldexp(1.0, ex - 3);", "const double q = ldexp(1.0, ex - 2);"),
}
PINS = [test_every_finite_value_round_trips, test_midpoints_round_to_even_mantissa,
        test_scale_is_the_smallest_power_of_two_in_range, test_error_within_half_an_ulp,
        test_saturation_and_bf16_inputs]


@pytest.mark.parametrize("name", sorted(MUTATIONS))
def test_fp8_pins_catch_mutation(name, tmp_path):
    old, new = MUTATIONS[name]
    src = open(SRC).read()
    assert src.count(old) == 1, f"mutation anchor for {name} not unique"
    mutated = tmp_path / "mutant.c"
    mutated.write_text(src.replace(old, new))
    lib = tmp_path / "libmutant.so"
    subprocess.check_call(["gcc", "-std=c11", "-O2", "-fopenmp", "-fPIC", "-shared",
                           "-o", str(lib), str(mutated), "-lm"])
    oracle._swap_library(str(lib))
    try:
        caught = False
        for f in PINS:
            try:
                f()
            except AssertionError:
                caught = True
                break
        assert caught, f"no pin caught mutation {name}"
    finally:
        oracle._swap_library(None)
