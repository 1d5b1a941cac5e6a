"""Pins of the oracle's row-wise NVFP4 quantiser (CPU only).

The pages say the shipped models were pretrained in NVFP4 ("LatentMoE
Explained", the Nemotron 3 Super paragraph) and give no recipe; the format
is NVIDIA's published one: E2M1 elements, an E4M3 scale per 16 elements, a
second-level scale (taken per row here, a power of two).  These pins hold
the oracle to the format's definition: every E2M1 value round-trips, ties
go to the even mantissa, block scales are the E4M3 rounding of the block
maximum over 6 s_r, elements are scaled by the single-precision reciprocal
of their decoded block scale, row scales are the smallest powers of two that
keep every block scale in E4M3's range, and the error stays within half a
grid step.
"""
import os
import subprocess

import numpy as np
import pytest

import oracle

E2M1 = np.array([0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0])   # from the format's definition


def _e2m1_values():
    """The positive E2M1 magnitudes from the encoding: subnormal 0.5 (E = 0,
    M = 1), normals 2^(E-1) (1 + M/2) for E = 1..3."""
    vals = {0.0, 0.5}
    for e in range(1, 4):
        for m in range(2):
            vals.add(2.0 ** (e - 1) * (1 + m / 2))
    return np.array(sorted(vals))


def _row(*blocks):
    return np.concatenate([np.asarray(b, dtype=np.float64) for b in blocks])[None, :]


ANCHOR = [2688.0] + [0.0] * 15     # a block with amax 6 * 448: row scale 1, block scale 448


def test_the_value_set_is_the_formats():
    v = _e2m1_values()
    np.testing.assert_array_equal(v, E2M1)


def test_every_e2m1_value_round_trips():
    v = _e2m1_values()
    row = _row(ANCHOR, list(v) + list(-v))          # block amax 6 -> block scale 1
    q, s, b = oracle.nvfp4_rows(row)
    assert s[0] == 1.0
    np.testing.assert_array_equal(b[0], [448.0, 1.0])
    np.testing.assert_array_equal(q, row)
    # the same values times an E4M3 block scale and a power-of-two row scale
    row2 = _row(np.array(ANCHOR) * 2.0 ** -5, list(0.625 * 2.0 ** -5 * v) + list(-0.625 * 2.0 ** -5 * v))
    q2, s2, b2 = oracle.nvfp4_rows(row2)
    assert s2[0] == 2.0 ** -5 and b2[0, 1] == 0.625
    np.testing.assert_array_equal(q2, row2)


def test_ties_round_to_the_even_mantissa():
    mids = [0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0]
    expect = [0.0, 1.0, 1.0, 2.0, 2.0, 4.0, 4.0]     # the neighbour with mantissa bit 0
    blk = mids + [6.0] + [-m for m in mids] + [5.5]
    q, _, b = oracle.nvfp4_rows(_row(ANCHOR, blk))
    assert b[0, 1] == 1.0
    np.testing.assert_array_equal(q[0, 16:], expect + [6.0] + [-e for e in expect] + [6.0])


def test_block_scale_is_the_e4m3_rounding_of_amax_over_6_sr():
    # t = amax / 6: 1.0625 lies halfway between 1 and 1.125 -> even mantissa 1;
    # 1.1 -> 1.125; 0.01 -> a subnormal E4M3 step (2^-9 multiples): 5 * 2^-9;
    # 1.4 * 2^-9 -> 2^-9, far enough below t that the block maximum saturates
    cases = [(6 * 1.0625, 1.0), (6 * 1.1, 1.125), (6 * 0.01, 5 * 2.0 ** -9), (6 * 448.0, 448.0),
             (6 * 1.4 * 2.0 ** -9, 2.0 ** -9)]
    row = _row(*[[a] + [0.0] * 15 for a, _ in cases])
    q, s, b = oracle.nvfp4_rows(row)
    assert s[0] == 1.0
    np.testing.assert_array_equal(b[0], [e for _, e in cases])
    # block maxima: 6.375 / 1 saturates to 6; 6.6 / 1.125 = 5.87 rounds to 6;
    # 0.06 / (5 * 2^-9) = 6.14 saturates; 2688 / 448 = 6 exactly; 8.4 saturates
    np.testing.assert_array_equal(q[0, ::16], [6.0, 6.0 * 1.125, 6.0 * 5 * 2.0 ** -9, 2688.0,
                                               6.0 * 2.0 ** -9])


def test_elements_are_scaled_by_the_rounded_reciprocal_of_the_block_scale():
    """code = E2M1(x * RN(1 / (b s_r))), not E2M1(x / (b s_r)): with b = 1.875
    (block maximum 11.25) the elements 2.34375 = 1.25 * 1.875 and 4.6875 =
    2.5 * 1.875 divide to the ties 1.25 and 2.5 exactly (which go to the even
    1 and 2), but 1 / 1.875 = 8/15 rounds up in single precision, so the
    products lie just above the ties and round to 1.5 and 3."""
    from fractions import Fraction
    assert Fraction(float(np.float32(1) / np.float32(1.875))) > Fraction(8, 15)
    q, s, b = oracle.nvfp4_rows(_row(ANCHOR, [11.25, 2.34375, 4.6875, -2.34375] + [0.0] * 12))
    assert s[0] == 1.0 and b[0, 1] == 1.875
    np.testing.assert_array_equal(q[0, 16:20], np.array([6.0, 1.5, 3.0, -1.5]) * 1.875)


def test_row_scale_is_the_smallest_power_of_two_in_range():
    rng = np.random.default_rng(0)
    w = rng.standard_normal((64, 96)) * np.exp(rng.uniform(-12, 8, size=(64, 1)))
    w[3] = 0.0
    q, s, b = oracle.nvfp4_rows(w)
    amax = np.abs(w).max(axis=1)
    assert s[3] == 1.0 and not np.any(q[3]) and not np.any(b[3])
    nz = amax > 0
    e = np.log2(s[nz])
    np.testing.assert_array_equal(e, np.round(e))
    assert np.all(amax[nz] <= 2688 * s[nz]) and np.all(amax[nz] > 1344 * s[nz])
    assert np.all(b <= 448.0)


def test_values_lie_on_the_grid_and_within_half_a_step():
    rng = np.random.default_rng(1)
    w = (rng.standard_normal((32, 256)) * 0.02).astype(np.float32)
    q, s, b = oracle.nvfp4_rows(w)
    scale = np.repeat(b, 16, axis=1) * s[:, None]            # b_j s_r per element
    nz = scale > 0
    y = np.abs(q[nz]) / scale[nz]
    assert np.all(np.isin(y, E2M1))
    x = np.abs(w.astype(np.float64)[nz]) / scale[nz]
    half = np.where(x < 2, 0.25, np.where(x < 4, 0.5, 1.0))
    sat = x > 6
    err = np.abs(np.abs(q[nz]) / scale[nz] - x)
    assert np.all(err[~sat] <= half[~sat] * (1 + 1e-6))
    # saturation only by the block scale's rounding: amax / (b s_r) <= 6 (1 + 2^-4)
    assert np.all(x[sat] <= 6.0 * (1 + 2.0 ** -4))
    for j in range(16):                                       # monotonic within a block
        blk = slice(16 * j, 16 * j + 16)
        o = np.argsort(w[0, blk])
        assert np.all(np.diff(q[0, blk][o]) >= 0)


def test_zero_blocks_and_bf16_inputs():
    q, s, b = oracle.nvfp4_rows(_row(ANCHOR, [0.0] * 16))
    assert b[0, 1] == 0.0 and not np.any(q[0, 16:])
    bits = (np.array([2688.0] + [0.0] * 15 + [1.0, 0.5, -3.0] + [0.0] * 13,
                     dtype=np.float32).view(np.uint32) >> 16).astype(np.uint16)
    q, s, b = oracle.nvfp4_rows(bits[None, :])
    np.testing.assert_array_equal(q[0, 16:19], [1.0, 0.5, -3.0])
    with pytest.raises(ValueError):
        oracle.nvfp4_rows(np.ones((2, 24)))


# ---- the pins above must catch plausible mistakes in the quantiser
SRC = os.path.join(os.path.dirname(oracle.__file__), "lmoe_oracle.c")
MUTATIONS = {
    "ties_away_from_zero": ("    /* an even k is an even mantissa on every segment of the grid */\n"
                            "    if (frac > 0.5 || (frac == 0.5 && fmod(k, 2.0) != 0.0)) k += 1.0;",
                            "    if (frac >= 0.5) k += 1.0;"),
    "blocks_of_32": ("  for (int j = 0; j < n / 16; ++j) {\n    float am = 0.0f;\n    for (int i = 16 * j; i < 16 * j + 16; ++i)",
                     "  for (int j = 0; j < n / 16; ++j) {\n    float am = 0.0f;\n    for (int i = 32 * (j / 2); i < 32 * (j / 2) + 32; ++i)"),
    "row_scale_for_e4m3_only": ("    while (e > -200 && ldexp(2688.0, e - 1) >= amax) --e;",
                                "    while (e > -200 && ldexp(2688.0, e - 1) >= amax) --e;\n    e -= 2;"),
    "block_scale_not_rounded": ("    const double b = e4m3_round((double)t);", "    const double b = (double)t;"),
    "uniform_grid": ("    const double q = a < 2.0 ? 0.5 : (a < 4.0 ? 1.0 : 2.0);",
                     "    const double q = 0.5;"),
    "division_instead_of_reciprocal": ("      const float y = x[i] * rcp;",
                                       "      const float y = x[i] / den;"),
    "no_saturation": ("  if (a >= 6.0) {\n    r = 6.0;\n  } else {",
                      "  if (a >= 60.0) {\n    r = 6.0;\n  } else {"),
}
PINS = [test_every_e2m1_value_round_trips, test_ties_round_to_the_even_mantissa,
        test_block_scale_is_the_e4m3_rounding_of_amax_over_6_sr,
        test_elements_are_scaled_by_the_rounded_reciprocal_of_the_block_scale,
        test_row_scale_is_the_smallest_power_of_two_in_range,
        test_values_lie_on_the_grid_and_within_half_a_step, test_zero_blocks_and_bf16_inputs]


@pytest.mark.parametrize("name", sorted(MUTATIONS))
def test_nvfp4_pins_catch_mutation(name, tmp_path):
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
            except (AssertionError, ValueError):
                caught = True
                break
        assert caught, f"no pin caught mutation {name}"
    finally:
        oracle._swap_library(None)
