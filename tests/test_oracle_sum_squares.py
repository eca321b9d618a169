"""Pins of the oracle's sum of squares for the fused RMS normalization.

The norm factor r_i = RN32(1/sqrt(sum_j h_ij^2 / K + eps)) of the RMS norm in
front of the layer ("SmoothQuant" explainer, Step 5: the inverse scale folded
into the normalization layer's weights) needs the sum of the squares of a
bf16 row.  The oracle defines it as the exact sum, rounded once to fp64 (no
order of summation), which these tests fix against Python's correctly
rounded math.fsum, against exact rationals (Fraction -> float is correctly
rounded), and against hand-built ties and sticky bits.
"""

import math
from fractions import Fraction

import numpy as np
import pytest

import oracle
from w8a8_smoothquant_int8_b200 import workloads as wk


def bits(vals):
    return wk.f32_to_bf16_bits(np.asarray(vals, np.float32))


def exact(h):
    return float(sum(Fraction(float(v)) ** 2 for v in wk.bf16_bits_to_f32(h)))


def rows():
    rng = np.random.default_rng(11)
    out = []
    out.append(bits(rng.standard_normal(4096)))                                  # N(0,1)
    out.append(bits(rng.standard_normal(1000) * np.exp(rng.standard_normal(1000) * 8)))
    # squares spanning the whole normal range of bf16 (2^-126 .. 2^120)
    e = rng.integers(-126, 121, 600)
    out.append(bits(rng.choice([-1.0, 1.0], 600) * (1 + rng.random(600)) * 2.0 ** e))
    # subnormal bf16 values (exponent field 0) with normal ones
    sub = (rng.integers(1, 128, 50).astype(np.uint16))
    out.append(np.concatenate([sub, bits(rng.standard_normal(30) * 1e-30)]))
    out.append(bits(np.zeros(17)))
    return out


def test_matches_fsum_and_exact_rationals():
    for h in rows():
        got = oracle.sum_squares_bf16(h)
        v = wk.bf16_bits_to_f32(h).astype(np.float64)
        assert got == math.fsum(v * v)  # the squares of bf16 values are exact in fp64
        assert got == exact(h)


def test_order_does_not_matter():
    rng = np.random.default_rng(12)
    h = rows()[2]
    ref = oracle.sum_squares_bf16(h)
    for _ in range(5):
        assert oracle.sum_squares_bf16(h[rng.permutation(len(h))]) == ref


def test_ties_round_to_even_and_sticky_bits():
    # 2^60 + 2^7 is halfway between 2^60 and 2^60 + 2^8 (the fp64 step at
    # 2^60): ties to even gives 2^60; any further positive term, however
    # small, moves it up to 2^60 + 2^8
    big = [2.0 ** 30]                     # square 2^60
    half = [2.0 ** 3, 2.0 ** 3]           # squares 2^6 + 2^6 = 2^7
    assert oracle.sum_squares_bf16(bits(big + half)) == 2.0 ** 60
    assert oracle.sum_squares_bf16(bits(big + half + [2.0 ** -60])) == 2.0 ** 60 + 2.0 ** 8
    # odd significand: 2^60 + 2^8 + 2^7 is a tie between 2^60 + 2^8 (odd) and
    # 2^60 + 2^9 (even): it goes up
    assert oracle.sum_squares_bf16(bits(big + [2.0 ** 4] + half)) == 2.0 ** 60 + 2.0 ** 9
    # just below the tie (2^7 - 2^-2): down
    below = big + [2.0 ** 3, np.float32(math.sqrt(2.0 ** 6 - 2.0 ** -2))]
    v = wk.bf16_bits_to_f32(bits(below)).astype(np.float64)
    assert math.fsum(v * v) == 2.0 ** 60
    assert oracle.sum_squares_bf16(bits(below)) == 2.0 ** 60


def test_an_ordered_fp64_sum_is_not_this_definition():
    # 2^20 followed by seven squares of 2^-34 (each below half a step of
    # 2^20) loses them all when summed in order; the exact sum keeps their
    # 1.75 * 2^-32 and rounds to 2^20 + 2^-31
    h = bits([2.0 ** 10] + [2.0 ** -17] * 7)
    v = wk.bf16_bits_to_f32(h).astype(np.float64)
    ordered = 0.0
    for x in v:
        ordered += x * x
    assert ordered == 2.0 ** 20
    assert oracle.sum_squares_bf16(h) == 2.0 ** 20 + 2.0 ** -31


def test_extremes():
    # the smallest square (2^-133)^2 = 2^-266 and the largest finite bf16
    assert oracle.sum_squares_bf16(np.array([1], np.uint16)) == 2.0 ** -266
    top = np.array([0x7F7F], np.uint16)  # (2 - 2^-7) * 2^127
    assert oracle.sum_squares_bf16(top) == exact(top)
    assert oracle.sum_squares_bf16(np.repeat(top, 1000)) == exact(np.repeat(top, 1000))
    inf = np.array([bits([1.0])[0], 0x7F80], np.uint16)
    assert oracle.sum_squares_bf16(inf) == math.inf


@pytest.mark.parametrize("seed", [0, 1, 2])
def test_random_widths(seed):
    rng = np.random.default_rng(100 + seed)
    for K in (1, 2, 15, 256, 4099):
        h = bits(rng.standard_normal(K) * 2.0 ** rng.integers(-60, 60, K))
        assert oracle.sum_squares_bf16(h) == exact(h)
