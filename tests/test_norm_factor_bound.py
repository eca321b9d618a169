"""Error bound of the fused norm kernel's fast reciprocal square root.

The streaming norm kernel computes r_i = RN32(RN64(1 / RN64(sqrt(t)))) (the
oracle's definition: RMS norm with correctly rounded fp64 square root and
division, "SmoothQuant" explainer Step 5 with the norm in front of the layer)
without a division: two steps of Newton's iteration for 1/sqrt(t),
    e = RN(1 - RN(t*y)*y),   y <- RN(y + RN(y/2)*e),
from the single-precision estimate y0 (hardware rsqrt, relative error below
2^-22 after widening t to fp32), then RN32(y), unless y lies within 2^-46
(relative) of a point halfway between two floats, where it takes the
correctly rounded square root and division.

This host test replays that sequence of rounded fp64 operations exactly
(every fused multiply-add rounded once from its exact rational value) and
checks the two facts the kernel relies on:
  1. |y - 1/sqrt(t)| < 2^-51.5 / sqrt(t) for estimates at the error bound;
  2. RN32(y) equals RN32 of the double-rounded value whenever y is not within
     2^-46 of a midpoint, including for t built to sit next to midpoints.
"""

import math
import random
from fractions import Fraction as F

import numpy as np


def rd(x: F) -> float:
    """Round an exact rational to the nearest double (ties to even):
    int / int true division in Python is correctly rounded."""
    return x.numerator / x.denominator


def newton_two_steps(t: float, y0: float) -> float:
    y = y0
    for _ in range(2):
        u = rd(F(t) * F(y))               # RN(t*y)
        e = rd(1 - F(u) * F(y))           # fma(-u, y, 1)
        h = rd(F(1, 2) * F(y))            # y/2, exact
        y = rd(F(h) * F(e) + F(y))        # fma(h, e, y)
    return y


def rel_err_sq(y: float, t: float) -> float:
    """|y*sqrt(t) - 1| from the exact value of y^2 t - 1 (to first order)."""
    return abs(float(F(y) ** 2 * F(t) - 1)) / 2


def f32_rn(x: float) -> np.float32:
    return np.float32(x)


def midpoint_distance(y: float) -> float:
    """Relative distance of y > 0 from the point halfway between the float
    below-or-at y and the next float up (the kernel's check)."""
    f = np.float32(y)
    if float(f) > y:  # the float at or below y
        f = np.nextafter(f, np.float32(0))
    fn = np.nextafter(f, np.float32(np.inf))
    mid = (F(float(f)) + F(float(fn))) / 2
    return abs(float((F(y) - mid) / F(y)))


def estimate(t: float, delta: float) -> float:
    # the single-precision estimate: 1/sqrt of t rounded to fp32, off by delta
    t32 = float(np.float32(t))
    return float(np.float32(1.0 / math.sqrt(t32) * (1.0 + delta)))


def test_newton_error_bound_across_the_fast_range():
    rng = random.Random(1234)
    worst = 0.0
    for _ in range(4000):
        t = 2.0 ** rng.uniform(-100, 100) * rng.uniform(1, 2)
        for delta in (2.0 ** -22, -(2.0 ** -22), rng.uniform(-1, 1) * 2.0 ** -22):
            y = newton_two_steps(t, estimate(t, delta))
            worst = max(worst, rel_err_sq(y, t))
    assert worst < 2.0 ** -51.5, math.log2(worst)
    # one step is not enough (the bound is not vacuous): ~2^-43 from 2^-22
    y0 = estimate(3.0, 2.0 ** -22)
    u = rd(F(3.0) * F(y0))
    y1 = rd(F(rd(F(1, 2) * F(y0))) * F(rd(1 - F(u) * F(y0))) + F(y0))
    assert rel_err_sq(y1, 3.0) > 2.0 ** -48


def _check_agreement(t: float, delta: float) -> bool:
    """True when the fast path is taken; asserts it gives the oracle's float."""
    y = newton_two_steps(t, estimate(t, delta))
    if midpoint_distance(y) <= 2.0 ** -46:
        return False  # the kernel takes the correctly rounded path
    z = 1.0 / math.sqrt(t)  # RN64(1 / RN64(sqrt(t))): both IEEE operations
    assert f32_rn(y) == f32_rn(z), (t, y, z)
    return True


def test_fast_path_agrees_with_the_double_rounded_value():
    rng = random.Random(99)
    fast = 0
    for _ in range(6000):
        t = 2.0 ** rng.uniform(-100, 100) * rng.uniform(1, 2)
        fast += _check_agreement(t, rng.uniform(-1, 1) * 2.0 ** -22)
    assert fast > 5900  # near-midpoint cases are rare


def test_fast_path_next_to_float_midpoints():
    # t = 1/m^2 rounded to a double, for m halfway between two floats (and
    # nudged by 2^-60 .. 2^-40): 1/sqrt(t) sits at or next to the midpoint.
    # Wherever the kernel would keep the Newton result it must agree with the
    # oracle; within 2^-46 it must leave the fast path.
    rng = random.Random(7)
    taken = skipped = 0
    for _ in range(600):
        f = np.float32(rng.uniform(0.01, 100.0))
        fn = np.nextafter(f, np.float32(np.inf))
        mid = (F(float(f)) + F(float(fn))) / 2
        for k in (None, -60, -52, -48, -46, -45, -44, -40):
            for sign in (1, -1):
                m = mid if k is None else mid * (1 + sign * F(2) ** k)
                t = rd(1 / (m * m))
                for delta in (2.0 ** -22, -(2.0 ** -22)):
                    if _check_agreement(t, delta):
                        taken += 1
                    else:
                        skipped += 1
    assert taken > 0 and skipped > 0
