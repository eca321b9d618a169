"""Host checks of the two arithmetic shortcuts of the streaming quantizers.

The per-token code is defined ("SmoothQuant" explainer, Step 6, with the
smoothing division of Step 2) as
    xt = RN32(x / s),   code = clamp(rne(RN32(xt / x_scale)), -128, 127),
and the CUDA kernels reach it without IEEE divisions on the common path:

1. xt by Markstein's correction from y = RN32(1/s):
       q = RN(x*y);  twice: r = RN(x - s*q) (fused),  q = RN(q + r*y) (fused),
   claimed equal to RN32(x/s) whenever |x| >= 2^-100 and the quotient lies in
   [2^-100, 2^120) (s in [2^-17, 2^100]).
2. the code from one fused multiply-add with 1.5*2^23 and a faithful inv of
   1/x_scale (one Newton step from the hardware reciprocal):
       big = RN(xt*inv + 1.5*2^23),  c = big - 1.5*2^23,
       d = RN(xt*inv - c)  (fused; exact),
   kept only when |d| <= 1/2 - 2^-13, else recomputed from the exact
   quotient; claimed to equal rne(RN32(xt/x_scale)) whenever it is kept.

Every fp32 operation is replayed exactly (one round-to-nearest-even of the
exact rational value per operation), on random operands and on operands
built next to rounding boundaries.
"""

import random
from fractions import Fraction as F

import numpy as np

from tests import fp_exact as fx

MAGIC = F(12582912)  # 1.5 * 2^23


def f32(v: float) -> F:
    return F(float(np.float32(v)))


def markstein(x: F, s: F) -> F:
    y = fx.rn32(1 / s)
    q = fx.rn32(x * y)
    for _ in range(2):
        r = fx.rn32(x - s * q)
        q = fx.rn32(q + r * y)
    return q


def neighbours(v: F, n: int):
    """v and the n float32 values on each side of it."""
    f = np.float32(float(v))
    out = [f]
    up = down = f
    for _ in range(n):
        up = np.nextafter(up, np.float32(np.inf))
        down = np.nextafter(down, np.float32(-np.inf))
        out += [up, down]
    return [F(float(a)) for a in out]


def test_markstein_quotient_is_the_ieee_quotient():
    rng = random.Random(5)
    for _ in range(3000):
        s = f32(2.0 ** rng.uniform(-17, 30) * rng.uniform(1, 2))
        # bf16 and f32 activations, including values whose quotient by s
        # sits next to a point halfway between two floats
        x = f32(rng.gauss(0, 1) * 2.0 ** rng.uniform(-20, 20))
        xb = fx.rn_bf16(x)
        for xv in (x, xb):
            if xv == 0:
                continue
            assert markstein(xv, s) == fx.rn32(xv / s), (xv, s)
        q = fx.rn32(x / s)
        mid = q + (fx.rn32(q * (1 + F(1, 2 ** 23))) - q) / 2  # toward the next float up
        for xv in neighbours(fx.rn32(mid * s), 2):
            if xv != 0:
                assert markstein(xv, s) == fx.rn32(xv / s), (xv, s)


def faithful_pair(scale: F):
    """The two floats bracketing 1/scale (both are faithful reciprocals)."""
    r = fx.rn32(1 / scale)
    f = np.float32(float(r))
    lo = f if r <= 1 / scale else np.nextafter(f, np.float32(0))
    hi = np.nextafter(lo, np.float32(np.inf))
    return F(float(lo)), F(float(hi))


def fast_code(xt: F, inv: F):
    big = fx.rn32(xt * inv + MAGIC)
    c = big - MAGIC
    d = fx.rn32(xt * inv - c)
    return int(c), d


def test_code_from_one_fused_multiply_add():
    rng = random.Random(11)
    kept = {"random": 0, "near tie": 0, "threshold": 0}
    redone = {"random": 0, "near tie": 0, "threshold": 0}
    for _ in range(1500):
        amax = f32(2.0 ** rng.uniform(-40, 40) * rng.uniform(1, 2))
        scale = fx.rn32(amax / 127)
        pts = [("random", f32(float(amax) * rng.uniform(-1, 1))) for _ in range(4)]
        # values whose quotient by the scale sits next to a half-integer
        k = rng.randrange(-127, 127)
        pts += [("near tie", v) for v in neighbours(fx.rn32((k + F(1, 2)) * scale), 3)]
        # and next to the threshold of the tie test, 2^-13 from the tie
        for off in (F(1, 2 ** 12), F(1, 2 ** 13) + F(1, 2 ** 15), F(1, 2 ** 13) - F(1, 2 ** 15)):
            for sg in (1, -1):
                pts.append(("threshold", fx.rn32((k + F(1, 2) + sg * off) * scale)))
        for kind, xt in pts:
            if abs(xt) > amax:
                continue
            want = fx.rne_int(fx.rn32(xt / scale))
            for inv in faithful_pair(scale):
                c, d = fast_code(xt, inv)
                if abs(d) <= F(1, 2) - F(1, 2 ** 13):
                    assert c == want, (xt, scale, inv, c, want)
                    kept[kind] += 1
                else:
                    redone[kind] += 1
    # random values almost always keep the fast code, values a few ulps from a
    # tie take the exact quotient, and both outcomes occur at the threshold
    assert kept["random"] > 100 * redone["random"]
    assert redone["near tie"] > 0 and kept["near tie"] == 0
    assert redone["threshold"] > 0 and kept["threshold"] > 0
