"""Pins of the oracle's fused RMS normalization + per-token quantization with
the smoothing scale folded into the norm weight.

"SmoothQuant" explainer, Step 5 ("the inverse scale can be folded into the
normalization layer's weights, so no extra operation is needed at run time")
and Step 6.  Fixed against a closed form (a constant row), an exact power-of-
two invariance, exact rationals with a high-precision square root, and
closeness to the unfused pipeline (norm to bf16, then divide by s and
quantize).
"""

from decimal import Decimal, getcontext
from fractions import Fraction

import numpy as np
import pytest

import oracle
from tests import fp_exact as fx
from w8a8_smoothquant_int8_b200 import workloads as wk


def bf16(a):
    return wk.f32_to_bf16_bits(np.asarray(a, np.float32))


def test_fold_is_rounded_quotient():
    rng = np.random.default_rng(1)
    g = (rng.standard_normal(50) * 0.2 + 1).astype(np.float32)
    s = (rng.random(50) * 5 + 0.1).astype(np.float32)
    gs = oracle.fold_norm_weight(g, s)
    for j in range(50):
        assert fx.frac(gs[j]) == fx.rn32(fx.frac(g[j]) / fx.frac(s[j]))


def test_constant_row_closed_form():
    # h = 3 everywhere, eps = 0: r = RN(1/3), RN(3 r) = 1, so with gamma_s = 1
    # every xt is 1, the scale RN(1/127) and every code 127
    H = bf16(np.full((2, 64), 3.0))
    Xq, xs = oracle.rmsnorm_quant_act(H, np.ones(64, np.float32), 0.0)
    assert (Xq == 127).all()
    assert (xs == np.float32(1.0 / 127.0)).all()


def test_power_of_two_invariance():
    # eps = 0: scaling a row by 2^k scales r by 2^-k exactly, so codes and
    # scales do not change
    rng = np.random.default_rng(2)
    H = bf16(rng.standard_normal((5, 96)) * 3)
    g = (rng.random(96) + 0.5).astype(np.float32)
    Xq, xs = oracle.rmsnorm_quant_act(H, g, 0.0)
    for k in (-7, 3, 12):
        Hk = bf16(wk.bf16_bits_to_f32(H) * np.float32(2.0 ** k))
        Xk, xk = oracle.rmsnorm_quant_act(Hk, g, 0.0)
        assert np.array_equal(Xk, Xq) and np.array_equal(xk, xs)


@pytest.mark.parametrize("seed", [0, 1])
def test_exact_rationals_with_precise_sqrt(seed):
    getcontext().prec = 60
    rng = np.random.default_rng(40 + seed)
    M, K = 3, 12
    H = bf16(rng.standard_normal((M, K)) * rng.choice([1, 1, 20], K))
    g = (rng.random(K) * 2 + 0.1).astype(np.float32)
    eps = np.float32(1e-5)
    Xq, xs = oracle.rmsnorm_quant_act(H, g, eps)
    Hv = wk.bf16_bits_to_f32(H)
    for i in range(M):
        ss = sum(fx.frac(v) ** 2 for v in Hv[i])
        t = ss / K + fx.frac(eps)
        rt = Decimal(1) / (Decimal(t.numerator) / Decimal(t.denominator)).sqrt()
        # r is the fp32 value nearest to 1/sqrt(t): check against its two neighbours
        r = fx.rn32(Fraction(rt))
        xt = [fx.rn32(fx.rn32(fx.frac(Hv[i, j]) * r) * fx.frac(g[j])) for j in range(K)]
        sc = fx.rn32(max(abs(v) for v in xt) / 127)
        assert fx.frac(xs[i]) == sc
        for j in range(K):
            assert Xq[i, j] == max(-128, min(127, fx.rne_int(fx.rn32(xt[j] / sc))))


def test_close_to_the_unfused_pipeline():
    # unfused: X = bf16(RN(RN(h r) gamma)), then xt = RN(X / s) and quantize;
    # fused: xt = RN(RN(h r) * RN(gamma / s)).  Their dequantized values agree
    # to the bf16 rounding of the norm output
    wl = wk.make_workload("parity_ragged")
    H = wl.X
    K = wl.K
    rng = np.random.default_rng(3)
    g = (1 + 0.1 * rng.standard_normal(K)).astype(np.float32)
    P = oracle.Prepared(wl)
    eps = np.float32(1e-6)
    Xq_f, xs_f = oracle.rmsnorm_quant_act(H, oracle.fold_norm_weight(g, P.s), eps)
    Hv = wk.bf16_bits_to_f32(H).astype(np.float64)
    r = (1.0 / np.sqrt((Hv ** 2).sum(1) / K + np.float64(eps))).astype(np.float32)
    xn = (Hv * r[:, None]).astype(np.float32).astype(np.float64) * g.astype(np.float64)
    X = wk.f32_to_bf16_bits(xn.astype(np.float32))
    Xq_u, xs_u = oracle.quant_act(X, P.s)
    fused = Xq_f.astype(np.float64) * xs_f[:, None]
    unfused = Xq_u.astype(np.float64) * xs_u[:, None]
    amax = np.abs(unfused).max(1, keepdims=True)
    assert (np.abs(fused - unfused) <= 2.0 ** -7 * amax + 1.01 * xs_u[:, None]).all()
