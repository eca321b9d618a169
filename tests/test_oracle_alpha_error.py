"""Pins of the oracle's layer-wise output error for one alpha.

"SmoothQuant" explainer, "Reading the diagnostics" (compare layer-wise output
error across alpha values) and "Variants and related ideas" (per-layer alpha
by calibration error).  Fixed against a case that quantizes exactly (error 0),
exact rationals on the worked example's layer, and the error's definition on
a brute-forced tiny layer.
"""

from fractions import Fraction

import numpy as np
import pytest

import oracle
from tests import fp_exact as fx
from w8a8_smoothquant_int8_b200 import workloads as wk


def bf16(a):
    return wk.f32_to_bf16_bits(np.asarray(a, np.float32))


def test_zero_error_when_every_value_is_a_code():
    # X and W take values c * 2^-6 with |c| <= 127 integers and every channel
    # maximum is 127 * 2^-6 in both, so at alpha = 0.5 the smoothing scale is
    # 1, every scale is exactly 2^-6 and every code is c: Y = X W^T exactly
    M, K, N = 4, 16, 8
    rng = np.random.default_rng(4)
    cx = rng.integers(-127, 128, (M, K))
    cx[:, 0] = 127
    cx[0, :] = 127
    cw = rng.integers(-127, 128, (N, K))
    cw[:, 0] = 127
    cw[0, :] = 127
    X = (cx * 2.0 ** -6).astype(np.float32)
    W = bf16(cw * 2.0 ** -6)
    assert np.array_equal(wk.bf16_bits_to_f32(W), (cw * 2.0 ** -6).astype(np.float32))
    s = oracle.compute_smoothing(np.abs(X).max(0), oracle.weight_absmax(W), 0.5)
    assert np.all(s == 1.0)
    err, ref = oracle.alpha_output_error(X, W, 0.5)
    assert err == 0.0 and ref > 0
    # with another alpha the scale is not 1 and rounding appears
    assert oracle.alpha_output_error(X, W, 0.25)[0] > 0


def test_worked_example_layer_exact_rationals():
    # the explainer's layer x = (40, 1), w = (0.5, 0.5), alpha = 0.5 on one
    # token: every step by hand in exact rationals, one rounding per step
    X = np.array([[40.0, 1.0]], np.float32)
    W = bf16([[0.5, 0.5]])
    s = oracle.compute_smoothing(np.abs(X).max(0), oracle.weight_absmax(W), 0.5)
    S = [fx.frac(v) for v in s]
    xt = [fx.rn32(fx.frac(X[0, j]) / S[j]) for j in range(2)]
    xsc = fx.rn32(max(abs(v) for v in xt) / 127)
    xq = [fx.rne_int(fx.rn32(v / xsc)) for v in xt]
    wp = [fx.rn32(Fraction(1, 2) * S[j]) for j in range(2)]
    wsc = fx.rn32(max(abs(v) for v in wp) / 127)
    wq = [fx.rne_int(fx.rn32(v / wsc)) for v in wp]
    y = (xq[0] * wq[0] + xq[1] * wq[1]) * xsc * wsc
    want_err = (y - Fraction(41, 2)) ** 2
    err, ref = oracle.alpha_output_error(X, W, 0.5)
    assert ref == 20.5 ** 2
    assert abs(Fraction(err) - want_err) <= want_err * Fraction(1, 10**9) + Fraction(1, 10**40)
    assert err > 0


def test_error_is_the_sum_of_squared_differences():
    wl = wk.make_workload("parity_ragged")
    X = wl.X_cal[:40]
    err, ref = oracle.alpha_output_error(X, wl.W, 0.5)
    # the same quantities from the oracle's pinned steps
    a = oracle.act_absmax_update(X)
    s = oracle.compute_smoothing(a, oracle.weight_absmax(wl.W), 0.5)
    Wq, ws = oracle.quantize_weight(wl.W, s)
    Xq, xs = oracle.quant_act(X, s)
    Y = (Xq.astype(np.int64) @ Wq.astype(np.int64).T) * xs[:, None].astype(np.float64) * ws[None, :]
    R = wk.bf16_bits_to_f32(X).astype(np.float64) @ wk.bf16_bits_to_f32(wl.W).astype(np.float64).T
    assert np.isclose(err, ((Y - R) ** 2).sum(), rtol=1e-9)
    assert np.isclose(ref, (R ** 2).sum(), rtol=1e-12)
    # smoothing with a sensible alpha beats no migration toward the weights
    e0, _ = oracle.alpha_output_error(X, wl.W, 0.0)
    assert err < e0
