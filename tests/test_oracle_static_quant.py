"""Pins of the oracle's per-tensor static activation quantization.

"SmoothQuant" explainer, Step 6 and "Calibration in practice": a per-tensor
static scale is fixed offline from the calibration range of the smoothed
activation (one scale for every token), the faster and riskier level of the
method; values the calibrated range does not cover are clamped, and the
number of clamped codes is reported.  Checked against the worked example as
printed, exact rationals, the special case that reduces to the per-token
quantizer, round-half-even at the edge of the range, and a closed form.
"""

import json
import os
from fractions import Fraction

import numpy as np
import pytest

import oracle
from tests import fp_exact as fx
from w8a8_smoothquant_int8_b200 import workloads as wk

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def f32(a):
    return np.asarray(a, np.float32)


@pytest.fixture(scope="module")
def worked():
    with open(os.path.join(GOLDEN, "worked_example.json")) as f:
        return json.load(f)


def test_worked_example_per_tensor_static(worked):
    # calibrate on the example's own tensor: the static scale is the page's
    # per-tensor scale, the small channel's code is 3 and dequantizes to 0.945
    X = f32([worked["x"]])
    s = np.ones(2, np.float32)
    scale = oracle.static_act_scale(np.abs(X).max(0), s)
    pt = worked["per_tensor"]
    assert round(float(scale), pt["scale_decimals"]) == pt["scale_approx"]
    Xq, xs, clipped = oracle.quant_act_static(X, s, scale)
    assert Xq[0].tolist() == [127, pt["q_small"]] and clipped == 0
    assert round(float(Xq[0, 1]) * float(xs[0]), pt["dequant_decimals"]) == pt["dequant_small_approx"]


def test_worked_example_outlier_static_range(worked):
    # a scale calibrated on (40, 1) meets the token (400, 1): the outlier is
    # clamped (one clipped code), the small channel keeps its code 3
    scale = oracle.static_act_scale(f32(worked["x"]), np.ones(2, np.float32))
    Xq, _, clipped = oracle.quant_act_static(f32([worked["outlier_400"]["x"]]), np.ones(2, np.float32),
                                             scale)
    assert Xq[0].tolist() == [127, worked["per_tensor"]["q_small"]] and clipped == 1


@pytest.mark.parametrize("seed", [0, 1, 2])
def test_static_brute_force_exact_rationals(seed):
    rng = np.random.default_rng(500 + seed)
    M, K = 5, 9
    X = (rng.standard_normal((M, K)) * rng.choice([1, 1, 30], K)).astype(np.float32)
    s = (rng.random(K) * 3 + 0.2).astype(np.float32)
    cal = np.abs(X[:3]).max(0)  # calibrated on three tokens: the others may clip
    scale = oracle.static_act_scale(cal, s)
    S = [fx.frac(v) for v in s]
    want_scale = fx.rn32(max(abs(fx.rn32(fx.frac(a) / S[j])) for j, a in enumerate(cal)) / 127)
    assert fx.frac(scale) == want_scale
    Xq, xs, clipped = oracle.quant_act_static(X, s, scale)
    n = 0
    for i in range(M):
        assert fx.frac(xs[i]) == want_scale
        for j in range(K):
            xt = fx.rn32(fx.frac(X[i, j]) / S[j])
            r = fx.rne_int(fx.rn32(xt / want_scale))
            n += r < -128 or r > 127
            assert Xq[i, j] == max(-128, min(127, r))
    assert clipped == n


def test_static_equals_dynamic_when_calibrated_on_the_token():
    # one token calibrated on itself: its per-token scale is the static scale
    rng = np.random.default_rng(3)
    X = (rng.standard_normal((1, 64)) * 5).astype(np.float32)
    s = (rng.random(64) + 0.5).astype(np.float32)
    dq, dxs = oracle.quant_act(X, s)
    sq, sxs, clipped = oracle.quant_act_static(X, s, oracle.static_act_scale(np.abs(X[0]), s))
    assert np.array_equal(dq, sq) and dxs[0] == sxs[0] and clipped == 0


def test_static_round_half_even_at_the_range_edge():
    # scale 2^-4 exactly; xt/scale = 127.5 rounds to 128 (even): clamped and
    # counted; 126.5 rounds to 126; -128.5 rounds to -128 (even): kept
    scale = np.float32(2.0 ** -4)
    X = f32([[127.5 / 16, 126.5 / 16, -128.5 / 16, -129.5 / 16, 0.0]])
    Xq, _, clipped = oracle.quant_act_static(X, np.ones(5, np.float32), scale)
    assert Xq[0].tolist() == [127, 126, -128, -128, 0]
    assert clipped == 2  # 128 and -130


def test_static_scale_closed_form_and_zero_scale():
    # a_j = s_j: every smoothed maximum is 1, the scale is RN(1/127)
    s = f32([0.5, 3.0, 7.25])
    assert oracle.static_act_scale(s, s) == np.float32(1.0 / 127.0)
    # a zero scale (no calibrated range): codes 0, every nonzero value counts
    Xq, xs, clipped = oracle.quant_act_static(f32([[1.0, 0.0, -2.0]]), np.ones(3, np.float32), 0.0)
    assert not Xq.any() and xs[0] == 0.0 and clipped == 2


def test_static_on_a_workload_clips_a_few_tokens():
    wl = wk.make_workload("parity_ragged")
    P = oracle.Prepared(wl)
    scale = oracle.static_act_scale(P.act_absmax, P.s)
    Xq, xs, clipped = oracle.quant_act_static(wl.X, P.s, scale)
    assert (xs == scale).all()
    # codes and the clipped count agree with a numpy restatement (fp32
    # quotients, numpy's round-half-even)
    X = wk.bf16_bits_to_f32(wl.X).astype(np.float64)
    xt = (X / P.s.astype(np.float64)).astype(np.float32).astype(np.float64)
    t = (xt / np.float64(scale)).astype(np.float32).astype(np.float64)
    r = np.round(t)  # numpy rounds half to even
    assert np.array_equal(Xq, np.clip(r, -128, 127).astype(np.int8))
    assert clipped == int(((r < -128) | (r > 127)).sum())
