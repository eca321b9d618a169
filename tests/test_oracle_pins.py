"""Pins of the CPU oracle to facts outside itself (no GPU needed).

Each test ties one oracle function to something the pages print, a closed
form, an invariant of the mathematics, a library routine computing the same
quantity by a different route, or exact rational brute force.  A dropped term,
wrong sign, wrong index, transposed operand, multiply-instead-of-divide or a
wrong rounding rule in the oracle fails at least one of them.
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


def bf16(a):
    return wk.f32_to_bf16_bits(np.asarray(a, np.float32))


def f32(a):
    return np.asarray(a, np.float32)


# --------------------------------------------------------------------------
# The explainer's worked example ("A worked example"), values as printed.
# --------------------------------------------------------------------------
@pytest.fixture(scope="module")
def worked():
    with open(os.path.join(GOLDEN, "worked_example.json")) as f:
        return json.load(f)


def test_worked_example_per_tensor(worked):
    # one token = one tensor: the per-token scale is the page's per-tensor scale
    X = f32([worked["x"]])
    Xq, xs = oracle.quant_act(X, np.ones(2, np.float32))
    pt = worked["per_tensor"]
    assert round(float(xs[0]), pt["scale_decimals"]) == pt["scale_approx"]
    assert Xq[0, 1] == pt["q_small"]
    assert Xq[0, 0] == 127
    assert round(float(Xq[0, 1]) * float(xs[0]), pt["dequant_decimals"]) == pt["dequant_small_approx"]


def test_worked_example_outlier_400(worked):
    o = worked["outlier_400"]
    Xq, xs = oracle.quant_act(f32([o["x"]]), np.ones(2, np.float32))
    assert round(float(xs[0]), o["scale_decimals"]) == o["scale_approx"]
    assert Xq[0, 1] == o["q_small"]  # the small channel vanishes


def test_worked_example_smoothed(worked):
    sm = worked["smoothed"]
    s = f32(sm["s"])
    X = f32([worked["x"]])
    W = bf16([worked["w"]])            # [N=1, K=2]
    Xq, xs = oracle.quant_act(X, s)
    assert round(float(xs[0]), sm["scale_decimals"]) == sm["scale_approx"]
    assert Xq[0, 1] == sm["q_small"]
    # dequantized smoothed activations recover (4, 1)
    assert np.allclose(Xq[0] * xs[0], sm["x_smoothed"], atol=xs[0] / 2 + 1e-7)
    # the folded weights are (5.0, 0.5)
    Wq, ws = oracle.quantize_weight(W, s)
    assert np.allclose(Wq[0] * ws[0], sm["w_scaled"], atol=ws[0] / 2 + 1e-7)
    # equivalence before rounding: the output is still 20.5
    assert oracle.smoothed_product_rows(X, W, s)[0, 0] == sm["output"]
    assert oracle.reference_rows(X, W, [], [], [], [0, 1], [-1])[0, 0] == worked["exact_output"]
    # after W8A8 the small channel survives and the output stays close to 20.5
    y = oracle.linear_lora_rows(Xq, xs, Wq, ws, [], [], [0, 1], [-1])["Y"][0, 0]
    assert abs(y - sm["output"]) < 0.05
    # integer check by hand: codes (127, 32) . (127, 13) = 16545
    assert oracle.gemm_rows(Xq, Wq)[0, 0] == 127 * 127 + 32 * 13


# --------------------------------------------------------------------------
# Smoothing scale (Step 3 and the sketch): closed forms and the alpha limits.
# --------------------------------------------------------------------------
def test_smoothing_closed_forms():
    a = f32([4.0, 9.0, 1.0, 100.0])
    w = f32([1.0, 4.0, 0.25, 0.01])
    s = oracle.compute_smoothing(a, w, 0.5)
    assert s.tolist() == [2.0, 1.5, 2.0, 100.0]   # sqrt(a/w)
    # alpha = 1: s = a ;  alpha = 0: s = 1/w (one IEEE division)
    a2 = np.random.default_rng(0).uniform(0.01, 300, 64).astype(np.float32)
    w2 = np.random.default_rng(1).uniform(0.001, 0.2, 64).astype(np.float32)
    assert np.array_equal(oracle.compute_smoothing(a2, w2, 1.0), a2)
    assert np.array_equal(oracle.compute_smoothing(a2, w2, 0.0), np.float32(1.0) / w2)


def test_smoothing_clamps():
    # dead channels are clamped at 1e-5 before the powers, and s itself at 1e-5
    s = oracle.compute_smoothing(f32([0.0, 0.0, 1e-12]), f32([0.0, 1.0, 1e6]), 0.5)
    lo = Fraction(float(np.float32(1e-5)))
    assert s[0] == np.float32(1.0)                     # (1e-5)^.5 / (1e-5)^.5
    assert s[1] == np.float32(np.sqrt(float(lo)))      # (1e-5)^.5 / 1^.5, rounded once
    assert s[2] == np.float32(1e-5)                    # tiny / huge -> clamp


def test_smoothing_balance_alpha_half():
    # alpha = 0.5 balances the two maxima: max|X_j/s_j| = max|W_j s_j| = sqrt(a_j w_j)
    wl = wk.make_workload("parity_ragged")
    a = oracle.act_absmax_update(wl.X_cal)
    w = oracle.weight_absmax(wl.W)
    s = oracle.compute_smoothing(a, w, 0.5).astype(np.float64)
    xc = wk.bf16_bits_to_f32(wl.X_cal).astype(np.float64)
    W = wk.bf16_bits_to_f32(wl.W).astype(np.float64)
    x_max = np.abs(xc / s).max(axis=0)
    w_max = np.abs(W * s).max(axis=0)
    target = np.sqrt(a.astype(np.float64) * w.astype(np.float64))
    assert np.allclose(x_max, target, rtol=1e-6)
    assert np.allclose(w_max, target, rtol=1e-6)
    # and the activation maxima are much flatter after smoothing
    assert (x_max.max() / np.median(x_max)) < 0.5 * (a.max() / np.median(a))


def test_smoothing_alpha_limits_flatten_one_side():
    wl = wk.make_workload("parity_heavy_f32")
    a = oracle.act_absmax_update(wl.X_cal)
    w = oracle.weight_absmax(wl.W)
    s1 = oracle.compute_smoothing(a, w, 1.0).astype(np.float64)
    s0 = oracle.compute_smoothing(a, w, 0.0).astype(np.float64)
    # alpha = 1: every calibration channel max becomes 1 after smoothing
    assert np.allclose(np.abs(wl.X_cal / s1).max(axis=0), 1.0, rtol=1e-7)
    # alpha = 0: every folded weight channel max becomes 1
    W = wk.bf16_bits_to_f32(wl.W).astype(np.float64)
    assert np.allclose(np.abs(W * s0).max(axis=0), 1.0, rtol=1e-6)


def test_absmax_is_columnwise_max():
    rng = np.random.default_rng(5)
    X = rng.standard_normal((37, 19)).astype(np.float32)
    assert np.array_equal(oracle.act_absmax_update(X), np.abs(X).max(axis=0))
    # running max over two batches equals the max over their union
    X2 = rng.standard_normal((11, 19)).astype(np.float32) * 3
    run = oracle.act_absmax_update(X2, oracle.act_absmax_update(X))
    assert np.array_equal(run, np.abs(np.concatenate([X, X2])).max(axis=0))
    Wb = bf16(rng.standard_normal((23, 19)))
    assert np.array_equal(oracle.weight_absmax(Wb), np.abs(wk.bf16_bits_to_f32(Wb)).max(axis=0))


# --------------------------------------------------------------------------
# Quantizers (Step 6 and the sketch's quantize_int8)
# --------------------------------------------------------------------------
def test_ties_round_half_to_even():
    # amax = 127/16 makes the scale exactly 1/16; values (n + 1/2)/16 are exact ties
    halves = np.array([0.5, 1.5, 2.5, 3.5, -0.5, -1.5, -2.5, 126.5, -126.5], np.float32)
    X = np.concatenate([[127.0], halves]).astype(np.float32)[None, :] / np.float32(16)
    Xq, xs = oracle.quant_act(X, np.ones(X.shape[1], np.float32))
    assert xs[0] == np.float32(1 / 16)
    assert Xq[0, 1:].tolist() == [0, 2, 2, 4, 0, -2, -2, 126, -126]


def test_identity_smoothing_is_sketch_quantizer():
    # with s = 1 the activation quantizer is the sketch's quantize_int8 along
    # each row; numpy evaluates that in float32 with IEEE division and np.round
    rng = np.random.default_rng(3)
    X = (rng.standard_normal((40, 96)) * rng.uniform(0.01, 50, (40, 1))).astype(np.float32)
    Xq, xs = oracle.quant_act(X, np.ones(96, np.float32))
    scale = np.abs(X).max(axis=1, keepdims=True) / np.float32(127)
    q = np.clip(np.round(X / scale), -128, 127).astype(np.int8)
    assert np.array_equal(xs, scale[:, 0])
    assert np.array_equal(Xq, q)
    Wb = bf16(rng.standard_normal((33, 96)) * 0.02)
    Wq, ws = oracle.quantize_weight(Wb, np.ones(96, np.float32))
    Wf = wk.bf16_bits_to_f32(Wb)
    wsc = np.abs(Wf).max(axis=1, keepdims=True) / np.float32(127)
    assert np.array_equal(ws, wsc[:, 0])
    assert np.array_equal(Wq, np.clip(np.round(Wf / wsc), -128, 127).astype(np.int8))


def test_quant_act_float32_route():
    # same quantity through numpy's float32 IEEE operations (one rounding per
    # operation, no fp64 intermediate): identical bits
    wl = wk.make_workload("parity_ragged")
    s = oracle.compute_smoothing(oracle.act_absmax_update(wl.X_cal), oracle.weight_absmax(wl.W), 0.5)
    Xq, xs = oracle.quant_act(wl.X, s)
    xt = wk.bf16_bits_to_f32(wl.X) / s[None, :]
    sc = np.abs(xt).max(axis=1) / np.float32(127)
    q = np.clip(np.round(xt / sc[:, None]), -128, 127).astype(np.int8)
    assert np.array_equal(xs, sc)
    assert np.array_equal(Xq, q)


def test_dequant_unsmooth_recovers_inputs():
    # Xq*x_scale*s ~= X within half a quantization step (division by s, not
    # multiplication); Wq*w_scale/s ~= W likewise (s folded into W, not 1/s)
    wl = wk.make_workload("parity_ragged")
    s = oracle.compute_smoothing(oracle.act_absmax_update(wl.X_cal), oracle.weight_absmax(wl.W), 0.5)
    Xq, xs = oracle.quant_act(wl.X, s)
    X = wk.bf16_bits_to_f32(wl.X).astype(np.float64)
    err = np.abs(Xq * xs[:, None].astype(np.float64) * s - X)
    bound = 0.5 * xs[:, None].astype(np.float64) * s * (1 + 1e-5) + 1e-30
    assert np.all(err <= bound)
    Wq, ws = oracle.quantize_weight(wl.W, s)
    W = wk.bf16_bits_to_f32(wl.W).astype(np.float64)
    errw = np.abs(Wq * ws[:, None].astype(np.float64) / s - W)
    assert np.all(errw <= 0.5 * ws[:, None] / s * (1 + 1e-5) + 1e-30)
    # -128 is never produced by symmetric absmax quantization
    assert Xq.min() >= -127 and Wq.min() >= -127


def test_zero_rows_and_channels():
    X = np.zeros((3, 32), np.float32)
    X[1, 5] = 2.0
    Xq, xs = oracle.quant_act(X, np.ones(32, np.float32))
    assert xs.tolist() == [0.0, np.float32(2.0 / 127), 0.0]
    assert Xq[0].tolist() == [0] * 32 and Xq[1, 5] == 127
    Wq, ws = oracle.quantize_weight(np.zeros((2, 32), np.uint16), np.ones(32, np.float32))
    assert ws.tolist() == [0.0, 0.0] and not Wq.any()


# --------------------------------------------------------------------------
# Brute force with exact rationals on tiny inputs (one rounding per step)
# --------------------------------------------------------------------------
def _exact_pipeline(X, s, W, A_s, B_s, row_ad):
    M, K = X.shape
    N = W.shape[0]
    Sx = [fx.frac(v) for v in s]
    Xq = np.zeros((M, K), np.int64)
    xs = []
    for i in range(M):
        xt = [fx.rn32(fx.frac(X[i, j]) / Sx[j]) for j in range(K)]
        sc = fx.rn32(max(abs(v) for v in xt) / 127)
        xs.append(sc)
        for j in range(K):
            Xq[i, j] = 0 if sc == 0 else max(-128, min(127, fx.rne_int(fx.rn32(xt[j] / sc))))
    Wf = wk.bf16_bits_to_f32(W)
    Wq = np.zeros((N, K), np.int64)
    ws = []
    for n in range(N):
        wp = [fx.rn32(fx.frac(Wf[n, k]) * Sx[k]) for k in range(K)]
        sc = fx.rn32(max(abs(v) for v in wp) / 127)
        ws.append(sc)
        for k in range(K):
            Wq[n, k] = 0 if sc == 0 else max(-128, min(127, fx.rne_int(fx.rn32(wp[k] / sc))))
    Y = []
    for i in range(M):
        a = row_ad[i]
        if a >= 0:
            Af = wk.bf16_bits_to_f32(A_s[a])
            Bf = wk.bf16_bits_to_f32(B_s[a])
            T = [sum((Xq[i, k] * xs[i]) * fx.frac(Af[j, k]) for k in range(K)) for j in range(Af.shape[0])]
        row = []
        for n in range(N):
            acc = sum(int(Xq[i, k]) * int(Wq[n, k]) for k in range(K))
            d = sum(T[j] * fx.frac(Bf[n, j]) for j in range(len(T))) if a >= 0 else Fraction(0)
            row.append(acc * xs[i] * ws[n] + d)
        Y.append(row)
    return Xq, xs, Wq, ws, Y


@pytest.mark.parametrize("seed", [0, 1, 2])
def test_brute_force_exact_rationals(seed):
    rng = np.random.default_rng(100 + seed)
    M, K, N, r = 4, 6, 5, 3
    X = (rng.standard_normal((M, K)) * rng.choice([1, 1, 30], K)).astype(np.float32)
    W = bf16(rng.standard_normal((N, K)) * 0.05)
    s = oracle.compute_smoothing(np.abs(X).max(0), oracle.weight_absmax(W), 0.5)
    A = bf16(rng.standard_normal((r, K)) / r)
    B = bf16(rng.standard_normal((N, r)) * 0.1)
    A_s, B_s = oracle.prepare_lora(A, B, s, 2.0 * r)
    so, sa = np.array([0, 2, M], np.int32), np.array([0, -1], np.int32)
    Xq, xs = oracle.quant_act(X, s)
    Wq, ws = oracle.quantize_weight(W, s)
    eXq, exs, eWq, ews, eY = _exact_pipeline(X, s, W, [A_s], [B_s], [0, 0, -1, -1])
    assert np.array_equal(Xq, eXq) and np.array_equal(Wq, eWq)
    assert [fx.frac(v) for v in xs] == exs and [fx.frac(v) for v in ws] == ews
    Y = oracle.linear_lora_rows(Xq, xs, Wq, ws, [A_s], [B_s], so, sa)["Y"]
    for i in range(M):
        for n in range(N):
            assert abs(Fraction(float(Y[i, n])) - eY[i][n]) <= abs(eY[i][n]) * Fraction(1, 10**12) + Fraction(1, 10**300)


def test_bf16_rounding_exact():
    # the oracle's bf16 rounding (significand arithmetic) vs exact rationals and
    # the bit-pattern rounding of the workload generator
    rng = np.random.default_rng(9)
    vals = np.concatenate([rng.standard_normal(2000).astype(np.float32) * 10,
                           f32([1 + 2 ** -8, 1 + 3 * 2 ** -8, -(1 + 2 ** -8), 2 ** -130, 3e38])])
    for v in vals:
        got = oracle.round_bf16(float(v))
        want = fx.rn_bf16(fx.frac(v))
        assert float(wk.bf16_bits_to_f32(np.array([got], np.uint16))[0]) == float(want)
    assert np.array_equal(np.array([oracle.round_bf16(float(v)) for v in vals], np.uint16),
                          wk.f32_to_bf16_bits(vals))


# --------------------------------------------------------------------------
# GEMM (Step 7) and LoRA delta (issue #12703 pitch)
# --------------------------------------------------------------------------
def test_gemm_matches_numpy_int64():
    rng = np.random.default_rng(11)
    Xq = rng.integers(-127, 128, (19, 77), dtype=np.int64).astype(np.int8)
    Wq = rng.integers(-127, 128, (13, 77), dtype=np.int64).astype(np.int8)
    want = Xq.astype(np.int64) @ Wq.astype(np.int64).T
    assert np.array_equal(oracle.gemm_rows(Xq, Wq), want)
    rows, cols = np.array([0, 18, 5]), np.array([12, 0, 7])
    assert np.array_equal(oracle.gemm_pairs(Xq, Wq, rows, cols), want[rows, cols])


def test_gemm_worst_case_fits_int32():
    K = 14336
    Xq = np.full((1, K), 127, np.int8)
    Wq = np.full((2, K), 127, np.int8)
    Wq[1] = -127
    acc = oracle.gemm_rows(Xq, Wq)
    assert acc.tolist() == [[K * 127 * 127, -K * 127 * 127]]
    assert K * 127 * 127 < 2 ** 31


def test_prepare_lora_float32_route():
    rng = np.random.default_rng(12)
    r, K, N = 16, 80, 48
    A = bf16(rng.standard_normal((r, K)) / r)
    B = bf16(rng.standard_normal((N, r)) * 0.01)
    s = rng.uniform(0.05, 20, K).astype(np.float32)
    A_s, B_s = oracle.prepare_lora(A, B, s, 32.0)
    assert np.array_equal(A_s, wk.f32_to_bf16_bits(wk.bf16_bits_to_f32(A) * s[None, :]))
    scale = np.float32(32.0) / np.float32(r)
    assert np.array_equal(B_s, wk.f32_to_bf16_bits(wk.bf16_bits_to_f32(B) * scale))


def _prepared(name):
    return oracle.Prepared(wk.make_workload(name))


def test_linear_lora_matches_numpy_fp64():
    P = _prepared("parity_heavy_f32")
    wl = P.wl
    out = P.rows()
    xh = P.Xq.astype(np.float64) * P.x_scale[:, None]
    base = (P.Xq.astype(np.int64) @ P.Wq.astype(np.int64).T)
    assert np.array_equal(out["acc"], base)
    ad = wk.row_adapter(wl.seg_offsets, wl.seg_adapter, wl.M, len(wl.adapters))
    delta = np.zeros((wl.M, wl.N))
    for a in range(len(wl.adapters)):
        m = ad == a
        A = wk.bf16_bits_to_f32(P.A_s[a]).astype(np.float64)
        B = wk.bf16_bits_to_f32(P.B_s[a]).astype(np.float64)
        delta[m] = (xh[m] @ A.T) @ B.T
    assert np.allclose(out["delta"], delta, rtol=1e-12, atol=1e-12 * np.abs(delta).max())
    Y = base * P.x_scale[:, None].astype(np.float64) * P.w_scale[None, :] + delta
    assert np.allclose(out["Y"], Y, rtol=1e-12, atol=1e-12 * np.abs(Y).max())
    assert (ad == -1).any() and (ad >= 0).any()


def test_lora_zero_B_and_no_adapter_give_base():
    P = _prepared("parity_ragged")
    wl = P.wl
    zeroB = [np.zeros_like(b) for b in P.B_s]
    y0 = oracle.linear_lora_rows(P.Xq, P.x_scale, P.Wq, P.w_scale, P.A_s, zeroB,
                                 wl.seg_offsets, wl.seg_adapter)
    none = oracle.linear_lora_rows(P.Xq, P.x_scale, P.Wq, P.w_scale, P.A_s, P.B_s,
                                   wl.seg_offsets, np.full_like(wl.seg_adapter, -1))
    assert not y0["delta"].any() and not none["delta"].any()
    assert np.array_equal(y0["Y"], none["Y"])
    base = P.Xq.astype(np.int64) @ P.Wq.astype(np.int64).T
    assert np.allclose(none["Y"], base * P.x_scale[:, None].astype(np.float64) * P.w_scale[None, :],
                       rtol=1e-14, atol=0)


def test_lora_unsmoothing_matches_unquantized_lora():
    # the LoRA path sees Xq*x_scale (~X/s); folding s into A recovers X@A^T
    P = _prepared("parity_ragged")
    wl = P.wl
    ref = oracle.reference_rows(wl.X, np.zeros_like(wl.W), [a.A for a in wl.adapters],
                                [a.B for a in wl.adapters], [a.lora_alpha for a in wl.adapters],
                                wl.seg_offsets, wl.seg_adapter)
    d = P.rows(want=("delta",))["delta"]
    assert np.abs(ref).max() > 0
    assert np.abs(d - ref).max() / np.abs(ref).max() < 2e-2


def test_equivalence_invariant():
    # (X diag(s)^-1)(diag(s) W) = X W to fp64 rounding, for any positive s
    wl = wk.make_workload("parity_heavy_f32")
    s = np.random.default_rng(4).uniform(0.01, 100, wl.K).astype(np.float32)
    rows = np.arange(0, wl.M, 7)
    lhs = oracle.smoothed_product_rows(wl.X, wl.W, s, rows)
    rhs = wl.X[rows].astype(np.float64) @ wk.bf16_bits_to_f32(wl.W).astype(np.float64).T
    assert np.abs(lhs - rhs).max() <= 1e-13 * np.abs(rhs).max()


@pytest.mark.parametrize("name", ["parity_ragged", "parity_heavy_f32"])
def test_w8a8_close_to_unquantized_and_smoothing_helps(name):
    P = _prepared(name)
    wl = P.wl
    ref = oracle.reference_rows(wl.X, wl.W, [a.A for a in wl.adapters], [a.B for a in wl.adapters],
                                [a.lora_alpha for a in wl.adapters], wl.seg_offsets, wl.seg_adapter)
    Y = P.rows(want=("Y",))["Y"]
    err_smooth = np.abs(Y - ref).max() / np.abs(ref).max()
    assert err_smooth < 3e-2
    # identical pipeline without smoothing (s = 1) on outlier-heavy inputs is worse
    ones = np.ones(wl.K, np.float32)
    Xq1, xs1 = oracle.quant_act(wl.X, ones)
    Wq1, ws1 = oracle.quantize_weight(wl.W, ones)
    A1, B1 = zip(*[oracle.prepare_lora(a.A, a.B, ones, a.lora_alpha) for a in wl.adapters])
    Y1 = oracle.linear_lora_rows(Xq1, xs1, Wq1, ws1, list(A1), list(B1), wl.seg_offsets,
                                 wl.seg_adapter, want=("Y",))["Y"]
    err_plain = np.abs(Y1 - ref).max() / np.abs(ref).max()
    assert err_smooth < err_plain


def test_token_adapter_rules():
    so = np.array([0, 3, 3, 7, 10], np.int32)
    sa = np.array([2, 0, -1, 5], np.int32)
    got = [oracle.token_adapter(so, sa, 3, i) for i in range(12)]
    assert got == [2, 2, 2, -1, -1, -1, -1, -1, -1, -1, -1, -1]
    sa2 = np.array([1, 0, 0, 2], np.int32)
    assert [oracle.token_adapter(so, sa2, 3, i) for i in (0, 3, 6, 7, 9, 10)] == [1, 0, 0, 2, 2, -1]
    assert np.array_equal(wk.row_adapter(so, sa2, 12, 3),
                          [oracle.token_adapter(so, sa2, 3, i) for i in range(12)])
