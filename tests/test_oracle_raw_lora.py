"""Pins of the oracle's raw-input reading of the LoRA path.

"[Feature]: LoRA support for W8A8 SmoothQuant", Pitch: the low-rank path runs
in BF16 after the INT8 GEMM and its result is added to the dequantized
output.  Read on the layer's own bf16 activations: T = X A^T with the
adapters as given (no smoothing fold), delta = T B_s^T with
B_s = bf16(B * lora_alpha / r), Y = dequantized W8A8 output + delta.
The checks below fix it independently of its own code: exact rationals on
tiny inputs, a closed form, a special case that reduces to the graded path,
and closeness to the unquantized layer's LoRA term.
"""

from fractions import Fraction

import numpy as np
import pytest

import oracle
from tests import fp_exact as fx
from w8a8_smoothquant_int8_b200 import workloads as wk


def bf16(a):
    return wk.f32_to_bf16_bits(np.asarray(a, np.float32))


@pytest.mark.parametrize("seed", [0, 1, 2])
def test_raw_brute_force_exact_rationals(seed):
    rng = np.random.default_rng(300 + seed)
    M, K, N, r = 4, 7, 5, 3
    Xf = rng.standard_normal((M, K)) * rng.choice([1, 1, 40], K)
    X = bf16(Xf)
    W = bf16(rng.standard_normal((N, K)) * 0.05)
    s = oracle.compute_smoothing(np.abs(wk.bf16_bits_to_f32(X)).max(0), oracle.weight_absmax(W), 0.5)
    A = bf16(rng.standard_normal((r, K)) / r)
    B = bf16(rng.standard_normal((N, r)) * 0.1)
    A_raw, B_s = oracle.prepare_lora(A, B, None, 2.0 * r)
    Xq, xs = oracle.quant_act(X, s)
    Wq, ws = oracle.quantize_weight(W, s)
    so, sa = np.array([0, 3, M], np.int32), np.array([0, -1], np.int32)
    out = oracle.linear_lora_raw_rows(X, Xq, xs, Wq, ws, [A_raw], [B_s], so, sa)
    Xv = wk.bf16_bits_to_f32(X)
    Av = wk.bf16_bits_to_f32(A)
    Bv = wk.bf16_bits_to_f32(B_s)
    for i in range(M):
        use = i < 3
        T = [sum(fx.frac(Xv[i, k]) * fx.frac(Av[j, k]) for k in range(K)) for j in range(r)]
        for n in range(N):
            d = sum(T[j] * fx.frac(Bv[n, j]) for j in range(r)) if use else Fraction(0)
            acc = sum(int(Xq[i, k]) * int(Wq[n, k]) for k in range(K))
            y = acc * fx.frac(xs[i]) * fx.frac(ws[n]) + d
            tol_d = abs(d) * Fraction(1, 10**12) + Fraction(1, 10**300)
            tol_y = abs(y) * Fraction(1, 10**12) + Fraction(1, 10**300)
            assert abs(Fraction(float(out["delta"][i, n])) - d) <= tol_d
            assert abs(Fraction(float(out["Y"][i, n])) - y) <= tol_y


def test_raw_prepare_keeps_A_and_scales_B():
    rng = np.random.default_rng(7)
    A = bf16(rng.standard_normal((16, 40)))
    B = bf16(rng.standard_normal((24, 16)))
    s = (rng.random(40) * 4 + 0.25).astype(np.float32)
    A_raw, B_raw = oracle.prepare_lora(A, B, None, 32.0)
    A_s, B_s = oracle.prepare_lora(A, B, s, 32.0)
    assert np.array_equal(A_raw, A)
    assert np.array_equal(B_raw, B_s)
    assert not np.array_equal(A_s, A)
    # B_s = bf16(B * 32/16) = B * 2 exactly (a power of two)
    assert np.array_equal(wk.bf16_bits_to_f32(B_raw), wk.bf16_bits_to_f32(B) * 2)


def test_raw_identity_adapter_closed_form():
    # A = [I | 0]: T[i, j] = X[i, j], so delta = X[:, :r] B_s^T; every product
    # of two bf16 values and every sum of r of them is exact in fp64
    rng = np.random.default_rng(8)
    M, K, N, r = 9, 33, 20, 8
    X = bf16(rng.standard_normal((M, K)) * 3)
    W = bf16(rng.standard_normal((N, K)) * 0.05)
    eye = np.zeros((r, K), np.float32)
    eye[np.arange(r), np.arange(r)] = 1.0
    A = bf16(eye)
    B = bf16(rng.standard_normal((N, r)))
    s = np.ones(K, np.float32)
    A_raw, B_s = oracle.prepare_lora(A, B, None, float(r))
    Xq, xs = oracle.quant_act(X, s)
    Wq, ws = oracle.quantize_weight(W, s)
    so, sa = np.array([0, M], np.int32), np.array([0], np.int32)
    out = oracle.linear_lora_raw_rows(X, Xq, xs, Wq, ws, [A_raw], [B_s], so, sa, want=("delta",))
    want = wk.bf16_bits_to_f32(X)[:, :r].astype(np.float64) @ wk.bf16_bits_to_f32(B_s).astype(np.float64).T
    assert np.array_equal(out["delta"], want)


def test_raw_zero_B_is_the_graded_base():
    wl = wk.make_workload("parity_ragged")
    P = oracle.Prepared(wl)
    A_raw = [a.A for a in wl.adapters]
    zeroB = [np.zeros_like(b) for b in P.B_s]
    raw = oracle.linear_lora_raw_rows(wl.X, P.Xq, P.x_scale, P.Wq, P.w_scale, A_raw, zeroB,
                                      wl.seg_offsets, wl.seg_adapter)
    graded = oracle.linear_lora_rows(P.Xq, P.x_scale, P.Wq, P.w_scale, P.A_s, zeroB,
                                     wl.seg_offsets, wl.seg_adapter, want=("Y",))
    assert not raw["delta"].any()
    assert np.array_equal(raw["Y"], graded["Y"])


@pytest.mark.parametrize("name", ["parity_ragged", "parity_decode"])
def test_raw_delta_close_to_unquantized_lora(name):
    # the only rounding between the raw delta and the unquantized layer's LoRA
    # term (alpha/r) (X A^T) B^T is B's bf16 rounding after the alpha/r scale
    wl = wk.make_workload(name)
    P = oracle.Prepared(wl)
    A_raw = [a.A for a in wl.adapters]
    raw = oracle.linear_lora_raw_rows(wl.X, P.Xq, P.x_scale, P.Wq, P.w_scale, A_raw, P.B_s,
                                      wl.seg_offsets, wl.seg_adapter, want=("delta",))
    ad = wk.row_adapter(wl.seg_offsets, wl.seg_adapter, wl.M, len(wl.adapters))
    X = wk.bf16_bits_to_f32(wl.X).astype(np.float64)
    ref = np.zeros_like(raw["delta"])
    for a, spec in enumerate(wl.adapters):
        m = ad == a
        if not m.any():
            continue
        A = wk.bf16_bits_to_f32(spec.A).astype(np.float64)
        B = wk.bf16_bits_to_f32(spec.B).astype(np.float64)
        ref[m] = (spec.lora_alpha / spec.r) * (X[m] @ A.T) @ B.T
    err = np.abs(raw["delta"] - ref).max() / np.abs(ref).max()
    assert err <= 2.0 ** -8
    assert (ad >= 0).any()
