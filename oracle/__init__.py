"""CPU oracle for the SmoothQuant W8A8 + per-request LoRA linear (numpy front end).

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
CPU-baseline leg of ``bench.py`` may import this package.  It wraps the plain C
oracle in ``sq_oracle.c`` (fp64 / int64) and shares nothing with the CUDA
library in ``w8a8_smoothquant_int8_b200``.

Each wrapper states the step of the method it computes; the C source cites the
page section for each.
"""

from __future__ import annotations

import ctypes
import os
import subprocess
from typing import List, Optional, Sequence

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "sq_oracle.c")
_HDR = os.path.join(_HERE, "sq_oracle.h")
_LIB = os.path.join(_HERE, "libsq_oracle.so")

F32, BF16 = 0, 1

_lib = None


def build(force: bool = False) -> str:
    """Compile the oracle with gcc (IEEE semantics: no fast-math, no FMA contraction)."""
    stale = (not os.path.exists(_LIB)) or any(
        os.path.getmtime(p) > os.path.getmtime(_LIB) for p in (_SRC, _HDR))
    if force or stale:
        tmp = _LIB + f".tmp{os.getpid()}"
        cmd = ["gcc", "-O3", "-std=c11", "-fopenmp", "-fPIC", "-shared",
               "-fno-fast-math", "-ffp-contract=off", "-Wall", "-Wextra",
               "-o", tmp, _SRC, "-lm"]
        subprocess.check_call(cmd)
        os.replace(tmp, _LIB)
    return _LIB


def lib():
    global _lib
    if _lib is None:
        L = ctypes.CDLL(build())
        P, I64, I32, F = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int, ctypes.c_float
        sig = {
            "sqo_num_threads": ([], I32),
            "sqo_round_bf16": ([F], ctypes.c_uint16),
            "sqo_act_absmax_update": ([P, I32, I64, I64, P], None),
            "sqo_weight_absmax": ([P, I64, I64, P], None),
            "sqo_compute_smoothing": ([P, P, I64, F, P], None),
            "sqo_quantize_weight": ([P, P, I64, I64, P, P], None),
            "sqo_quant_act": ([P, I32, P, I64, I64, P, P], None),
            "sqo_prepare_lora": ([P, P, P, I64, I64, I64, F, P, P], None),
            "sqo_static_act_scale": ([P, P, I64], F),
            "sqo_fold_norm_weight": ([P, P, I64, P], None),
            "sqo_rmsnorm_quant_act": ([P, P, F, I64, I64, P, P], None),
            "sqo_sum_squares_bf16": ([P, I64], ctypes.c_double),
            "sqo_quant_act_static": ([P, I32, P, F, I64, I64, P, P], I64),
            "sqo_gemm_rows": ([P, P, I64, I64, I64, P, I64, P], None),
            "sqo_gemm_pairs": ([P, P, I64, P, P, I64, P], None),
            "sqo_token_adapter": ([P, P, I64, I32, I64], I32),
            "sqo_linear_lora_rows": ([P, P, P, P, I64, I64, I64, I32, P, P, P, P, P, I64,
                                      P, I64, P, P, P], None),
            "sqo_linear_lora_raw_rows": ([P, P, P, P, P, I64, I64, I64, I32, P, P, P, P, P,
                                          I64, P, I64, P, P], None),
            "sqo_reference_rows": ([P, I32, P, I64, I64, I64, I32, P, P, P, P, P, P, I64,
                                    P, I64, P], None),
            "sqo_smoothed_product_rows": ([P, I32, P, P, I64, I64, P, I64, P], None),
        }
        for name, (args, res) in sig.items():
            fn = getattr(L, name)
            fn.argtypes = args
            fn.restype = res
        _lib = L
    return _lib


def _p(a: Optional[np.ndarray]):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def _c(a, dtype):
    return np.ascontiguousarray(a, dtype=dtype)


def _xdtype(X: np.ndarray) -> int:
    if X.dtype == np.float32:
        return F32
    if X.dtype == np.uint16:
        return BF16
    raise TypeError("X must be float32 or uint16 (bf16 bits)")


def num_threads() -> int:
    return int(lib().sqo_num_threads())


def round_bf16(f: float) -> int:
    return int(lib().sqo_round_bf16(float(f)))


def act_absmax_update(X: np.ndarray, act_absmax: Optional[np.ndarray] = None) -> np.ndarray:
    """Running per-input-channel max |X| over a calibration batch."""
    X = np.ascontiguousarray(X)
    M, K = X.shape
    out = np.zeros(K, np.float32) if act_absmax is None else _c(act_absmax, np.float32).copy()
    lib().sqo_act_absmax_update(_p(X), _xdtype(X), M, K, _p(out))
    return out


def weight_absmax(W: np.ndarray) -> np.ndarray:
    """Per-input-channel max |W| over output channels (W is [N, K] bf16 bits)."""
    W = _c(W, np.uint16)
    N, K = W.shape
    out = np.zeros(K, np.float32)
    lib().sqo_weight_absmax(_p(W), N, K, _p(out))
    return out


def compute_smoothing(act_absmax: np.ndarray, w_absmax: np.ndarray, alpha: float) -> np.ndarray:
    """s_j = max(a_j,1e-5)^alpha / max(w_j,1e-5)^(1-alpha), clamped at 1e-5, fp32."""
    a = _c(act_absmax, np.float32)
    w = _c(w_absmax, np.float32)
    s = np.zeros(a.shape[0], np.float32)
    lib().sqo_compute_smoothing(_p(a), _p(w), a.shape[0], float(np.float32(alpha)), _p(s))
    return s


def quantize_weight(W: np.ndarray, s: np.ndarray):
    """Fold s into W along K, then per-output-channel INT8. Returns (Wq, w_scale)."""
    W = _c(W, np.uint16)
    s = _c(s, np.float32)
    N, K = W.shape
    Wq = np.zeros((N, K), np.int8)
    ws = np.zeros(N, np.float32)
    lib().sqo_quantize_weight(_p(W), _p(s), N, K, _p(Wq), _p(ws))
    return Wq, ws


def quant_act(X: np.ndarray, s: np.ndarray):
    """Divide by s, then per-token INT8. Returns (Xq, x_scale)."""
    X = np.ascontiguousarray(X)
    s = _c(s, np.float32)
    M, K = X.shape
    Xq = np.zeros((M, K), np.int8)
    xs = np.zeros(M, np.float32)
    lib().sqo_quant_act(_p(X), _xdtype(X), _p(s), M, K, _p(Xq), _p(xs))
    return Xq, xs


def static_act_scale(act_absmax: np.ndarray, s: np.ndarray) -> np.float32:
    """Per-tensor (static) activation scale from the calibration maxima."""
    a = _c(act_absmax, np.float32)
    s = _c(s, np.float32)
    return np.float32(lib().sqo_static_act_scale(_p(a), _p(s), a.shape[0]))


def quant_act_static(X: np.ndarray, s: np.ndarray, scale):
    """Per-tensor static quantization: (Xq, x_scale [all = scale], clipped count)."""
    X = np.ascontiguousarray(X)
    s = _c(s, np.float32)
    M, K = X.shape
    Xq = np.zeros((M, K), np.int8)
    xs = np.zeros(M, np.float32)
    n = lib().sqo_quant_act_static(_p(X), _xdtype(X), _p(s), float(np.float32(scale)), M, K,
                                   _p(Xq), _p(xs))
    return Xq, xs, int(n)


def fold_norm_weight(gamma: np.ndarray, s: np.ndarray) -> np.ndarray:
    """gamma_s = RN32(gamma / s): Step 5's inverse scale folded into a norm weight."""
    g = _c(gamma, np.float32)
    s = _c(s, np.float32)
    out = np.zeros_like(g)
    lib().sqo_fold_norm_weight(_p(g), _p(s), g.shape[0], _p(out))
    return out


def sum_squares_bf16(h: np.ndarray) -> float:
    """Exact sum of the squares of a bf16 row, rounded once to fp64."""
    h = _c(h, np.uint16).ravel()
    return float(lib().sqo_sum_squares_bf16(_p(h), h.shape[0]))


def rmsnorm_quant_act(H: np.ndarray, gamma_s: np.ndarray, eps: float):
    """RMS normalization with the folded weight, then per-token INT8 (bf16 H)."""
    H = _c(H, np.uint16)
    g = _c(gamma_s, np.float32)
    M, K = H.shape
    Xq = np.zeros((M, K), np.int8)
    xs = np.zeros(M, np.float32)
    lib().sqo_rmsnorm_quant_act(_p(H), _p(g), float(np.float32(eps)), M, K, _p(Xq), _p(xs))
    return Xq, xs


def prepare_lora(A: np.ndarray, B: np.ndarray, s: Optional[np.ndarray], lora_alpha: float):
    """A_s = bf16(A*s) along K (A unchanged when s is None: the raw-input
    reading), B_s = bf16(B*lora_alpha/r). Returns bf16 bits."""
    A = _c(A, np.uint16)
    B = _c(B, np.uint16)
    s = None if s is None else _c(s, np.float32)
    r, K = A.shape
    N = B.shape[0]
    assert B.shape == (N, r)
    A_s = np.zeros((r, K), np.uint16)
    B_s = np.zeros((N, r), np.uint16)
    lib().sqo_prepare_lora(_p(A), _p(B), _p(s), r, K, N, float(np.float32(lora_alpha)),
                           _p(A_s), _p(B_s))
    return A_s, B_s


def gemm_rows(Xq: np.ndarray, Wq: np.ndarray, rows: Optional[Sequence[int]] = None) -> np.ndarray:
    """Exact int64 Xq[rows] @ Wq^T."""
    Xq = _c(Xq, np.int8)
    Wq = _c(Wq, np.int8)
    M, K = Xq.shape
    N = Wq.shape[0]
    rows = np.arange(M, dtype=np.int64) if rows is None else _c(rows, np.int64)
    acc = np.zeros((rows.shape[0], N), np.int64)
    lib().sqo_gemm_rows(_p(Xq), _p(Wq), M, N, K, _p(rows), rows.shape[0], _p(acc))
    return acc


def gemm_pairs(Xq: np.ndarray, Wq: np.ndarray, rows, cols) -> np.ndarray:
    Xq = _c(Xq, np.int8)
    Wq = _c(Wq, np.int8)
    rows = _c(rows, np.int64)
    cols = _c(cols, np.int64)
    acc = np.zeros(rows.shape[0], np.int64)
    lib().sqo_gemm_pairs(_p(Xq), _p(Wq), Xq.shape[1], _p(rows), _p(cols), rows.shape[0], _p(acc))
    return acc


def token_adapter(seg_offsets, seg_adapter, n_adapters: int, i: int) -> int:
    so = _c(seg_offsets, np.int32)
    sa = _c(seg_adapter, np.int32)
    return int(lib().sqo_token_adapter(_p(so), _p(sa), sa.shape[0], n_adapters, i))


def _ptr_array(arrs: List[np.ndarray]):
    arr = (ctypes.c_void_p * max(1, len(arrs)))()
    for i, a in enumerate(arrs):
        arr[i] = a.ctypes.data
    return arr


def linear_lora_rows(Xq, x_scale, Wq, w_scale, A_s: List[np.ndarray], B_s: List[np.ndarray],
                     seg_offsets, seg_adapter, rows: Optional[Sequence[int]] = None,
                     want=("Y", "delta", "acc")):
    """Dequantized W8A8 output plus the LoRA delta for the selected tokens (fp64).

    Returns a dict with any of "Y" [rows, N] f64, "delta" [rows, N] f64, "acc" [rows, N] i64.
    """
    Xq = _c(Xq, np.int8)
    Wq = _c(Wq, np.int8)
    xs = _c(x_scale, np.float32)
    ws = _c(w_scale, np.float32)
    M, K = Xq.shape
    N = Wq.shape[0]
    A_s = [_c(a, np.uint16) for a in A_s]
    B_s = [_c(b, np.uint16) for b in B_s]
    ranks = np.array([a.shape[0] for a in A_s] or [0], np.int64)
    so = _c(seg_offsets, np.int32)
    sa = _c(seg_adapter, np.int32)
    rows = np.arange(M, dtype=np.int64) if rows is None else _c(rows, np.int64)
    R = rows.shape[0]
    out = {}
    Y = np.zeros((R, N), np.float64) if "Y" in want else None
    D = np.zeros((R, N), np.float64) if "delta" in want else None
    A = np.zeros((R, N), np.int64) if "acc" in want else None
    lib().sqo_linear_lora_rows(_p(Xq), _p(xs), _p(Wq), _p(ws), M, N, K, len(A_s),
                               _ptr_array(A_s), _ptr_array(B_s), _p(ranks), _p(so), _p(sa),
                               sa.shape[0], _p(rows), R, _p(Y), _p(D), _p(A))
    for k, v in (("Y", Y), ("delta", D), ("acc", A)):
        if v is not None:
            out[k] = v
    return out


def linear_lora_raw_rows(X, Xq, x_scale, Wq, w_scale, A: List[np.ndarray], B_s: List[np.ndarray],
                         seg_offsets, seg_adapter, rows: Optional[Sequence[int]] = None,
                         want=("Y", "delta")):
    """Raw-input reading of the LoRA path (fp64): T = X A^T from the bf16
    activations and the adapters as given, delta = T B_s^T, Y = dequantized
    W8A8 output + delta, for the selected tokens.  X must be bf16 bits."""
    X = _c(X, np.uint16)
    Xq = _c(Xq, np.int8)
    Wq = _c(Wq, np.int8)
    xs = _c(x_scale, np.float32)
    ws = _c(w_scale, np.float32)
    M, K = Xq.shape
    N = Wq.shape[0]
    assert X.shape == (M, K)
    A = [_c(a, np.uint16) for a in A]
    B_s = [_c(b, np.uint16) for b in B_s]
    ranks = np.array([a.shape[0] for a in A] or [0], np.int64)
    so = _c(seg_offsets, np.int32)
    sa = _c(seg_adapter, np.int32)
    rows = np.arange(M, dtype=np.int64) if rows is None else _c(rows, np.int64)
    R = rows.shape[0]
    Y = np.zeros((R, N), np.float64) if "Y" in want else None
    D = np.zeros((R, N), np.float64) if "delta" in want else None
    lib().sqo_linear_lora_raw_rows(_p(X), _p(Xq), _p(xs), _p(Wq), _p(ws), M, N, K, len(A),
                                   _ptr_array(A), _ptr_array(B_s), _p(ranks), _p(so), _p(sa),
                                   sa.shape[0], _p(rows), R, _p(Y), _p(D))
    out = {}
    for k, v in (("Y", Y), ("delta", D)):
        if v is not None:
            out[k] = v
    return out


def reference_rows(X, W, A: List[np.ndarray], B: List[np.ndarray], lora_alpha: Sequence[float],
                   seg_offsets, seg_adapter, rows: Optional[Sequence[int]] = None) -> np.ndarray:
    """Unquantized fp64 X@W^T + (alpha/r)(X@A^T)@B^T for the selected tokens."""
    X = np.ascontiguousarray(X)
    W = _c(W, np.uint16)
    M, K = X.shape
    N = W.shape[0]
    A = [_c(a, np.uint16) for a in A]
    B = [_c(b, np.uint16) for b in B]
    ranks = np.array([a.shape[0] for a in A] or [0], np.int64)
    la = np.array(list(lora_alpha) or [0.0], np.float64)
    so = _c(seg_offsets, np.int32)
    sa = _c(seg_adapter, np.int32)
    rows = np.arange(M, dtype=np.int64) if rows is None else _c(rows, np.int64)
    Y = np.zeros((rows.shape[0], N), np.float64)
    lib().sqo_reference_rows(_p(X), _xdtype(X), _p(W), M, N, K, len(A), _ptr_array(A),
                             _ptr_array(B), _p(ranks), _p(la), _p(so), _p(sa), sa.shape[0],
                             _p(rows), rows.shape[0], _p(Y))
    return Y


def smoothed_product_rows(X, W, s, rows: Optional[Sequence[int]] = None) -> np.ndarray:
    """fp64 sum_k (X/s)(s*W): the smoothing transform before any rounding."""
    X = np.ascontiguousarray(X)
    W = _c(W, np.uint16)
    s = _c(s, np.float32)
    M, K = X.shape
    N = W.shape[0]
    rows = np.arange(M, dtype=np.int64) if rows is None else _c(rows, np.int64)
    Y = np.zeros((rows.shape[0], N), np.float64)
    lib().sqo_smoothed_product_rows(_p(X), _xdtype(X), _p(W), _p(s), N, K, _p(rows),
                                    rows.shape[0], _p(Y))
    return Y


def alpha_output_error(X, W, alpha: float, rows: Optional[Sequence[int]] = None):
    """Layer-wise output error of the W8A8 layer for one alpha, on the
    calibration tokens X themselves ("Reading the diagnostics": compare
    layer-wise output error across alpha values; "Per-layer alpha").

    a = per-channel max |X|, w = per-channel max |W|, s = smoothing(a, w, alpha),
    Y = dequantized W8A8 output (fp64), Y_ref = X W^T (fp64).
    Returns (sum over rows of (Y - Y_ref)^2, sum of Y_ref^2)."""
    X = np.ascontiguousarray(X)
    a = act_absmax_update(X)
    s = compute_smoothing(a, weight_absmax(W), alpha)
    Wq, ws = quantize_weight(W, s)
    Xq, xs = quant_act(X, s)
    M = X.shape[0]
    rows = np.arange(M, dtype=np.int64) if rows is None else _c(rows, np.int64)
    none = np.array([0, M], np.int32), np.array([-1], np.int32)
    Y = linear_lora_rows(Xq, xs, Wq, ws, [], [], none[0], none[1], rows, want=("Y",))["Y"]
    ref = reference_rows(X, W, [], [], [], none[0], none[1], rows)
    return float(((Y - ref) ** 2).sum()), float((ref ** 2).sum())


class Prepared:
    """Everything the oracle derives offline and on the hot path for one workload."""

    def __init__(self, wl, want_acc_rows: Optional[Sequence[int]] = None):
        self.wl = wl
        self.act_absmax = act_absmax_update(wl.X_cal)
        self.w_absmax = weight_absmax(wl.W)
        self.s = compute_smoothing(self.act_absmax, self.w_absmax, wl.alpha)
        self.Wq, self.w_scale = quantize_weight(wl.W, self.s)
        self.Xq, self.x_scale = quant_act(wl.X, self.s)
        self.A_s, self.B_s = [], []
        for ad in wl.adapters:
            a, b = prepare_lora(ad.A, ad.B, self.s, ad.lora_alpha)
            self.A_s.append(a)
            self.B_s.append(b)

    def rows(self, rows=None, want=("Y", "delta", "acc")):
        wl = self.wl
        return linear_lora_rows(self.Xq, self.x_scale, self.Wq, self.w_scale, self.A_s, self.B_s,
                                wl.seg_offsets, wl.seg_adapter, rows, want)
