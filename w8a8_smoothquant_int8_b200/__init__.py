"""SmoothQuant W8A8 linear with a per-request LoRA delta on B200 (sm_100a).

Python binding of the C ABI in ``include/sq_w8a8.h``: the functions below have
the same names as the C entry points and only marshal arguments (torch CUDA
tensors -> device pointers, the current torch stream -> cudaStream_t).  Every
step runs in the library's CUDA kernels; there is no Python or CPU fallback.

Layouts (see the header): X [M,K] bf16/f32, W [N,K] bf16, Wq [N,K] int8,
Xq [M,K] int8, scales fp32, Y [M,N] bf16.  The LoRA adapters live in a
``LoraPack`` (packed A_pack [R,K], B_pack [N,R], per-adapter offset and rank).
"""

from __future__ import annotations

import ctypes
from typing import List, Optional, Sequence

from . import _native

__all__ = [
    "SQError", "LoraPack", "sq_status_string", "sq_version", "sq_device_supported",
    "sq_get_device_error", "sq_set_wait_timeout_ns", "sq_set_gemm_events", "sq_selftest_wait_timeout", "sq_act_absmax_update", "sq_weight_absmax",
    "sq_compute_smoothing", "sq_quantize_weight", "sq_prepare_lora", "sq_lora_pack_width",
    "sq_pack_lora", "sq_quant_act",
    "sq_linear_lora_workspace_size", "sq_linear_lora", "sq_linear_lora_noalloc", "sq_gemm_i32",
    "sq_lora_delta", "sq_lora_t_workspace_size", "sq_lora_shrink_raw", "sq_linear_lora_from_t",
    "sq_lora_delta_from_t", "sq_static_act_scale", "sq_quant_act_static",
    "sq_alpha_error_workspace_size", "sq_alpha_output_error", "sq_alpha_sweep", "alpha_sweep",
    "sq_fold_norm_weight", "sq_rmsnorm_quant_act",
]

SQ_DTYPE_F32 = 0
SQ_DTYPE_BF16 = 1
SQ_MAX_LORA_COLS = 1024
SQ_MAX_K = 57344


class SQError(RuntimeError):
    def __init__(self, status: int, fn: str):
        self.status = int(status)
        msg = _native.load().sq_status_string(self.status).decode()
        super().__init__(f"{fn}: {msg} (status {self.status})")


def _lib():
    return _native.load()


def _check(status: int, fn: str):
    if status != 0:
        raise SQError(status, fn)


def _ptr(t) -> Optional[int]:
    if t is None:
        return None
    if isinstance(t, int):
        return t
    return t.data_ptr()


def _stream(stream) -> Optional[int]:
    if stream is not None:
        return stream if isinstance(stream, int) else stream.cuda_stream
    import torch
    return torch.cuda.current_stream().cuda_stream


def _xdtype(X) -> int:
    import torch
    if X.dtype == torch.bfloat16:
        return SQ_DTYPE_BF16
    if X.dtype == torch.float32:
        return SQ_DTYPE_F32
    raise TypeError("activations must be bfloat16 or float32")


def sq_status_string(status: int) -> str:
    return _lib().sq_status_string(int(status)).decode()


def sq_version() -> int:
    return int(_lib().sq_version())


def sq_device_supported(device: int = 0) -> int:
    return int(_lib().sq_device_supported(int(device)))


def sq_get_device_error(clear: bool = True) -> int:
    code = ctypes.c_int(0)
    _check(_lib().sq_get_device_error(ctypes.byref(code), int(bool(clear))), "sq_get_device_error")
    return code.value


def sq_set_wait_timeout_ns(ns: int) -> None:
    _check(_lib().sq_set_wait_timeout_ns(int(ns)), "sq_set_wait_timeout_ns")


def sq_selftest_wait_timeout(timeout_ns: int, stream=None) -> None:
    """Launch a bounded wait on a barrier nothing arrives on (failure-detection test)."""
    _check(_lib().sq_selftest_wait_timeout(int(timeout_ns), _stream(stream)), "sq_selftest_wait_timeout")


def sq_set_gemm_events(before=None, after=None) -> None:
    """Record torch.cuda.Event objects around the fused GEMM launch (None: off)."""
    b = None if before is None else before.cuda_event
    a = None if after is None else after.cuda_event
    _check(_lib().sq_set_gemm_events(b, a), "sq_set_gemm_events")


def sq_act_absmax_update(X, act_absmax, stream=None) -> None:
    M, K = X.shape
    _check(_lib().sq_act_absmax_update(_ptr(X), _xdtype(X), M, K, _ptr(act_absmax), _stream(stream)),
           "sq_act_absmax_update")


def sq_weight_absmax(W, w_absmax, stream=None) -> None:
    N, K = W.shape
    _check(_lib().sq_weight_absmax(_ptr(W), N, K, _ptr(w_absmax), _stream(stream)), "sq_weight_absmax")


def sq_compute_smoothing(act_absmax, w_absmax, alpha: float, s, stream=None) -> None:
    K = act_absmax.shape[0]
    _check(_lib().sq_compute_smoothing(_ptr(act_absmax), _ptr(w_absmax), K, float(alpha), _ptr(s),
                                       _stream(stream)), "sq_compute_smoothing")


def sq_quantize_weight(W, s, Wq, w_scale, stream=None) -> None:
    N, K = W.shape
    _check(_lib().sq_quantize_weight(_ptr(W), _ptr(s), N, K, _ptr(Wq), _ptr(w_scale), _stream(stream)),
           "sq_quantize_weight")


def sq_lora_pack_width(ranks: Sequence[int]) -> int:
    arr = (ctypes.c_int64 * max(1, len(ranks)))(*[int(r) for r in ranks])
    return int(_lib().sq_lora_pack_width(arr, len(ranks)))


def sq_pack_lora(As: List, Bs: List, lora_alphas: Sequence[float], s, R: int, A_pack, B_pack,
                 lora_offset, lora_rank, stream=None) -> None:
    """Every adapter (A [r,K], B [N,r] bf16 device tensors) into one pack and
    its offset/rank tables (sq_pack_lora)."""
    n = len(As)
    K = As[0].shape[1]
    N = Bs[0].shape[0]
    pa = (ctypes.c_void_p * n)(*[_ptr(a) for a in As])
    pb = (ctypes.c_void_p * n)(*[_ptr(b) for b in Bs])
    rk = (ctypes.c_int64 * n)(*[int(a.shape[0]) for a in As])
    al = (ctypes.c_float * n)(*[float(x) for x in lora_alphas])
    _check(_lib().sq_pack_lora(pa, pb, rk, al, n, _ptr(s), K, N, int(R), _ptr(A_pack),
                               _ptr(B_pack), _ptr(lora_offset), _ptr(lora_rank), _stream(stream)),
           "sq_pack_lora")


def sq_prepare_lora(A, B, s, lora_alpha: float, R: int, off: int, A_pack, B_pack, stream=None) -> None:
    r, K = A.shape
    N = B.shape[0]
    _check(_lib().sq_prepare_lora(_ptr(A), _ptr(B), _ptr(s), r, K, N, float(lora_alpha), R, off,
                                  _ptr(A_pack), _ptr(B_pack), _stream(stream)), "sq_prepare_lora")


def sq_static_act_scale(act_absmax, s, scale, stream=None) -> None:
    """Per-tensor static activation scale (one f32 device tensor) from calibration maxima."""
    _check(_lib().sq_static_act_scale(_ptr(act_absmax), _ptr(s), act_absmax.shape[0], _ptr(scale),
                                      _stream(stream)), "sq_static_act_scale")


def sq_quant_act_static(X, s, scale, Xq, x_scale, clip_count, stream=None) -> None:
    """Per-tensor static quantization; clip_count (one int64 device tensor) is incremented."""
    M, K = X.shape
    _check(_lib().sq_quant_act_static(_ptr(X), _xdtype(X), _ptr(s), _ptr(scale), M, K, _ptr(Xq),
                                      _ptr(x_scale), _ptr(clip_count), _stream(stream)),
           "sq_quant_act_static")


def sq_fold_norm_weight(gamma, s, gamma_s, stream=None) -> None:
    """gamma_s = gamma / s (the smoothing folded into an RMS-norm weight)."""
    _check(_lib().sq_fold_norm_weight(_ptr(gamma), _ptr(s), gamma.shape[0], _ptr(gamma_s),
                                      _stream(stream)), "sq_fold_norm_weight")


def sq_rmsnorm_quant_act(H, gamma_s, eps: float, Xq, x_scale, stream=None) -> None:
    """RMS normalization with the folded weight fused with per-token INT8."""
    M, K = H.shape
    _check(_lib().sq_rmsnorm_quant_act(_ptr(H), _ptr(gamma_s), float(eps), M, K, _ptr(Xq),
                                       _ptr(x_scale), _stream(stream)), "sq_rmsnorm_quant_act")


def sq_quant_act(X, s, Xq, x_scale, stream=None) -> None:
    M, K = X.shape
    _check(_lib().sq_quant_act(_ptr(X), _xdtype(X), _ptr(s), M, K, _ptr(Xq), _ptr(x_scale),
                               _stream(stream)), "sq_quant_act")


def sq_linear_lora_workspace_size(M: int, R: int) -> int:
    return int(_lib().sq_linear_lora_workspace_size(int(M), int(R)))


class LoraPack:
    """Adapters packed side by side for the fused kernels (device tensors).

    ``A_pack`` [R,K] and ``B_pack`` [N,R] bf16 hold A*s and B*lora_alpha/r;
    ``offset`` and ``rank`` [n_adapters] int32 locate each adapter.
    """

    def __init__(self, A_pack, B_pack, offset, rank, R: int, n_adapters: int):
        self.A_pack, self.B_pack, self.offset, self.rank = A_pack, B_pack, offset, rank
        self.R, self.n_adapters = int(R), int(n_adapters)

    @staticmethod
    def layout(ranks: Sequence[int]):
        offs, off = [], 0
        for r in ranks:
            offs.append(off)
            off += (int(r) + 15) // 16 * 16
        return offs, off

    @classmethod
    def build(cls, As: List, Bs: List, lora_alphas: Sequence[float], s, stream=None) -> "LoraPack":
        """Pack adapters (A [r,K], B [N,r] bf16 device tensors) with sq_pack_lora.

        s=None packs A unchanged, for the raw-input entry points
        (sq_lora_shrink_raw / sq_linear_lora_from_t)."""
        import torch
        K = s.shape[0] if s is not None else As[0].shape[1]
        N = Bs[0].shape[0] if Bs else 0
        ranks = [a.shape[0] for a in As]
        _, R = cls.layout(ranks)
        dev = s.device if s is not None else As[0].device
        A_pack = torch.empty((max(R, 1), K), dtype=torch.bfloat16, device=dev)
        B_pack = torch.empty((max(N, 1), max(R, 1)), dtype=torch.bfloat16, device=dev)
        offset = torch.zeros(max(1, len(ranks)), dtype=torch.int32, device=dev)
        rank = torch.zeros(max(1, len(ranks)), dtype=torch.int32, device=dev)
        if ranks:
            sq_pack_lora(As, Bs, lora_alphas, s, R, A_pack, B_pack, offset, rank, stream)
        return cls(A_pack, B_pack, offset, rank, R, len(ranks))


def _lora_args(lora: Optional[LoraPack]):
    if lora is None:
        return None, None, None, None, 0, 0
    return (_ptr(lora.A_pack), _ptr(lora.B_pack), _ptr(lora.offset), _ptr(lora.rank),
            lora.n_adapters, lora.R)


def _ws(workspace):
    if workspace is None:
        return None, 0
    return _ptr(workspace), workspace.numel() * workspace.element_size()


def sq_linear_lora(Xq, x_scale, Wq, w_scale, lora: Optional[LoraPack], seg_offsets, seg_adapter, Y,
                   workspace=None, stream=None) -> None:
    M, K = Xq.shape
    N = Wq.shape[0]
    a, b, o, r, n_ad, R = _lora_args(lora)
    S = 0 if seg_adapter is None else seg_adapter.shape[0]
    wp, wb = _ws(workspace)
    _check(_lib().sq_linear_lora(_ptr(Xq), _ptr(x_scale), _ptr(Wq), _ptr(w_scale), M, N, K, a, b, o,
                                 r, n_ad, R, _ptr(seg_offsets), _ptr(seg_adapter), S, _ptr(Y), wp, wb,
                                 _stream(stream)), "sq_linear_lora")


def sq_linear_lora_noalloc(Xq, x_scale, Wq, w_scale, lora: Optional[LoraPack], seg_offsets,
                           seg_adapter, Y, stream=None) -> None:
    """sq_linear_lora for callers that cannot allocate device memory: the
    scratch is the library's static 16 MiB device array (shared by all calls,
    so calls that overlap on the GPU race)."""
    M, K = Xq.shape
    N = Wq.shape[0]
    a, b, o, r, n_ad, R = _lora_args(lora)
    S = 0 if seg_adapter is None else seg_adapter.shape[0]
    _check(_lib().sq_linear_lora_noalloc(_ptr(Xq), _ptr(x_scale), _ptr(Wq), _ptr(w_scale), M, N, K,
                                         a, b, o, r, n_ad, R, _ptr(seg_offsets), _ptr(seg_adapter),
                                         S, _ptr(Y), _stream(stream)), "sq_linear_lora_noalloc")


def sq_gemm_i32(Xq, Wq, acc, stream=None) -> None:
    M, K = Xq.shape
    N = Wq.shape[0]
    _check(_lib().sq_gemm_i32(_ptr(Xq), _ptr(Wq), M, N, K, _ptr(acc), _stream(stream)), "sq_gemm_i32")


def sq_alpha_error_workspace_size(M: int, N: int, K: int) -> int:
    return int(_lib().sq_alpha_error_workspace_size(M, N, K))


def sq_alpha_output_error(X, W, alpha: float, err, workspace, stream=None) -> None:
    """err (2 float64, device) = (sum (Y - X W^T)^2, sum (X W^T)^2) for one alpha."""
    M, K = X.shape
    N = W.shape[0]
    wp, wb = _ws(workspace)
    _check(_lib().sq_alpha_output_error(_ptr(X), _xdtype(X), _ptr(W), M, N, K, float(alpha),
                                        _ptr(err), wp, wb, _stream(stream)),
           "sq_alpha_output_error")


def sq_alpha_sweep(X, W, alphas: Sequence[float], err, rel, best, workspace, stream=None) -> None:
    """err [2n], rel [n] (float64) and best [1] (float32) device tensors from
    one sweep over the host list `alphas` (see sq_alpha_sweep in the header)."""
    M, K = X.shape
    N = W.shape[0]
    arr = (ctypes.c_float * max(1, len(alphas)))(*[float(a) for a in alphas])
    wp, wb = _ws(workspace)
    _check(_lib().sq_alpha_sweep(_ptr(X), _xdtype(X), _ptr(W), M, N, K, arr, len(alphas),
                                 _ptr(err), _ptr(rel), _ptr(best), wp, wb, _stream(stream)),
           "sq_alpha_sweep")


def alpha_sweep(X_cal, W, alphas: Sequence[float], stream=None):
    """Per-layer migration strength by calibration error: the relative
    squared output error of the W8A8 layer for each alpha on the calibration
    tokens, and the alpha with the smallest (sq_alpha_sweep).  Returns
    (errors as a list, best alpha)."""
    import torch
    M, K = X_cal.shape
    N = W.shape[0]
    dev = X_cal.device
    ws = torch.empty(max(sq_alpha_error_workspace_size(M, N, K), 256), dtype=torch.uint8, device=dev)
    err = torch.empty(2 * len(alphas), dtype=torch.float64, device=dev)
    rel = torch.empty(len(alphas), dtype=torch.float64, device=dev)
    best = torch.empty(1, dtype=torch.float32, device=dev)
    sq_alpha_sweep(X_cal, W, alphas, err, rel, best, ws, stream)
    return rel.cpu().tolist(), float(best.cpu()[0])


def sq_lora_t_workspace_size(M: int, R: int) -> int:
    return int(_lib().sq_lora_t_workspace_size(M, R))


def sq_lora_shrink_raw(X, lora: LoraPack, seg_offsets, seg_adapter, workspace, stream=None) -> None:
    """T = X A^T (raw bf16 activations, adapters packed with s=None) into `workspace`."""
    M, K = X.shape
    S = 0 if seg_adapter is None else seg_adapter.shape[0]
    wp, wb = _ws(workspace)
    _check(_lib().sq_lora_shrink_raw(_ptr(X), M, K, _ptr(lora.A_pack), _ptr(lora.offset),
                                     _ptr(lora.rank), lora.n_adapters, lora.R, _ptr(seg_offsets),
                                     _ptr(seg_adapter), S, wp, wb, _stream(stream)),
           "sq_lora_shrink_raw")


def sq_linear_lora_from_t(Xq, x_scale, Wq, w_scale, lora: Optional[LoraPack], Y, workspace,
                          stream=None) -> None:
    """Y = dequantized W8A8 output + T B_pack^T with T from sq_lora_shrink_raw."""
    M, K = Xq.shape
    N = Wq.shape[0]
    R = 0 if lora is None else lora.R
    B = None if lora is None else lora.B_pack
    wp, wb = _ws(workspace)
    _check(_lib().sq_linear_lora_from_t(_ptr(Xq), _ptr(x_scale), _ptr(Wq), _ptr(w_scale), M, N, K,
                                        _ptr(B), R, _ptr(Y), wp, wb, _stream(stream)),
           "sq_linear_lora_from_t")


def sq_lora_delta_from_t(Xq, N: int, lora: Optional[LoraPack], delta, workspace,
                         stream=None) -> None:
    M, K = Xq.shape
    R = 0 if lora is None else lora.R
    B = None if lora is None else lora.B_pack
    wp, wb = _ws(workspace)
    _check(_lib().sq_lora_delta_from_t(_ptr(Xq), M, N, K, _ptr(B), R, _ptr(delta), wp, wb,
                                       _stream(stream)), "sq_lora_delta_from_t")


def sq_lora_delta(Xq, x_scale, N: int, lora: Optional[LoraPack], seg_offsets, seg_adapter, delta,
                  workspace=None, stream=None) -> None:
    M, K = Xq.shape
    a, b, o, r, n_ad, R = _lora_args(lora)
    S = 0 if seg_adapter is None else seg_adapter.shape[0]
    wp, wb = _ws(workspace)
    _check(_lib().sq_lora_delta(_ptr(Xq), _ptr(x_scale), M, N, K, a, b, o, r, n_ad, R,
                                _ptr(seg_offsets), _ptr(seg_adapter), S, _ptr(delta), wp, wb,
                                _stream(stream)), "sq_lora_delta")
