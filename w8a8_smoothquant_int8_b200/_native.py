"""ctypes view of libsq_w8a8.so (the C ABI declared in include/sq_w8a8.h).

The library must exist; there is no fallback.  A missing or unloadable
library raises at import of the first call.
"""

from __future__ import annotations

import ctypes
import os

from .build import LIB

P = ctypes.c_void_p
I64 = ctypes.c_int64
I32 = ctypes.c_int
U64 = ctypes.c_uint64
F32 = ctypes.c_float
SZ = ctypes.c_size_t

# name -> (argtypes, restype); mirrors include/sq_w8a8.h
SIGNATURES = {
    "sq_status_string": ([I32], ctypes.c_char_p),
    "sq_version": ([], I32),
    "sq_device_supported": ([I32], I32),
    "sq_get_device_error": ([ctypes.POINTER(I32), I32], I32),
    "sq_set_wait_timeout_ns": ([U64], I32),
    "sq_set_gemm_events": ([P, P], I32),
    "sq_selftest_wait_timeout": ([U64, P], I32),
    "sq_act_absmax_update": ([P, I32, I64, I64, P, P], I32),
    "sq_weight_absmax": ([P, I64, I64, P, P], I32),
    "sq_compute_smoothing": ([P, P, I64, F32, P, P], I32),
    "sq_quantize_weight": ([P, P, I64, I64, P, P, P], I32),
    "sq_prepare_lora": ([P, P, P, I64, I64, I64, F32, I64, I64, P, P, P], I32),
    "sq_lora_pack_width": ([P, I32], I64),
    "sq_pack_lora": ([P, P, P, P, I32, P, I64, I64, I64, P, P, P, P, P], I32),
    "sq_quant_act": ([P, I32, P, I64, I64, P, P, P], I32),
    "sq_linear_lora_workspace_size": ([I64, I64], SZ),
    "sq_linear_lora": ([P, P, P, P, I64, I64, I64, P, P, P, P, I32, I64, P, P, I64, P, P, SZ, P],
                       I32),
    "sq_linear_lora_noalloc": ([P, P, P, P, I64, I64, I64, P, P, P, P, I32, I64, P, P, I64, P, P],
                               I32),
    "sq_gemm_i32": ([P, P, I64, I64, I64, P, P], I32),
    "sq_lora_delta": ([P, P, I64, I64, I64, P, P, P, P, I32, I64, P, P, I64, P, P, SZ, P], I32),
    "sq_lora_t_workspace_size": ([I64, I64], SZ),
    "sq_fold_norm_weight": ([P, P, I64, P, P], I32),
    "sq_rmsnorm_quant_act": ([P, P, F32, I64, I64, P, P, P], I32),
    "sq_alpha_error_workspace_size": ([I64, I64, I64], SZ),
    "sq_alpha_output_error": ([P, I32, P, I64, I64, I64, F32, P, P, SZ, P], I32),
    "sq_alpha_sweep": ([P, I32, P, I64, I64, I64, P, I32, P, P, P, P, SZ, P], I32),
    "sq_static_act_scale": ([P, P, I64, P, P], I32),
    "sq_quant_act_static": ([P, I32, P, P, I64, I64, P, P, P, P], I32),
    "sq_lora_shrink_raw": ([P, I64, I64, P, P, P, I32, I64, P, P, I64, P, SZ, P], I32),
    "sq_linear_lora_from_t": ([P, P, P, P, I64, I64, I64, P, I64, P, P, SZ, P], I32),
    "sq_lora_delta_from_t": ([P, I64, I64, I64, P, I64, P, P, SZ, P], I32),
}

_lib = None


def load(path: str = LIB):
    global _lib
    if _lib is None:
        if not os.path.exists(path):
            raise RuntimeError(
                f"CUDA library {path} is not built; run `python -m w8a8_smoothquant_int8_b200.build`")
        lib = ctypes.CDLL(path)
        for name, (args, res) in SIGNATURES.items():
            fn = getattr(lib, name)
            fn.argtypes = args
            fn.restype = res
        _lib = lib
    return _lib
