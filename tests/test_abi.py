"""The C ABI library loads without a GPU, exports every entry point that
include/sq_w8a8.h declares, and rejects bad arguments on the host before any
launch (no compute call is made here).  Calls whose arguments pass the host
checks, with fake device addresses, are made only where no CUDA device is
present: there they stop at the device check; on a GPU they would reach a
kernel."""

import ctypes
import os
import re

import pytest

from w8a8_smoothquant_int8_b200 import _native, build

HEADER = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "include",
                      "sq_w8a8.h")

OK, INVALID, SHAPE, DEVICE, CUDA, TIMEOUT, WORKSPACE, SEGMENTS = range(8)


@pytest.fixture(scope="module")
def lib():
    build.build()
    return _native.load()


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(sq_[a-z0-9_]+)\s*\(", text)))


def test_header_declares_the_boundary():
    names = declared_functions()
    for required in ("sq_compute_smoothing", "sq_quantize_weight", "sq_quant_act", "sq_linear_lora"):
        assert required in names


def test_library_exports_every_declared_symbol(lib):
    names = declared_functions()
    assert len(names) >= 15
    for n in names:
        assert hasattr(lib, n), n
        assert n in _native.SIGNATURES, n


def test_status_strings(lib):
    for code in range(8):
        assert lib.sq_status_string(code)
    assert b"unknown" in lib.sq_status_string(99)
    assert lib.sq_version() >= 100


def test_workspace_size(lib):
    assert lib.sq_linear_lora_workspace_size(2048, 0) == 0
    assert lib.sq_linear_lora_workspace_size(0, 16) == 0
    ws = lib.sq_linear_lora_workspace_size(2048, 16)
    assert ws >= 2 * 2048 * 16 * 2 + 16 * 8 and ws % 256 == 0


A = 1 << 20  # a 16-byte-aligned fake address: never dereferenced, validation fails first


def _no_device():
    try:
        import torch
        return not torch.cuda.is_available()
    except Exception:
        return True


NO_DEVICE = _no_device()


def test_quant_act_validation(lib):
    f = lib.sq_quant_act
    assert f(A, 1, A, 4, 15, A, A, None) == SHAPE          # K % 16
    assert f(A, 1, A, 4, 57344 + 16, A, A, None) == SHAPE  # K too large
    assert f(A, 1, A, -1, 16, A, A, None) == INVALID       # negative M
    assert f(A, 7, A, 4, 16, A, A, None) == INVALID        # dtype
    assert f(A + 8, 1, A, 4, 16, A, A, None) == INVALID    # misaligned X
    assert f(None, 1, A, 4, 16, A, A, None) == INVALID     # null X
    # well-formed arguments reach the device check: no device here
    if NO_DEVICE:
        assert f(A, 1, A, 4, 16, A, A, None) in (CUDA, DEVICE)


def test_linear_lora_validation(lib):
    f = lib.sq_linear_lora
    ws = lib.sq_linear_lora_workspace_size(256, 32)
    args = dict(Xq=A, xs=A, Wq=A, ws_=A, M=256, N=512, K=1024, Ap=A, Bp=A, off=A, rk=A, nad=2, R=32,
                so=A, sa=A, S=3, Y=A, w=A, wb=ws, st=None)

    def call(**kw):
        a = dict(args, **kw)
        return f(a["Xq"], a["xs"], a["Wq"], a["ws_"], a["M"], a["N"], a["K"], a["Ap"], a["Bp"], a["off"],
                 a["rk"], a["nad"], a["R"], a["so"], a["sa"], a["S"], a["Y"], a["w"], a["wb"], a["st"])

    assert call(N=100) == SHAPE               # N % 16
    assert call(K=1000) == SHAPE              # K % 16
    assert call(R=24) == SHAPE                # R % 16
    assert call(R=2048) == SHAPE              # R > 1024
    assert call(nad=-1) == INVALID
    assert call(wb=ws - 1) == WORKSPACE
    assert call(w=A + 16) == WORKSPACE        # workspace must be 256-byte aligned
    assert call(w=None) == WORKSPACE
    assert call(Bp=None) == INVALID
    assert call(Y=A + 4) == INVALID
    if NO_DEVICE:
        assert call() in (CUDA, DEVICE)
    # no LoRA: the LoRA pointers and the workspace may be null
    if NO_DEVICE:
        assert call(R=0, Ap=None, Bp=None, off=None, rk=None, so=None, sa=None, S=0, w=None, wb=0) in (CUDA, DEVICE)


def test_offline_validation(lib):
    assert lib.sq_compute_smoothing(A, A, 64, 1.5, A, None) == INVALID
    assert lib.sq_compute_smoothing(A, A, 64, -0.1, A, None) == INVALID
    assert lib.sq_quantize_weight(A, A, 8, 24, A, A, None) == SHAPE
    assert lib.sq_prepare_lora(A, A, A, 8, 64, 32, 16.0, 16, 8, A, A, None) == SHAPE   # off % 16
    assert lib.sq_prepare_lora(A, A, A, 20, 64, 32, 16.0, 16, 0, A, A, None) == INVALID  # r > R
    assert lib.sq_prepare_lora(A, A, A, 0, 64, 32, 16.0, 16, 0, A, A, None) == INVALID
    assert lib.sq_set_wait_timeout_ns(0) == INVALID
    code = ctypes.c_int(0)
    assert lib.sq_get_device_error(None, 0) == INVALID


def test_raw_lora_entry_validation(lib):
    # raw-input reading of the LoRA path: T from bf16 activations, then Y
    assert lib.sq_lora_t_workspace_size(0, 16) == 0
    assert lib.sq_lora_t_workspace_size(64, 0) == 0
    tws = lib.sq_lora_t_workspace_size(64, 32)   # any M: no decode special case
    assert tws >= 2 * 64 * 32 * 2 + 4 * 8 and tws % 256 == 0
    f = lib.sq_lora_shrink_raw
    good = (A, 64, 1024, A, A, A, 2, 32, A, A, 3, A, tws, None)

    def shrink(**kw):
        names = ("X", "M", "K", "Ap", "off", "rk", "nad", "R", "so", "sa", "S", "w", "wb", "st")
        a = dict(zip(names, good), **kw)
        return f(*[a[n] for n in names])

    assert shrink(K=1000) == SHAPE
    assert shrink(R=24) == SHAPE
    assert shrink(R=0) == INVALID
    assert shrink(wb=tws - 1) == WORKSPACE
    assert shrink(w=A + 16) == WORKSPACE
    assert shrink(X=A + 2) == INVALID
    assert shrink(off=None) == INVALID
    if NO_DEVICE:
        assert shrink() in (CUDA, DEVICE)
    g = lib.sq_linear_lora_from_t
    assert g(A, A, A, A, 64, 100, 1024, A, 32, A, A, tws, None) == SHAPE      # N % 16
    assert g(A, A, A, A, 64, 128, 1024, A, 24, A, A, tws, None) == SHAPE      # R % 16
    assert g(A, A, A, A, 64, 128, 1024, None, 32, A, A, tws, None) == INVALID  # B_pack
    assert g(A, A, A, A, 64, 128, 1024, A, 32, A, A, tws - 1, None) == WORKSPACE
    if NO_DEVICE:
        assert g(A, A, A, A, 64, 128, 1024, A, 32, A, A, tws, None) in (CUDA, DEVICE)
    if NO_DEVICE:
        assert g(A, A, A, A, 64, 128, 1024, None, 0, A, None, 0, None) in (CUDA, DEVICE)  # plain W8A8
    h = lib.sq_lora_delta_from_t
    assert h(A, 64, 128, 1024, A, 32, A + 4, A, tws, None) == INVALID        # delta alignment
    if NO_DEVICE:
        assert h(A, 64, 128, 1024, A, 32, A, A, tws, None) in (CUDA, DEVICE)
    # s == NULL is the raw-input packing (A unchanged), not an argument error
    if NO_DEVICE:
        assert lib.sq_prepare_lora(A, A, None, 8, 64, 32, 16.0, 16, 0, A, A, None) in (CUDA, DEVICE)


def test_static_quant_entry_validation(lib):
    assert lib.sq_static_act_scale(A, A, 1000, A, None) == SHAPE        # K % 16
    assert lib.sq_static_act_scale(A, A, 0, A, None) == INVALID
    assert lib.sq_static_act_scale(A, A, 64, A + 2, None) == INVALID    # scale alignment
    if NO_DEVICE:
        assert lib.sq_static_act_scale(A, A, 64, A, None) in (CUDA, DEVICE)
    f = lib.sq_quant_act_static
    assert f(A, 1, A, A, 64, 1000, A, A, A, None) == SHAPE               # K % 16
    assert f(A, 7, A, A, 64, 1024, A, A, A, None) == INVALID             # dtype
    assert f(A, 1, A, A, 64, 1024, A, A, A + 4, None) == INVALID         # counter alignment
    assert f(A, 1, A, None, 64, 1024, A, A, A, None) == INVALID
    assert f(A + 2, 1, A, A, 64, 1024, A, A, A, None) == INVALID
    if NO_DEVICE:
        assert f(A, 1, A, A, 64, 1024, A, A, A, None) in (CUDA, DEVICE)


def test_alpha_error_entry_validation(lib):
    assert lib.sq_alpha_error_workspace_size(0, 64, 64) == 0
    wsz = lib.sq_alpha_error_workspace_size(64, 128, 256)
    assert wsz >= 128 * 256 + 64 * 256 + 2 * 64 * 128 and wsz % 256 == 0
    f = lib.sq_alpha_output_error
    assert f(A, 1, A, 64, 128, 1000, 0.5, A, A, wsz, None) == SHAPE    # K % 16
    assert f(A, 1, A, 64, 100, 256, 0.5, A, A, wsz, None) == SHAPE     # N % 16
    assert f(A, 1, A, 64, 128, 256, 1.5, A, A, wsz, None) == INVALID   # alpha
    assert f(A, 1, A, 64, 128, 256, 0.5, A + 4, A, wsz, None) == INVALID  # err alignment
    assert f(A, 1, A, 64, 128, 256, 0.5, A, A, wsz - 1, None) == WORKSPACE
    if NO_DEVICE:
        assert f(A, 1, A, 64, 128, 256, 0.5, A, A, wsz, None) in (CUDA, DEVICE)


def test_pack_lora_entry_validation(lib):
    def i64(*v):
        return (ctypes.c_int64 * len(v))(*v)

    def ptrs(n, v=A):
        return (ctypes.c_void_p * n)(*([v] * n))

    def f32(*v):
        return (ctypes.c_float * len(v))(*v)

    assert lib.sq_lora_pack_width(i64(8, 16, 64), 3) == 96
    assert lib.sq_lora_pack_width(i64(8, 0), 2) == -1
    assert lib.sq_lora_pack_width(i64(257), 1) == -1
    f = lib.sq_pack_lora
    r, al = i64(8, 16, 64), f32(16.0, 32.0, 128.0)
    if NO_DEVICE:
        assert f(ptrs(3), ptrs(3), r, al, 3, A, 256, 64, 96, A, A, A, A, None) in (CUDA, DEVICE)
    assert f(ptrs(3), ptrs(3), r, al, 3, A, 256, 64, 80, A, A, A, A, None) == INVALID  # R
    assert f(ptrs(3), ptrs(3), r, al, 3, A, 250, 64, 96, A, A, A, A, None) == SHAPE    # K % 16
    assert f(ptrs(3), ptrs(3, None), r, al, 3, A, 256, 64, 96, A, A, A, A, None) == INVALID
    assert f(ptrs(3), ptrs(3), r, al, 0, A, 256, 64, 96, A, A, A, A, None) == INVALID
    wide = i64(*([256] * 5))
    assert f(ptrs(5), ptrs(5), wide, f32(*([1.0] * 5)), 5, A, 256, 64, 1280, A, A, A, A,
             None) == SHAPE


def test_alpha_sweep_entry_validation(lib):
    wsz = lib.sq_alpha_error_workspace_size(64, 128, 256)
    f = lib.sq_alpha_sweep

    def alphas(*v):
        return (ctypes.c_float * max(1, len(v)))(*v)

    good = alphas(0.0, 0.5, 1.0)
    assert f(A, 1, A, 64, 128, 256, good, 0, A, A, A, A, wsz, None) == INVALID    # no alpha
    assert f(A, 1, A, 64, 128, 256, alphas(*([0.5] * 65)), 65, A, A, A, A, wsz, None) == INVALID
    assert f(A, 1, A, 64, 128, 256, alphas(0.5, -0.1), 2, A, A, A, A, wsz, None) == INVALID
    assert f(A, 1, A, 64, 128, 256, None, 3, A, A, A, A, wsz, None) == INVALID
    assert f(A, 1, A, 64, 100, 256, good, 3, A, A, A, A, wsz, None) == SHAPE      # N % 16
    assert f(A, 1, A, 64, 128, 256, good, 3, A + 4, A, A, A, wsz, None) == INVALID  # err align
    assert f(A, 1, A, 64, 128, 256, good, 3, A, A, A, A, wsz - 1, None) == WORKSPACE
    if NO_DEVICE:
        assert f(A, 1, A, 64, 128, 256, good, 3, A, A, A, A, wsz, None) in (CUDA, DEVICE)


def test_norm_fold_entry_validation(lib):
    assert lib.sq_fold_norm_weight(A, A, 1000, A, None) == SHAPE
    assert lib.sq_fold_norm_weight(A + 4, A, 64, A, None) == INVALID
    if NO_DEVICE:
        assert lib.sq_fold_norm_weight(A, A, 64, A, None) in (CUDA, DEVICE)
    f = lib.sq_rmsnorm_quant_act
    assert f(A, A, 1e-6, 64, 1000, A, A, None) == SHAPE         # K % 16
    assert f(A, A, 1e-6, 64, 65536, A, A, None) == SHAPE        # beyond 32768 channels
    assert f(A, A, -1.0, 64, 1024, A, A, None) == INVALID       # eps < 0
    assert f(A + 2, A, 1e-6, 64, 1024, A, A, None) == INVALID
    if NO_DEVICE:
        assert f(A, A, 1e-6, 64, 1024, A, A, None) in (CUDA, DEVICE)
