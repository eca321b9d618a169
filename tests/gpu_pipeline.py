"""Run a workload through the CUDA library's C ABI (via the Python binding)
and bring the results back as numpy arrays.  Test helper; GPU only."""

from __future__ import annotations

import numpy as np
import torch

import w8a8_smoothquant_int8_b200 as sq
from w8a8_smoothquant_int8_b200 import workloads as wk


def to_dev(a: np.ndarray, dtype=None) -> torch.Tensor:
    t = torch.from_numpy(np.ascontiguousarray(a))
    if a.dtype == np.uint16:
        t = t.view(torch.bfloat16)
    if dtype is not None:
        t = t.to(dtype)
    return t.cuda()


def bf16_bits(t: torch.Tensor) -> np.ndarray:
    return t.contiguous().view(torch.int16).cpu().numpy().view(np.uint16)


class GpuRun:
    """Every step of the hot path and its offline preparation on the GPU."""

    def __init__(self, wl: wk.Workload, s_host: np.ndarray = None):
        self.wl = wl
        M, K, N = wl.M, wl.K, wl.N
        dev = torch.device("cuda")
        self.X = to_dev(wl.X)
        self.X_cal = to_dev(wl.X_cal)
        self.W = to_dev(wl.W)
        self.act_absmax = torch.zeros(K, dtype=torch.float32, device=dev)
        sq.sq_act_absmax_update(self.X_cal, self.act_absmax)
        self.w_absmax = torch.empty(K, dtype=torch.float32, device=dev)
        sq.sq_weight_absmax(self.W, self.w_absmax)
        self.s_gpu = torch.empty(K, dtype=torch.float32, device=dev)
        sq.sq_compute_smoothing(self.act_absmax, self.w_absmax, wl.alpha, self.s_gpu)
        # downstream steps take a given s (the oracle's) so that their outputs
        # can be compared bit for bit; pow is not correctly rounded anywhere
        self.s = self.s_gpu if s_host is None else to_dev(s_host)
        self.Wq = torch.empty((N, K), dtype=torch.int8, device=dev)
        self.w_scale = torch.empty(N, dtype=torch.float32, device=dev)
        sq.sq_quantize_weight(self.W, self.s, self.Wq, self.w_scale)
        self.As = [to_dev(a.A) for a in wl.adapters]
        self.Bs = [to_dev(a.B) for a in wl.adapters]
        self.lora = (sq.LoraPack.build(self.As, self.Bs, [a.lora_alpha for a in wl.adapters], self.s)
                     if wl.adapters else None)
        self.seg_offsets = to_dev(wl.seg_offsets)
        self.seg_adapter = to_dev(wl.seg_adapter)
        self.Xq = torch.empty((M, K), dtype=torch.int8, device=dev)
        self.x_scale = torch.empty(M, dtype=torch.float32, device=dev)
        R = self.lora.R if self.lora else 0
        self.workspace = torch.empty(max(sq.sq_linear_lora_workspace_size(M, R), 256),
                                     dtype=torch.uint8, device=dev)
        self.Y = torch.empty((M, N), dtype=torch.bfloat16, device=dev)

    def quant(self):
        sq.sq_quant_act(self.X, self.s, self.Xq, self.x_scale)

    def linear(self):
        sq.sq_linear_lora(self.Xq, self.x_scale, self.Wq, self.w_scale, self.lora, self.seg_offsets,
                          self.seg_adapter, self.Y, self.workspace)

    def step(self):
        self.quant()
        self.linear()

    def gemm_i32(self) -> np.ndarray:
        acc = torch.empty((self.wl.M, self.wl.N), dtype=torch.int32, device="cuda")
        sq.sq_gemm_i32(self.Xq, self.Wq, acc)
        return acc.cpu().numpy()

    def delta(self) -> np.ndarray:
        d = torch.empty((self.wl.M, self.wl.N), dtype=torch.float32, device="cuda")
        sq.sq_lora_delta(self.Xq, self.x_scale, self.wl.N, self.lora, self.seg_offsets,
                         self.seg_adapter, d, self.workspace)
        return d.cpu().numpy()

    def Y_f32(self) -> np.ndarray:
        return self.Y.float().cpu().numpy()


def rel_err(got: np.ndarray, ref: np.ndarray) -> float:
    den = np.abs(ref).max()
    return float(np.abs(got.astype(np.float64) - ref).max() / (den if den > 0 else 1.0))


def ulp_diff_f32(a: np.ndarray, b: np.ndarray) -> int:
    ia = a.astype(np.float32).view(np.int32).astype(np.int64)
    ib = b.astype(np.float32).view(np.int32).astype(np.int64)
    return int(np.abs(ia - ib).max()) if ia.size else 0
