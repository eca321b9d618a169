"""GPU parity of the folded norm weight and the fused RMS norm + per-token
quantization with the oracle ("SmoothQuant" explainer, Steps 5 and 6).

The fold is bit-exact.  The fused kernel is bit-exact wherever its fp64 sum
of squares is exact; where a row's squares span more than fp64 can hold, the
oracle's in-order sum and the kernel's tree sum may round differently and
move r_i by one ulp, which can move a code near a rounding tie by one: at
most 1e-4 of the rows may differ, each by at most one code step and two ulps
of x_scale.  Through the linear layer Y stays within the 1e-2 bar.
"""

import numpy as np
import pytest

import oracle
from w8a8_smoothquant_int8_b200 import workloads as wk

pytestmark = pytest.mark.gpu

EPS = 1e-6


def _gpu_norm_quant(H, gamma, s, eps=EPS):
    import torch
    import w8a8_smoothquant_int8_b200 as sq
    from tests.gpu_pipeline import to_dev
    Hd, g, sd = to_dev(H), to_dev(gamma), to_dev(s)
    gs = torch.empty_like(g)
    sq.sq_fold_norm_weight(g, sd, gs)
    M, K = H.shape
    Xq = torch.empty((M, K), dtype=torch.int8, device="cuda")
    xs = torch.empty(M, dtype=torch.float32, device="cuda")
    sq.sq_rmsnorm_quant_act(Hd, gs, eps, Xq, xs)
    return gs.cpu().numpy(), Xq.cpu().numpy(), xs.cpu().numpy()


@pytest.mark.parametrize("name", ["parity_ragged", "parity_decode",
                                  "llama3_8b_qkv_m2048_k4096_n6144",
                                  "llama3_8b_down_m16384_k14336_n4096"])
def test_norm_fold_and_quant(name):
    wl = wk.make_workload(name)
    a = oracle.act_absmax_update(wl.X_cal)
    s = oracle.compute_smoothing(a, oracle.weight_absmax(wl.W), wl.alpha)
    gamma = wk.norm_gamma(wl.K, wl.seed)
    gs_ref = oracle.fold_norm_weight(gamma, s)
    Xq_ref, xs_ref = oracle.rmsnorm_quant_act(wl.X, gs_ref, EPS)
    gs, Xq, xs = _gpu_norm_quant(wl.X, gamma, s)
    assert np.array_equal(gs.view(np.uint32), gs_ref.view(np.uint32))
    bad = np.nonzero((xs.view(np.uint32) != xs_ref.view(np.uint32)) | (Xq != Xq_ref).any(1))[0]
    assert len(bad) <= max(1, int(1e-4 * wl.M)), bad[:10]
    for i in bad:
        assert np.abs(Xq[i].astype(np.int64) - Xq_ref[i]).max() <= 1
        assert abs(int(xs[i].view(np.int32)) - int(xs_ref[i].view(np.int32))) <= 2


def test_norm_quant_constant_and_zero_rows():
    # a constant row (every code 127, scale RN(1/127) with eps = 0) and a zero
    # row (scale 0, codes 0)
    K = 256
    H = wk.f32_to_bf16_bits(np.stack([np.full(K, 3.0), np.zeros(K)]).astype(np.float32))
    gamma = np.ones(K, np.float32)
    s = np.ones(K, np.float32)
    _, Xq, xs = _gpu_norm_quant(H, gamma, s, eps=0.0)
    assert (Xq[0] == 127).all() and xs[0] == np.float32(1.0 / 127.0)
    assert not Xq[1].any() and xs[1] == 0.0


def test_norm_fold_through_the_linear_layer():
    from tests.gpu_pipeline import GpuRun, rel_err, to_dev
    import torch
    import w8a8_smoothquant_int8_b200 as sq
    wl = wk.make_workload("llama3_8b_qkv_m2048_k4096_n6144")
    P = oracle.Prepared(wl)
    g = GpuRun(wl, s_host=P.s)
    gamma = wk.norm_gamma(wl.K, wl.seed)
    gs = torch.empty(wl.K, dtype=torch.float32, device="cuda")
    sq.sq_fold_norm_weight(to_dev(gamma), g.s, gs)
    sq.sq_rmsnorm_quant_act(g.X, gs, EPS, g.Xq, g.x_scale)
    g.linear()
    Xq, xs = oracle.rmsnorm_quant_act(wl.X, oracle.fold_norm_weight(gamma, P.s), EPS)
    rows = np.unique(np.concatenate([[0, wl.M - 1], np.random.default_rng(8).choice(wl.M, 24)]))
    ref = oracle.linear_lora_rows(Xq, xs, P.Wq, P.w_scale, P.A_s, P.B_s, wl.seg_offsets,
                                  wl.seg_adapter, rows, want=("Y",))["Y"]
    assert rel_err(g.Y_f32()[rows], ref) <= 1e-2
