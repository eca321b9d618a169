"""GPU parity of the per-tensor static activation quantization with the oracle.

"SmoothQuant" explainer, Step 6 and "Calibration in practice": one activation
scale for every token, fixed offline from the calibration range.  Bars: the
scale, the codes and the per-token scales bit-exact, the clipped-code count
exact; the static codes through the fused linear layer within the Y bar.
"""

import numpy as np
import pytest

import oracle
from w8a8_smoothquant_int8_b200 import workloads as wk

pytestmark = pytest.mark.gpu

Y_TOL = 1e-2


def _gpu_static(X_host, s_host, act_absmax_host):
    import torch
    import w8a8_smoothquant_int8_b200 as sq
    from tests.gpu_pipeline import to_dev
    X = to_dev(X_host)
    s = to_dev(s_host)
    a = to_dev(act_absmax_host)
    scale = torch.empty(1, dtype=torch.float32, device="cuda")
    sq.sq_static_act_scale(a, s, scale)
    M, K = X_host.shape
    Xq = torch.empty((M, K), dtype=torch.int8, device="cuda")
    xs = torch.empty(M, dtype=torch.float32, device="cuda")
    cnt = torch.zeros(1, dtype=torch.int64, device="cuda")
    sq.sq_quant_act_static(X, s, scale, Xq, xs, cnt)
    return (scale.cpu().numpy()[0], Xq.cpu().numpy(), xs.cpu().numpy(), int(cnt.cpu().numpy()[0]))


NAMES = ["tiny_m16_k256_n256", "parity_ragged", "parity_heavy_f32", "parity_decode",
         "llama3_8b_qkv_m2048_k4096_n6144", "llama3_8b_gateup_m8192_k4096_n28672",
         "llama3_8b_down_m16384_k14336_n4096"]


@pytest.mark.parametrize("name", NAMES)
def test_static_quant_bit_exact(name):
    wl = wk.make_workload(name)
    a = oracle.act_absmax_update(wl.X_cal)
    s = oracle.compute_smoothing(a, oracle.weight_absmax(wl.W), wl.alpha)
    scale = oracle.static_act_scale(a, s)
    Xq, xs, clipped = oracle.quant_act_static(wl.X, s, scale)
    g_scale, g_Xq, g_xs, g_clipped = _gpu_static(wl.X, s, a)
    assert np.float32(g_scale).view(np.uint32) == np.float32(scale).view(np.uint32)
    assert np.array_equal(g_xs.view(np.uint32), xs.view(np.uint32))
    assert np.array_equal(g_Xq, Xq)
    assert g_clipped == clipped


def test_static_quant_range_edge_and_zero_scale():
    # scale 2^-4: 127.5 -> 128 (even) is clipped, 126.5 -> 126, -128.5 -> -128
    K = 16
    X = np.zeros((3, K), np.float32)
    X[0, :5] = np.array([127.5, 126.5, -128.5, -129.5, 1e30], np.float32) / 16
    X[1, :] = np.arange(K, dtype=np.float32) - 8
    s = np.ones(K, np.float32)
    a = np.full(K, 127.0 / 16, np.float32)          # static scale exactly 2^-4
    g_scale, g_Xq, _, g_clipped = _gpu_static(X, s, a)
    assert g_scale == np.float32(2.0 ** -4)
    Xq, _, clipped = oracle.quant_act_static(X, s, np.float32(2.0 ** -4))
    assert np.array_equal(g_Xq, Xq) and g_clipped == clipped
    assert g_Xq[0, :5].tolist() == [127, 126, -128, -128, 127]
    # zero calibration range: scale 0, codes 0, every nonzero value counted
    g_scale, g_Xq, g_xs, g_clipped = _gpu_static(X, s, np.zeros(K, np.float32))
    assert g_scale == 0.0 and not g_Xq.any() and not g_xs.any()
    assert g_clipped == int(np.count_nonzero(X))


@pytest.mark.parametrize("name", ["parity_ragged", "llama3_8b_qkv_m2048_k4096_n6144"])
def test_static_codes_through_the_linear_layer(name):
    import torch
    import w8a8_smoothquant_int8_b200 as sq
    from tests.gpu_pipeline import GpuRun, rel_err, to_dev
    wl = wk.make_workload(name)
    P = oracle.Prepared(wl)
    g = GpuRun(wl, s_host=P.s)
    scale = torch.empty(1, dtype=torch.float32, device="cuda")
    sq.sq_static_act_scale(to_dev(P.act_absmax), g.s, scale)
    cnt = torch.zeros(1, dtype=torch.int64, device="cuda")
    sq.sq_quant_act_static(g.X, g.s, scale, g.Xq, g.x_scale, cnt)
    g.linear()
    Xq, xs, _ = oracle.quant_act_static(wl.X, P.s, oracle.static_act_scale(P.act_absmax, P.s))
    rows = np.unique(np.concatenate([[0, wl.M - 1], np.random.default_rng(5).choice(wl.M, 24)]))
    ref = oracle.linear_lora_rows(Xq, xs, P.Wq, P.w_scale, P.A_s, P.B_s, wl.seg_offsets,
                                  wl.seg_adapter, rows, want=("Y",))["Y"]
    assert rel_err(g.Y_f32()[rows], ref) <= Y_TOL
