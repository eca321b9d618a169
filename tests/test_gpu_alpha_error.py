"""GPU parity of the layer-wise output error for one alpha with the oracle.

"SmoothQuant" explainer, "Reading the diagnostics" (compare layer-wise output
error across alpha values) and "Variants and related ideas" (per-layer alpha
by calibration error).  The GPU's layer output Y is bf16 and its reference
X W^T fp32; the expected error takes the oracle's fp64 Y rounded to bf16
against its fp64 reference.  Bars: the reference energy to 1e-4, the error
to 1%, and the sweep picks the same alpha.
"""

import numpy as np
import pytest

import oracle
from w8a8_smoothquant_int8_b200 import workloads as wk

pytestmark = pytest.mark.gpu

ALPHAS = [0.0, 0.25, 0.5, 0.75, 1.0]


def oracle_error_bf16(X, W, alpha):
    """(sum (bf16(Y) - X W^T)^2, sum (X W^T)^2) from the oracle's steps."""
    a = oracle.act_absmax_update(X)
    s = oracle.compute_smoothing(a, oracle.weight_absmax(W), alpha)
    Wq, ws = oracle.quantize_weight(W, s)
    Xq, xs = oracle.quant_act(X, s)
    M = X.shape[0]
    so, sa = np.array([0, M], np.int32), np.array([-1], np.int32)
    Y = oracle.linear_lora_rows(Xq, xs, Wq, ws, [], [], so, sa, want=("Y",))["Y"]
    Yb = wk.bf16_bits_to_f32(wk.f32_to_bf16_bits(Y.astype(np.float32))).astype(np.float64)
    R = oracle.reference_rows(X, W, [], [], [], so, sa)
    return float(((Yb - R) ** 2).sum()), float((R ** 2).sum())


@pytest.mark.parametrize("name,rows,alphas", [
    ("tiny_m16_k256_n256", None, ALPHAS),
    ("parity_ragged", None, ALPHAS),
    ("parity_heavy_f32", None, ALPHAS),
    ("llama3_8b_qkv_m2048_k4096_n6144", 64, [0.25, 0.5, 0.75]),
])
def test_alpha_error_matches_oracle(name, rows, alphas):
    import w8a8_smoothquant_int8_b200 as sq
    from tests.gpu_pipeline import to_dev
    wl = wk.make_workload(name)
    Xc = wl.X_cal if rows is None else wl.X_cal[:rows]
    rel, best = sq.alpha_sweep(to_dev(Xc), to_dev(wl.W), alphas)
    ref_rel = []
    for i, a in enumerate(alphas):
        err, ref = oracle_error_bf16(Xc, wl.W, a)
        ref_rel.append(err / ref)
        assert abs(rel[i] - err / ref) <= 0.01 * (err / ref) + 1e-12, (a, rel[i], err / ref)
    assert best == alphas[int(np.argmin(ref_rel))]


def test_alpha_error_raw_sums():
    import torch
    import w8a8_smoothquant_int8_b200 as sq
    from tests.gpu_pipeline import to_dev
    wl = wk.make_workload("parity_ragged")
    X, W = to_dev(wl.X_cal), to_dev(wl.W)
    ws = torch.empty(sq.sq_alpha_error_workspace_size(X.shape[0], W.shape[0], X.shape[1]),
                     dtype=torch.uint8, device="cuda")
    err = torch.empty(2, dtype=torch.float64, device="cuda")
    sq.sq_alpha_output_error(X, W, 0.5, err, ws)
    e, r = err.cpu().numpy()
    oe, orf = oracle_error_bf16(wl.X_cal, wl.W, 0.5)
    assert abs(r - orf) <= 1e-4 * orf
    assert abs(e - oe) <= 0.01 * oe
    # the same call again gives the same sums (fixed reduction inputs, fresh buffer)
    sq.sq_alpha_output_error(X, W, 0.5, err, ws)
    e2, r2 = err.cpu().numpy()
    assert abs(e2 - e) <= 1e-9 * e and abs(r2 - r) <= 1e-9 * r


def test_alpha_sweep_entry_outputs():
    # the C entry's device outputs: the sums per alpha equal single calls of
    # sq_alpha_output_error, rel is their ratio, best the first minimum
    import torch
    import w8a8_smoothquant_int8_b200 as sq
    from tests.gpu_pipeline import to_dev
    wl = wk.make_workload("parity_ragged")
    X, W = to_dev(wl.X_cal), to_dev(wl.W)
    M, K, N = X.shape[0], X.shape[1], W.shape[0]
    ws = torch.empty(sq.sq_alpha_error_workspace_size(M, N, K), dtype=torch.uint8, device="cuda")
    alphas = [0.5, 0.25, 0.5, 0.75]
    err = torch.empty(2 * len(alphas), dtype=torch.float64, device="cuda")
    rel = torch.empty(len(alphas), dtype=torch.float64, device="cuda")
    best = torch.empty(1, dtype=torch.float32, device="cuda")
    sq.sq_alpha_sweep(X, W, alphas, err, rel, best, ws)
    e = err.cpu().numpy().reshape(-1, 2)
    r = rel.cpu().numpy()
    one = torch.empty(2, dtype=torch.float64, device="cuda")
    for t, a in enumerate(alphas):
        sq.sq_alpha_output_error(X, W, a, one, ws)
        # (the sums are fp64 atomics: equal up to their order of addition)
        assert np.allclose(one.cpu().numpy(), e[t], rtol=1e-9, atol=0)
        assert r[t] == e[t, 0] / e[t, 1]
    assert float(best.cpu()[0]) == alphas[int(np.argmin(r))]
