"""Edge cases of the CUDA path, checked against the CPU oracle.

Quantizer: exact round-half-even ties, values a hair either side of a tie,
zero and single-value rows, huge outliers next to tiny values, values whose
quotient leaves the normal range, f32 and bf16 inputs.  Linear layer: empty
M / N / K, no adapters, segments without adapters, an out-of-range adapter
index (reported on the device, treated as no adapter).
"""

import numpy as np
import pytest

import oracle
from w8a8_smoothquant_int8_b200 import workloads as wk

pytestmark = pytest.mark.gpu


def _gpu_quant(X, s):
    import torch
    import w8a8_smoothquant_int8_b200 as sq
    from tests.gpu_pipeline import to_dev
    Xd, sd = to_dev(X), to_dev(s)
    M, K = X.shape
    Xq = torch.empty((M, K), dtype=torch.int8, device="cuda")
    xs = torch.empty(M, dtype=torch.float32, device="cuda")
    sq.sq_quant_act(Xd, sd, Xq, xs)
    return Xq.cpu().numpy(), xs.cpu().numpy()


def _check_quant(X, s):
    Xq, xs = _gpu_quant(X, s)
    oq, oxs = oracle.quant_act(X, s)
    assert np.array_equal(xs.view(np.uint32), oxs.view(np.uint32))
    bad = np.argwhere(Xq != oq)
    assert bad.size == 0, f"{len(bad)} codes differ, first {bad[:5].tolist()}"


def test_quant_exact_ties():
    halves = np.array([0.5, 1.5, 2.5, 3.5, -0.5, -1.5, -2.5, 126.5, -126.5, 64.5, -64.5, 7.5],
                      np.float32)
    row = np.concatenate([[127.0], halves, np.zeros(3)]).astype(np.float32) / np.float32(16)
    X = np.stack([row, -row, row * 4, row / 1024])
    _check_quant(X, np.ones(X.shape[1], np.float32))


def test_quant_near_ties():
    rng = np.random.default_rng(21)
    M, K = 64, 512
    scale = np.float32(2.0 ** -5)
    n = rng.integers(-126, 126, (M, K)).astype(np.float32)
    ulps = rng.integers(-200, 200, (M, K)).astype(np.float32)
    X = ((n + np.float32(0.5)) * scale).astype(np.float32)
    X = (X + ulps * np.spacing(np.abs(X)).astype(np.float32)).astype(np.float32)
    X[:, 0] = 127 * scale  # fixes the row scale at 2^-5
    _check_quant(X, np.ones(K, np.float32))
    # the same with a non-trivial smoothing scale (quotients no longer exact)
    s = rng.uniform(0.5, 2.0, K).astype(np.float32)
    _check_quant((X * s).astype(np.float32), s)


def test_quant_zero_single_and_extreme_rows():
    K = 256
    rng = np.random.default_rng(5)
    X = rng.standard_normal((8, K)).astype(np.float32)
    X[0] = 0.0                       # all-zero row: scale 0, codes 0
    X[1] = 0.0
    X[1, 17] = -3.0                  # single value
    X[2, 5] = 1e30                   # huge outlier next to ordinary values
    X[3] *= 1e-38                    # tiny values (subnormal quotients)
    X[4] = np.float32(3e38) * np.sign(X[4])  # near the top of the range
    X[5, ::2] = -0.0
    s = rng.uniform(0.01, 100, K).astype(np.float32)
    _check_quant(X, s)
    _check_quant(X, np.ones(K, np.float32))


def test_quant_bf16_wide_smoothing_range():
    rng = np.random.default_rng(8)
    M, K = 96, 1024
    X = wk.f32_to_bf16_bits(rng.standard_normal((M, K)).astype(np.float32) *
                            rng.choice([1, 1, 1, 80], K).astype(np.float32))
    s = (10.0 ** rng.uniform(-5, 5, K)).astype(np.float32)
    _check_quant(X, s)


def _linear_case(M, N, K, ranks=(16,), seg=None, ad=None):
    import torch
    import w8a8_smoothquant_int8_b200 as sq
    from tests.gpu_pipeline import to_dev
    rng = np.random.default_rng(M * 7 + N * 3 + K)
    X = wk.f32_to_bf16_bits(rng.standard_normal((M, K)).astype(np.float32))
    W = wk.f32_to_bf16_bits(rng.standard_normal((N, K)).astype(np.float32) * 0.02)
    s = rng.uniform(0.5, 2, K).astype(np.float32)
    Wq, ws = oracle.quantize_weight(W, s)
    Xq, xs = oracle.quant_act(X, s)
    As = [wk.f32_to_bf16_bits(rng.standard_normal((r, K)).astype(np.float32) / r) for r in ranks]
    Bs = [wk.f32_to_bf16_bits(rng.standard_normal((N, r)).astype(np.float32) * 0.01) for r in ranks]
    seg = np.array([0, M] if seg is None else seg, np.int32)
    ad = np.array([0] if ad is None else ad, np.int32)

    def dev(a, dtype):
        t = torch.empty(a.shape, dtype=dtype, device="cuda")
        if a.size:
            t.copy_(to_dev(a).view(dtype) if a.dtype == np.uint16 else to_dev(a))
        return t

    lora = None
    if ranks and K and N:
        lora = sq.LoraPack.build([to_dev(a) for a in As], [to_dev(b) for b in Bs],
                                 [2.0 * r for r in ranks], to_dev(s))
    R = lora.R if lora else 0
    ws_buf = torch.empty(max(sq.sq_linear_lora_workspace_size(M, R), 256), dtype=torch.uint8,
                         device="cuda")
    Y = torch.full((max(M, 1), max(N, 1)), 7.0, dtype=torch.bfloat16, device="cuda")[:M, :N]
    sq.sq_linear_lora(dev(Xq, torch.int8), dev(xs, torch.float32), dev(Wq, torch.int8),
                      dev(ws, torch.float32), lora, to_dev(seg), to_dev(ad), Y, ws_buf)
    torch.cuda.synchronize()
    A_s, B_s = [], []
    for a, b, r in zip(As, Bs, ranks):
        x, y = oracle.prepare_lora(a, b, s, 2.0 * r)
        A_s.append(x)
        B_s.append(y)
    ref = (oracle.linear_lora_rows(Xq, xs, Wq, ws, A_s, B_s, seg, ad, want=("Y",))["Y"]
           if M and N else np.zeros((M, N)))
    return Y.float().cpu().numpy(), ref


def test_linear_empty_shapes():
    for M, N, K in [(0, 64, 64), (32, 0, 64)]:
        Y, ref = _linear_case(M, N, K)
        assert Y.shape == (M, N)
    Y, ref = _linear_case(40, 48, 0, ranks=())
    assert not Y.any()


def test_linear_no_adapters_and_none_segments():
    from tests.gpu_pipeline import rel_err
    Y, ref = _linear_case(200, 272, 160, ranks=())
    assert rel_err(Y, ref) <= 1e-2
    Y, ref = _linear_case(200, 272, 160, ranks=(16, 32), seg=[0, 50, 120, 200], ad=[-1, -1, -1])
    assert rel_err(Y, ref) <= 1e-2


def test_linear_bad_adapter_index_is_reported():
    import w8a8_smoothquant_int8_b200 as sq
    from tests.gpu_pipeline import rel_err
    sq.sq_get_device_error(clear=True)
    # rows of the segment naming adapter 5 (of 1) get no LoRA, as in the oracle
    Y, ref = _linear_case(130, 256, 128, ranks=(16,), seg=[0, 60, 130], ad=[0, 5])
    assert rel_err(Y, ref) <= 1e-2
    assert sq.sq_get_device_error(clear=True) == 7  # SQ_ERR_BAD_SEGMENTS
    assert sq.sq_get_device_error(clear=True) == 0
