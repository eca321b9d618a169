"""GPU parity of the raw-input reading of the LoRA path with the oracle.

"[Feature]: LoRA support for W8A8 SmoothQuant", Pitch (LoRA in BF16 after the
INT8 GEMM, added to the dequantized output) read on the layer's own bf16
activations: T = X A^T (sq_lora_shrink_raw, adapters packed with s == NULL),
then Y = dequantized W8A8 output + T B_pack^T (sq_linear_lora_from_t).
Bars as for the graded path: the packed A bit-exact, Y within
max|Y-Y_ref|/max|Y_ref| <= 1e-2, the delta alone within 5e-3.
"""

import numpy as np
import pytest

import oracle
from w8a8_smoothquant_int8_b200 import workloads as wk

pytestmark = pytest.mark.gpu

Y_TOL = 1e-2
DELTA_TOL = 5e-3


class RawRun:
    def __init__(self, name, **kw):
        import torch
        import w8a8_smoothquant_int8_b200 as sq
        from tests.gpu_pipeline import GpuRun, to_dev
        self.sq, self.torch = sq, torch
        self.wl = wk.make_workload(name, **kw)
        self.P = oracle.Prepared(self.wl)
        self.g = GpuRun(self.wl, s_host=self.P.s)
        self.g.quant()
        wl = self.wl
        self.lora = sq.LoraPack.build(self.g.As, self.g.Bs, [a.lora_alpha for a in wl.adapters], None)
        self.ws = torch.empty(max(sq.sq_lora_t_workspace_size(wl.M, self.lora.R), 256),
                              dtype=torch.uint8, device="cuda")
        self.X = to_dev(wl.X)

    def shrink(self, seg_adapter=None):
        sa = self.g.seg_adapter if seg_adapter is None else seg_adapter
        self.sq.sq_lora_shrink_raw(self.X, self.lora, self.g.seg_offsets, sa, self.ws)

    def Y(self):
        self.sq.sq_linear_lora_from_t(self.g.Xq, self.g.x_scale, self.g.Wq, self.g.w_scale,
                                      self.lora, self.g.Y, self.ws)
        return self.g.Y.float().cpu().numpy()

    def delta(self):
        d = self.torch.empty((self.wl.M, self.wl.N), dtype=self.torch.float32, device="cuda")
        self.sq.sq_lora_delta_from_t(self.g.Xq, self.wl.N, self.lora, d, self.ws)
        return d.cpu().numpy()

    def ref(self, rows=None, want=("Y", "delta"), seg_adapter=None):
        wl, P = self.wl, self.P
        sa = wl.seg_adapter if seg_adapter is None else seg_adapter
        A_raw = [a.A for a in wl.adapters]
        return oracle.linear_lora_raw_rows(wl.X, P.Xq, P.x_scale, P.Wq, P.w_scale, A_raw, P.B_s,
                                           wl.seg_offsets, sa, rows, want)


SMALL = ["parity_ragged", "parity_decode", "parity_segments_large"]


@pytest.fixture(scope="module", params=SMALL)
def small(request):
    return RawRun(request.param)


def test_raw_pack_keeps_A_bit_exact(small):
    from tests.gpu_pipeline import bf16_bits
    wl, lora = small.wl, small.lora
    offs, _ = small.sq.LoraPack.layout([a.r for a in wl.adapters])
    A_pack = bf16_bits(lora.A_pack)
    B_pack = bf16_bits(lora.B_pack)
    for a, off in zip(wl.adapters, offs):
        A_raw, B_s = oracle.prepare_lora(a.A, a.B, None, a.lora_alpha)
        assert np.array_equal(A_pack[off:off + a.r], A_raw)
        assert np.array_equal(B_pack[:, off:off + a.r], B_s)
        rpad = (a.r + 15) // 16 * 16
        assert not A_pack[off + a.r:off + rpad].any()


def test_raw_delta_and_Y_within_tolerance(small):
    from tests.gpu_pipeline import rel_err
    small.shrink()
    ref = small.ref()
    assert rel_err(small.delta(), ref["delta"]) <= DELTA_TOL
    assert rel_err(small.Y(), ref["Y"]) <= Y_TOL
    ad = wk.row_adapter(small.wl.seg_offsets, small.wl.seg_adapter, small.wl.M,
                        len(small.wl.adapters))
    # tokens without an adapter get exactly no delta
    if (ad < 0).any():
        assert not small.delta()[ad < 0].any()


def test_raw_without_adapters_is_plain_w8a8(small):
    # every segment without an adapter: T = 0 and Y equals the plain W8A8 layer
    import torch
    none = torch.full_like(small.g.seg_adapter, -1)
    small.shrink(seg_adapter=none)
    assert not small.delta().any()
    y_raw = small.Y()
    small.sq.sq_linear_lora(small.g.Xq, small.g.x_scale, small.g.Wq, small.g.w_scale, None, None,
                            None, small.g.Y)
    assert np.array_equal(y_raw, small.g.Y.float().cpu().numpy())


@pytest.mark.parametrize("name", ["llama3_8b_qkv_m2048_k4096_n6144",
                                  "llama3_8b_gateup_m8192_k4096_n28672"])
def test_raw_full_size_sampled(name):
    from tests.gpu_pipeline import rel_err
    run = RawRun(name)
    run.shrink()
    rng = np.random.default_rng(17)
    M = run.wl.M
    rows = np.array(sorted({0, M - 1, 255, 256} | set(rng.choice(M, 24, replace=False).tolist())),
                    np.int64)
    ref = run.ref(rows)
    assert rel_err(run.Y()[rows], ref["Y"]) <= Y_TOL
    assert rel_err(run.delta()[rows], ref["delta"]) <= DELTA_TOL
