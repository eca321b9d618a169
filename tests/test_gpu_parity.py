"""Parity of the CUDA path with the CPU oracle, element by element.

Bars: Xq, x_scale, Wq, w_scale, the packed LoRA operands and the int32
accumulators bit-exact; the smoothing scale within 1 ulp (fp64 pow is not
correctly rounded on either side); Y (bf16) within max|Y-Y_ref|/max|Y_ref|
<= 1e-2 and the LoRA delta alone within 5e-3 of the same measure.
"""

import numpy as np
import pytest

import oracle
from w8a8_smoothquant_int8_b200 import workloads as wk

pytestmark = pytest.mark.gpu

Y_TOL = 1e-2
DELTA_TOL = 5e-3

SMALL = ["tiny_m16_k256_n256", "parity_ragged", "parity_heavy_f32", "parity_decode",
         "parity_waves", "parity_segments", "parity_segments_large"]


def _run(name, **kw):
    from tests.gpu_pipeline import GpuRun
    wl = wk.make_workload(name, **kw)
    P = oracle.Prepared(wl)
    g = GpuRun(wl, s_host=P.s)
    g.quant()
    return wl, P, g


@pytest.fixture(scope="module", params=SMALL)
def small(request):
    return _run(request.param)


def test_smoothing_scale_within_one_ulp(small):
    from tests.gpu_pipeline import ulp_diff_f32
    wl, P, g = small
    assert np.array_equal(g.act_absmax.cpu().numpy(), P.act_absmax)
    assert np.array_equal(g.w_absmax.cpu().numpy(), P.w_absmax)
    assert ulp_diff_f32(g.s_gpu.cpu().numpy(), P.s) <= 1


def test_weight_quant_bit_exact(small):
    wl, P, g = small
    assert np.array_equal(g.w_scale.cpu().numpy().view(np.uint32), P.w_scale.view(np.uint32))
    assert np.array_equal(g.Wq.cpu().numpy(), P.Wq)


def test_quant_act_bit_exact(small):
    wl, P, g = small
    assert np.array_equal(g.x_scale.cpu().numpy().view(np.uint32), P.x_scale.view(np.uint32))
    assert np.array_equal(g.Xq.cpu().numpy(), P.Xq)


def test_lora_pack_bit_exact(small):
    from tests.gpu_pipeline import bf16_bits
    wl, P, g = small
    A_pack = bf16_bits(g.lora.A_pack)
    B_pack = bf16_bits(g.lora.B_pack)
    offs, R = g.lora.layout([a.r for a in wl.adapters])
    assert g.lora.R == R
    # the table written by sq_pack_lora
    assert g.lora.offset.cpu().tolist() == offs
    assert g.lora.rank.cpu().tolist() == [a.r for a in wl.adapters]
    for a, off in enumerate(offs):
        r = wl.adapters[a].r
        rpad = (r + 15) // 16 * 16
        assert np.array_equal(A_pack[off:off + r], P.A_s[a])
        assert not A_pack[off + r:off + rpad].any()
        assert np.array_equal(B_pack[:, off:off + r], P.B_s[a])
        assert not B_pack[:, off + r:off + rpad].any()


def test_gemm_i32_bit_exact(small):
    wl, P, g = small
    acc = g.gemm_i32()
    assert np.array_equal(acc.astype(np.int64), oracle.gemm_rows(P.Xq, P.Wq))


def test_linear_lora_within_tolerance(small):
    from tests.gpu_pipeline import rel_err
    wl, P, g = small
    g.linear()
    ref = P.rows(want=("Y",))["Y"]
    assert rel_err(g.Y_f32(), ref) <= Y_TOL


def test_lora_delta_within_tolerance(small):
    from tests.gpu_pipeline import rel_err
    wl, P, g = small
    ref = P.rows(want=("delta",))["delta"]
    d = g.delta()
    ad = wk.row_adapter(wl.seg_offsets, wl.seg_adapter, wl.M, len(wl.adapters))
    assert not d[ad < 0].any()
    assert rel_err(d, ref) <= DELTA_TOL


# ----------------------------------------------------------------------------
# Full-size workloads, sampled outputs, in the launch configuration the
# benchmark times (same entry points, same shapes).
# ----------------------------------------------------------------------------
FULL = ["llama3_8b_qkv_m2048_k4096_n6144", "llama3_8b_gateup_m8192_k4096_n28672",
        "llama3_8b_down_m16384_k14336_n4096", "llama3_8b_oproj_decode_m64_k4096_n4096"]


def _sample_rows(M, rng, n=24):
    # tile edges, random rows, and one random row of every 256-row tile
    rows = {0, M - 1, min(127, M - 1), min(128, M - 1)}
    rows |= set(rng.choice(M, size=min(M, n), replace=False).tolist())
    for t0 in range(0, M, 256):
        rows.add(int(rng.integers(t0, min(M, t0 + 256))))
    return np.array(sorted(rows), np.int64)


@pytest.mark.parametrize("name", FULL)
def test_full_size_sampled(name):
    from tests.gpu_pipeline import rel_err
    wl, P, g = _run(name)
    rng = np.random.default_rng(7)
    # quantization outputs are cheap to check everywhere
    assert np.array_equal(g.x_scale.cpu().numpy().view(np.uint32), P.x_scale.view(np.uint32))
    assert np.array_equal(g.Xq.cpu().numpy(), P.Xq)
    assert np.array_equal(g.Wq.cpu().numpy(), P.Wq)
    assert np.array_equal(g.w_scale.cpu().numpy().view(np.uint32), P.w_scale.view(np.uint32))
    rows = _sample_rows(wl.M, rng)
    out = P.rows(rows)
    acc = g.gemm_i32()
    assert np.array_equal(acc[rows].astype(np.int64), out["acc"])
    # random (token, channel) pairs over the whole output
    ri = rng.integers(0, wl.M, 4096)
    ci = rng.integers(0, wl.N, 4096)
    assert np.array_equal(acc[ri, ci].astype(np.int64), oracle.gemm_pairs(P.Xq, P.Wq, ri, ci))
    g.linear()
    assert rel_err(g.Y_f32()[rows], out["Y"]) <= Y_TOL
    assert rel_err(g.delta()[rows], out["delta"]) <= DELTA_TOL


# The tensor-memory form of the shrink splits K over a cluster of CTAs when
# there are few 128-token blocks, as wide as all clusters stay resident at
# once: 4096 tokens at K=4096 (clusters of four), 6144 tokens (clusters of
# three would not all be resident: two) and 4096 tokens at K=14336.
@pytest.mark.parametrize("name,M", [("llama3_8b_gateup_m8192_k4096_n28672", 4096),
                                    ("llama3_8b_gateup_m8192_k4096_n28672", 6144),
                                    ("llama3_8b_down_m16384_k14336_n4096", 4096)])
def test_shrink_cluster_splits_sampled(name, M):
    from tests.gpu_pipeline import rel_err
    wl, P, g = _run(name, M=M)
    rows = _sample_rows(wl.M, np.random.default_rng(11))
    out = P.rows(rows, want=("Y", "delta"))
    g.linear()
    assert rel_err(g.Y_f32()[rows], out["Y"]) <= Y_TOL
    assert rel_err(g.delta()[rows], out["delta"]) <= DELTA_TOL
