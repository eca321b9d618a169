"""sq_linear_lora_noalloc: the linear layer for callers that cannot allocate
device memory (an engine that plans all device memory ahead and hands its
plugins no allocator, or code that must not call cudaMalloc at that point).
Its scratch is the library's static device array instead of a caller
workspace; its output must match sq_linear_lora's, call after call.

Collected last (file name) so that a run stopping at the first failure has
run every other test first; it also passes alone in a fresh process.
"""

import numpy as np
import pytest

import oracle
from w8a8_smoothquant_int8_b200 import workloads as wk

pytestmark = pytest.mark.gpu

Y_TOL = 1e-2


@pytest.mark.parametrize("name", ["parity_ragged", "parity_decode"])
def test_noalloc_matches_workspace_entry_point_twice(name):
    import torch
    import w8a8_smoothquant_int8_b200 as sq
    from tests.gpu_pipeline import GpuRun, rel_err
    wl = wk.make_workload(name)
    P = oracle.Prepared(wl)
    g = GpuRun(wl, s_host=P.s)
    g.quant()
    g.linear()  # the existing entry point, caller workspace
    ref = g.Y_f32()
    assert rel_err(ref, P.rows(want=("Y",))["Y"]) <= Y_TOL
    for _ in range(2):  # two calls in a row share the static scratch
        Y = torch.full_like(g.Y, float("nan"))
        sq.sq_linear_lora_noalloc(g.Xq, g.x_scale, g.Wq, g.w_scale, g.lora, g.seg_offsets,
                                  g.seg_adapter, Y)
        torch.cuda.synchronize()
        got = Y.float().cpu().numpy()
        assert np.isfinite(got).all()
        assert rel_err(got, ref.astype(np.float64)) <= Y_TOL
    assert sq.sq_get_device_error(clear=True) == 0


def test_noalloc_rejects_sizes_beyond_its_scratch():
    import torch
    import w8a8_smoothquant_int8_b200 as sq
    M, R = 8192, 1024  # T planes alone need 32 MiB > 16 MiB
    assert sq.sq_linear_lora_workspace_size(M, R) > 16 << 20
    d = torch.empty(16, dtype=torch.int8, device="cuda")
    st = sq._lib().sq_linear_lora_noalloc(d.data_ptr(), d.data_ptr(), d.data_ptr(), d.data_ptr(),
                                          M, 256, 256, d.data_ptr(), d.data_ptr(), d.data_ptr(),
                                          d.data_ptr(), 4, R, d.data_ptr(), d.data_ptr(), 1,
                                          d.data_ptr(), None)
    assert st == 6  # SQ_ERR_WORKSPACE
