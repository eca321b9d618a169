"""sq_linear_lora_noalloc: the linear layer for callers that cannot allocate
device memory (an engine that plans all device memory ahead and hands its
plugins no allocator, or code that must not call cudaMalloc at that point).
Its scratch is the library's static device array instead of a caller
workspace; it runs the same kernels, so its output must equal
sq_linear_lora's bit for bit, call after call.  Between the two checked
calls the array is filled by calls with other data (another workload, the
same tokens with other adapters or none), so a kernel that read scratch left
by an earlier call would show.

Collected last (file name) so that a run stopping at the first failure has
run every other test first; it also passes alone in a fresh process.
"""

import numpy as np
import pytest

import oracle
from w8a8_smoothquant_int8_b200 import workloads as wk

pytestmark = pytest.mark.gpu

Y_TOL = 1e-2


def _run(name):
    from tests.gpu_pipeline import GpuRun
    wl = wk.make_workload(name)
    P = oracle.Prepared(wl)
    g = GpuRun(wl, s_host=P.s)
    g.quant()
    return wl, P, g


def _with_workspace(g, seg_adapter):
    g.Y.fill_(float("nan"))
    import w8a8_smoothquant_int8_b200 as sq
    sq.sq_linear_lora(g.Xq, g.x_scale, g.Wq, g.w_scale, g.lora, g.seg_offsets, seg_adapter, g.Y,
                      g.workspace)
    return g.Y.clone()


def _noalloc(g, seg_adapter):
    import torch
    import w8a8_smoothquant_int8_b200 as sq
    Y = torch.full_like(g.Y, float("nan"))
    sq.sq_linear_lora_noalloc(g.Xq, g.x_scale, g.Wq, g.w_scale, g.lora, g.seg_offsets,
                              seg_adapter, Y)
    return Y


@pytest.mark.parametrize("name,other", [("parity_ragged", "parity_decode"),
                                        ("parity_decode", "parity_ragged")])
def test_noalloc_matches_workspace_entry_point_twice(name, other):
    import torch
    import w8a8_smoothquant_int8_b200 as sq
    from tests.gpu_pipeline import rel_err
    wl, P, g = _run(name)
    _, _, h = _run(other)
    ref = _with_workspace(g, g.seg_adapter)  # the existing entry point, caller workspace
    torch.cuda.synchronize()
    assert rel_err(ref.float().cpu().numpy(), P.rows(want=("Y",))["Y"]) <= Y_TOL
    # the same tokens with their adapters moved around, and with none
    moved = torch.roll(g.seg_adapter, 1)
    none = torch.full_like(g.seg_adapter, -1)
    ref_moved = _with_workspace(g, moved)
    ref_none = _with_workspace(g, none)
    ref_other = _with_workspace(h, h.seg_adapter)
    first = _noalloc(g, g.seg_adapter)
    assert torch.equal(first, ref)
    # the static scratch now holds other data each time
    assert torch.equal(_noalloc(h, h.seg_adapter), ref_other)
    assert torch.equal(_noalloc(g, moved), ref_moved)
    assert torch.equal(_noalloc(g, none), ref_none)
    second = _noalloc(g, g.seg_adapter)
    assert torch.equal(second, ref)
    torch.cuda.synchronize()
    assert sq.sq_get_device_error(clear=True) == 0


def test_noalloc_pack_without_adapters_is_plain_w8a8():
    # R > 0 with no adapters (or no segments) is plain W8A8, as for
    # sq_linear_lora: no scratch is needed and the call succeeds
    import torch
    import w8a8_smoothquant_int8_b200 as sq
    wl, P, g = _run("parity_ragged")
    empty = sq.LoraPack(g.lora.A_pack, g.lora.B_pack, g.lora.offset, g.lora.rank, g.lora.R, 0)
    Y_ws = torch.full_like(g.Y, float("nan"))
    sq.sq_linear_lora(g.Xq, g.x_scale, g.Wq, g.w_scale, None, None, None, Y_ws)
    Y = torch.full_like(g.Y, float("nan"))
    sq.sq_linear_lora_noalloc(g.Xq, g.x_scale, g.Wq, g.w_scale, empty, g.seg_offsets,
                              g.seg_adapter, Y)
    torch.cuda.synchronize()
    assert torch.equal(Y, Y_ws)
    assert sq.sq_get_device_error(clear=True) == 0


def test_noalloc_rejects_sizes_beyond_its_scratch():
    import torch
    import w8a8_smoothquant_int8_b200 as sq
    M, R = 8192, 1024  # T planes alone need 32 MiB > 16 MiB
    assert sq.sq_linear_lora_workspace_size(M, R) > 16 << 20
    d = torch.empty(16, dtype=torch.int8, device="cuda")
    p = d.data_ptr()

    def call(K):
        return sq._lib().sq_linear_lora_noalloc(p, p, p, p, M, 256, K, p, p, p, p, 4, R, p, p, 1,
                                                p, None)

    assert call(256) == 6   # SQ_ERR_WORKSPACE
    assert call(250) == 2   # a shape error comes first: SQ_ERR_UNSUPPORTED_SHAPE
