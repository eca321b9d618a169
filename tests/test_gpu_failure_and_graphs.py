"""Failure detection and CUDA-graph replay.

Every spin-wait in the kernels is bounded.  With a bound of 1 ns a wait
gives up after one probe: the kernels must stop, report SQ_ERR_DEVICE_TIMEOUT
through sq_get_device_error, and leave the context usable (the next calls
with the normal bound give correct results).  The shapes have more K stages
than the pipelines' rings hold, so the producer's probe for a free stage
comes before any consumer can have freed one.  Nothing here faults or hangs
the GPU.

The hot path only enqueues work (no allocation, no synchronization), so a
step can be captured in a CUDA graph and replayed; replays must reproduce the
eager result bit for bit.
"""

import numpy as np
import pytest

import oracle
from w8a8_smoothquant_int8_b200 import workloads as wk

pytestmark = pytest.mark.gpu

TIMEOUT = 5  # SQ_ERR_DEVICE_TIMEOUT


def test_wait_on_a_barrier_nothing_sets_times_out():
    import time
    import torch
    import w8a8_smoothquant_int8_b200 as sq
    sq.sq_get_device_error(clear=True)
    t0 = time.perf_counter()
    sq.sq_selftest_wait_timeout(2_000_000)  # 2 ms bound
    torch.cuda.synchronize()
    assert time.perf_counter() - t0 < 5.0
    assert sq.sq_get_device_error(clear=True) == TIMEOUT
    assert sq.sq_get_device_error(clear=True) == 0
    x = torch.ones(4, device="cuda")
    assert float((x * 2).sum()) == 8.0  # the context is fine


@pytest.mark.parametrize("name", ["parity_ragged", "parity_segments", "parity_segments_large",
                                  "llama3_8b_oproj_decode_m64_k4096_n4096"])
def test_wait_bound_runs_out_cleanly(name):
    import torch
    import w8a8_smoothquant_int8_b200 as sq
    from tests.gpu_pipeline import GpuRun, rel_err
    wl = wk.make_workload(name)
    P = oracle.Prepared(wl)
    g = GpuRun(wl, s_host=P.s)
    g.quant()
    torch.cuda.synchronize()
    sq.sq_get_device_error(clear=True)
    try:
        sq.sq_set_wait_timeout_ns(1)
        acc = torch.empty((wl.M, wl.N), dtype=torch.int32, device="cuda")
        sq.sq_gemm_i32(g.Xq, g.Wq, acc)
        g.linear()
        torch.cuda.synchronize()
        assert sq.sq_get_device_error(clear=True) == TIMEOUT
    finally:
        sq.sq_set_wait_timeout_ns(2_000_000_000)
    # the context still works
    g.linear()
    torch.cuda.synchronize()
    assert sq.sq_get_device_error(clear=True) == 0
    assert rel_err(g.Y_f32(), P.rows(want=("Y",))["Y"]) <= 1e-2


@pytest.mark.parametrize("name", ["parity_ragged", "parity_decode"])
def test_graph_replay_matches_eager(name):
    import torch
    from tests.gpu_pipeline import GpuRun
    wl = wk.make_workload(name)
    g = GpuRun(wl)
    g.step()
    torch.cuda.synchronize()
    eager = g.Y.clone()
    g.Y.zero_()
    graph = torch.cuda.CUDAGraph()
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        g.step()  # warm the stream before capture
        torch.cuda.synchronize()
        with torch.cuda.graph(graph, stream=s):
            g.step()
    torch.cuda.synchronize()
    for _ in range(3):
        g.Y.zero_()
        graph.replay()
        torch.cuda.synchronize()
        assert torch.equal(g.Y.view(torch.int16), eager.view(torch.int16))
