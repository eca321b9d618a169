#!/usr/bin/env python
"""Benchmark of the SmoothQuant W8A8 + per-request LoRA linear on B200.

One step = one pass of the whole hot path over one batch: sq_quant_act
(smoothing + per-token INT8) followed by sq_linear_lora (LoRA shrink, then
the fused INT8 GEMM + dequant + LoRA delta).

The default run measures four workloads, one after another, in one process:
the headline is the compute-bound down projection (M=16384 tokens, K=14336,
N=4096, four rank-32 adapters over 64 request segments), the largest
single-GPU workload; the fused QKV (M=2048, K=4096, N=6144, one rank-16
adapter), the multi-tenant gate/up (M=8192, K=4096, N=28672, eight adapters
over 32 segments) and the memory-bound decode step (M=64, K=4096, N=4096, 64
rank-16 adapters, one per token) are reported beside it under "workloads",
each with its own roofline, CPU baseline and end-to-end figure.
`--workload NAME` measures one workload alone.

Timing: W untimed warm-up steps, then K timed steps.  Before every step a
256 MiB buffer is written and a second 256 MiB buffer is read (untimed), so
that L2 (126 MB) holds none of the step's inputs and no dirty lines whose
write-back would be charged to the step; each step is bracketed by CUDA
events on the stream the kernels run on, and on every eighth timed step the
layer call's kernels also by their own event pair (recorded by the library;
an event between the shrink and the GEMM keeps the GEMM from starting during
the shrink's tail, so it is not recorded on every step).  Multi-GPU runs are
independent replicas (the layer has no exchange step): each rank runs the
same workload, times are maxed over ranks and the throughput counts all
ranks' work.

The decode workload is also run 1000 times back to back (a CUDA graph of
steps, replayed), cycling through enough copies of Wq and the adapters that
L2 cannot hold them between uses; its per-step latency is reported as
"repeated".

End to end (the "e2e" key): the same step through pinned host buffers, X
copied in and Y copied out every step, with consecutive steps pipelined over
three streams (copy in, kernels, copy out) as a serving loop runs them; the
serial form (one step at a time) is reported beside it.

--impl reference times the CPU oracle (fp64/int64 C, OpenMP) on the host
cores for the headline workload and metric, one bounded sample of tokens per
step.
"""

from __future__ import annotations

import argparse
import datetime
import json
import math
import os
import statistics
import subprocess
import sys
import tempfile
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

from w8a8_smoothquant_int8_b200 import workloads as wk  # noqa: E402

GEMM_EVENT_EVERY = 8  # timed steps per step that also times the layer's kernels alone
# nominal figures, reported beside the measured denominators for context:
# dense int8 tensor-core ops per SM per clock (4.5 POPS over 148 SMs near
# 1.9 GHz) and the HBM3e bandwidth of the part
NOMINAL_INT8_OPS_PER_SM_CLK = 16384
NOMINAL_HBM_GBS = 8000.0

METRIC = "W8A8+LoRA linear INT8 TOPS & tokens/s; % of INT8 tensor peak / HBM roofline"
HEADLINE = "llama3_8b_down_m16384_k14336_n4096"
BESIDE = ["llama3_8b_gateup_m8192_k4096_n28672", "llama3_8b_qkv_m2048_k4096_n6144",
          "llama3_8b_oproj_decode_m64_k4096_n4096"]
FLUSH_BYTES = 256 << 20
DECODE_REPEAT = 1000
# seconds of oracle work for the CPU baseline of the headline workload and of
# each workload beside it (a bounded sample of its tokens)
CPU_SECONDS_HEADLINE = 12.0
CPU_SECONDS_BESIDE = 2.0


def parse():
    p = argparse.ArgumentParser()
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=50)
    p.add_argument("--warmup", type=int, default=10)
    p.add_argument("--impl", choices=["ours", "reference"], default="ours")
    p.add_argument("--workload", default="all", choices=["all"] + sorted(wk.SPECS),
                   help="'all' (default): the headline workload and the three beside it")
    p.add_argument("--e2e-steps", type=int, default=10)
    p.add_argument("--no-cpu-baseline", action="store_true")
    p.add_argument("--act-quant", choices=["dynamic", "static"], default="dynamic",
                   help="per-token scales (default) or one calibrated per-tensor scale "
                        "(sq_quant_act_static)")
    p.add_argument("--norm-fold", action="store_true",
                   help="the activations are a normalization's input: RMS norm with 1/s folded "
                        "into its weight, fused with the per-token quantization "
                        "(sq_rmsnorm_quant_act)")
    p.add_argument("--lora-input", choices=["dequant", "raw"], default="dequant",
                   help="what the LoRA path reads: the dequantized codes (default) or the "
                        "raw bf16 activations (sq_lora_shrink_raw + sq_linear_lora_from_t)")
    return p.parse_args()


# DRAM bytes (read + write) of one launch of the dominant kernel, per
# workload, from an ncu capture of that kernel source (sha256 of the file that
# holds it); any other source or workload reports null.
KERNEL_TRAFFIC = {
    "llama3_8b_qkv_m2048_k4096_n6144": {
        "file": "gemm_sm100.cu",
        "source_sha256": "bddc86184aecdea6f0229daa3e334b286019ae9edbacfc434408135e3b1c6db2",
        "bytes": 34082816 + 1157888,
    },
    "llama3_8b_gateup_m8192_k4096_n28672": {
        "file": "gemm_sm100.cu",
        "source_sha256": "bddc86184aecdea6f0229daa3e334b286019ae9edbacfc434408135e3b1c6db2",
        "bytes": 395806464 + 447846656,
    },
    "llama3_8b_down_m16384_k14336_n4096": {
        "file": "gemm_sm100.cu",
        "source_sha256": "bddc86184aecdea6f0229daa3e334b286019ae9edbacfc434408135e3b1c6db2",
        "bytes": 1241112320 + 124009984,
    },
    # the layer call: decode_shrink_kernel + decode_gemm_kernel
    "llama3_8b_oproj_decode_m64_k4096_n4096": {
        "file": "decode.cu",
        "source_sha256": "303cf96cc6ba475c9509c595f2b8466d4e030b25a52bd6ec6694955e74ca76d7",
        "bytes": 8672256 + 25544192,
    },
}


def kernel_traffic(workload: str):
    import hashlib
    ent = KERNEL_TRAFFIC.get(workload)
    if ent is None:
        return None
    src = os.path.join(ROOT, "w8a8_smoothquant_int8_b200", "csrc", ent["file"])
    try:
        with open(src, "rb") as f:
            sha = hashlib.sha256(f.read()).hexdigest()
    except OSError:
        return None
    return ent["bytes"] if sha == ent["source_sha256"] else None


def measured_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            d = json.load(f)
        return d, "measured"
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}, "fallback"


DECODE_MAX_M = 64  # the library's streaming (decode) form handles M <= 64


def decode_layer_bytes(wl) -> int:
    """Algorithmic HBM bytes of one sq_linear_lora call in the decode form:
    Wq and w_scale, the codes and scales of the tokens, the A' and B' rows of
    every adapter some token uses, and Y."""
    ad = wk.row_adapter(wl.seg_offsets, wl.seg_adapter, wl.M, len(wl.adapters))
    used = sorted(set(int(a) for a in ad if a >= 0))
    lora = sum(2 * wl.adapters[a].r * (wl.K + wl.N) for a in used)
    return int(wl.N * wl.K + 4 * wl.N + wl.M * wl.K + 4 * wl.M + lora + 2 * wl.M * wl.N)


def quant_bytes(wl) -> int:
    """Algorithmic HBM bytes of sq_quant_act: X read, codes and scales written."""
    xb = 2 if wl.x_is_bf16 else 4
    return int(wl.M * wl.K * (xb + 1) + 4 * wl.M + 4 * wl.K)


def lora_flops(wl) -> int:
    ad = wk.row_adapter(wl.seg_offsets, wl.seg_adapter, wl.M, len(wl.adapters))
    r = np.array([wl.adapters[a].r if a >= 0 else 0 for a in ad], np.int64)
    return int(2 * r.sum() * (wl.K + wl.N))


# ---------------------------------------------------------------------------
# ranks: every rank runs a replica; times are maxed over ranks
# ---------------------------------------------------------------------------
def reduce_max(values, device=None):
    """Element-wise maximum of `values` over all ranks (identity with one process)."""
    import torch
    import torch.distributed as dist
    t = torch.tensor(list(values), dtype=torch.float64, device=device)
    if dist.is_available() and dist.is_initialized() and dist.get_world_size() > 1:
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return [float(x) for x in t.cpu()]


def job_tops(ops_per_step: int, steps: int, world: int, total_ms: float) -> float:
    """Whole-job throughput: the work of every rank over the slowest rank's time."""
    return ops_per_step * steps * world / (total_ms * 1e-3) / 1e12


# ---------------------------------------------------------------------------
# clocks during the timed region
# ---------------------------------------------------------------------------
class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.path = tempfile.mktemp(prefix="sq_clocks_", suffix=".csv")
        self.proc = None
        self.gpu = gpu_index

    def start(self):
        try:
            self.f = open(self.path, "w")
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-i", str(self.gpu), "-lms", "100"], stdout=self.f, stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None
        time.sleep(0.3)

    def stop(self):
        if self.proc is None:
            return None
        time.sleep(0.25)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        self.f.close()
        rows = []
        with open(self.path) as f:
            for line in f:
                parts = [x.strip() for x in line.split(",")]
                if len(parts) < 9:
                    continue
                try:
                    rows.append(dict(sm=float(parts[1]), max=float(parts[2]), power=float(parts[3]),
                                     hw=parts[5], hwt=parts[6], swt=parts[7], pcap=parts[8]))
                except ValueError:
                    continue
        os.unlink(self.path)
        if not rows:
            return None
        loaded = [r for r in rows if r["power"] > 250.0] or rows
        reasons = set()
        for r in loaded:
            for key, name in (("hw", "hw_slowdown"), ("hwt", "hw_thermal_slowdown"),
                              ("swt", "sw_thermal_slowdown"), ("pcap", "sw_power_cap")):
                if r[key].lower().startswith("active"):
                    reasons.add(name)
        return {"sm_mhz": statistics.median(r["sm"] for r in loaded),
                "sm_max_mhz": max(r["max"] for r in rows),
                "reasons": sorted(reasons), "samples": len(loaded)}


# ---------------------------------------------------------------------------
# CPU oracle (reported baseline; test infrastructure, timed as it stands)
# ---------------------------------------------------------------------------
def oracle_step(P, wl, rows, raw=False):
    import oracle
    Xq, xs = oracle.quant_act(wl.X[rows], P.s)
    ad = wk.row_adapter(wl.seg_offsets, wl.seg_adapter, wl.M, len(wl.adapters))
    # the sampled tokens keep their own adapters: one segment per token
    so = np.arange(len(rows) + 1, dtype=np.int32)
    sa = ad[rows].astype(np.int32)
    if raw:
        oracle.linear_lora_raw_rows(wl.X[rows], Xq, xs, P.Wq, P.w_scale, [a.A for a in wl.adapters],
                                    P.B_s, so, sa, want=("Y",))
    else:
        oracle.linear_lora_rows(Xq, xs, P.Wq, P.w_scale, P.A_s, P.B_s, so, sa, want=("Y",))


def cpu_baseline(wl, seconds: float, raw=False):
    """The oracle over a bounded sample of the workload's tokens: a 16-token
    probe sizes the sample to about `seconds` of work (the whole workload if
    it is shorter), then the sample is timed in one pass."""
    import oracle
    P = oracle.Prepared(wl)
    probe = np.arange(min(16, wl.M))
    t0 = time.perf_counter()
    oracle_step(P, wl, probe, raw)
    t_probe = max(time.perf_counter() - t0, 1e-6)
    n = int(min(wl.M, max(len(probe), len(probe) * seconds / t_probe)))
    rows = np.sort(np.random.default_rng(0).choice(wl.M, size=n, replace=False)) \
        if n < wl.M else np.arange(wl.M)
    t0 = time.perf_counter()
    oracle_step(P, wl, rows, raw)
    dt = time.perf_counter() - t0
    ops = 2 * len(rows) * wl.N * wl.K
    what = "all" if n == wl.M else f"{n} random"
    return {"value": ops / dt / 1e12, "unit": "TOPS", "cores": oracle.num_threads(),
            "kind": "oracle",
            "sample": f"{what} of {wl.M} tokens, whole hot path (quantize, int64 GEMM, fp64 "
                      f"dequant + LoRA on the {'raw activations' if raw else 'dequantized codes'}), "
                      f"one pass, {dt:.2f} s",
            "tokens_per_s": len(rows) / dt}


def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    import oracle
    name = HEADLINE if args.workload == "all" else args.workload
    wl = wk.make_workload(name)
    P = oracle.Prepared(wl)
    sample = min(wl.M, 64)
    rng = np.random.default_rng(0)
    times = []
    for i in range(args.warmup + args.steps):
        rows = np.sort(rng.choice(wl.M, size=sample, replace=False))
        t0 = time.perf_counter()
        oracle_step(P, wl, rows, args.lora_input == "raw")
        dt = time.perf_counter() - t0
        if i >= args.warmup:
            times.append(dt)
    t = sum(times)
    ops = 2 * sample * wl.N * wl.K * len(times)
    value = ops / t / 1e12
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "TOPS", "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * t / len(times),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "int64",
        "data": "synthetic",
        "config": {"workload": wl.spec.name, "M": wl.M, "K": wl.K, "N": wl.N,
                   "sample_tokens_per_step": sample},
        "tokens_per_s": sample * len(times) / t,
        "cpu_baseline": {"value": value, "unit": "TOPS", "cores": oracle.num_threads(),
                         "kind": "oracle",
                         "sample": f"{sample} random tokens of {wl.M} per step, whole hot path"},
        "e2e": {"value": value, "unit": "TOPS", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


# ---------------------------------------------------------------------------
# GPU path
# ---------------------------------------------------------------------------
def measure(name, args, dev, world, local_rank, cpu_seconds):
    """Time one workload; returns its entry (value, roofline, e2e, ...)."""
    import torch
    import torch.distributed as dist

    import w8a8_smoothquant_int8_b200 as sq

    wl = wk.make_workload(name)
    raw = args.lora_input == "raw"
    cpu = None
    if cpu_seconds > 0:
        cpu = cpu_baseline(wl, cpu_seconds, raw=raw)

    M, K, N = wl.M, wl.K, wl.N

    def h2d(a):
        t = torch.from_numpy(np.ascontiguousarray(a))
        if a.dtype == np.uint16:
            t = t.view(torch.bfloat16)
        return t.to(dev)

    # offline preparation (not timed): calibration, smoothing, weight quant, LoRA pack
    X = h2d(wl.X)
    W = h2d(wl.W)
    act_absmax = torch.zeros(K, dtype=torch.float32, device=dev)
    sq.sq_act_absmax_update(h2d(wl.X_cal), act_absmax)
    w_absmax = torch.empty(K, dtype=torch.float32, device=dev)
    sq.sq_weight_absmax(W, w_absmax)
    s = torch.empty(K, dtype=torch.float32, device=dev)
    sq.sq_compute_smoothing(act_absmax, w_absmax, wl.alpha, s)
    Wq = torch.empty((N, K), dtype=torch.int8, device=dev)
    w_scale = torch.empty(N, dtype=torch.float32, device=dev)
    sq.sq_quantize_weight(W, s, Wq, w_scale)
    del W
    if raw and not wl.x_is_bf16:
        raise SystemExit("--lora-input raw needs bf16 activations")
    lora = sq.LoraPack.build([h2d(a.A) for a in wl.adapters], [h2d(a.B) for a in wl.adapters],
                             [a.lora_alpha for a in wl.adapters], None if raw else s)
    seg_offsets = h2d(wl.seg_offsets)
    seg_adapter = h2d(wl.seg_adapter)
    Xq = torch.empty((M, K), dtype=torch.int8, device=dev)
    x_scale = torch.empty(M, dtype=torch.float32, device=dev)
    ws_bytes = (sq.sq_lora_t_workspace_size(M, lora.R) if raw
                else sq.sq_linear_lora_workspace_size(M, lora.R))
    ws = torch.empty(max(ws_bytes, 256), dtype=torch.uint8, device=dev)
    Y = torch.empty((M, N), dtype=torch.bfloat16, device=dev)
    flush = torch.empty(FLUSH_BYTES // 4, dtype=torch.int32, device=dev)
    flush_read = torch.ones(FLUSH_BYTES // 4, dtype=torch.int32, device=dev)

    def flush_l2(v):
        # write one buffer larger than L2, then read another one: L2 ends up
        # holding clean lines of neither the inputs nor the outputs
        flush.fill_(v)
        flush_read.max()

    static = args.act_quant == "static"
    norm = args.norm_fold
    if norm:
        if static or not wl.x_is_bf16:
            raise SystemExit("--norm-fold takes bf16 activations and per-token scales")
        gamma_s = torch.empty(K, dtype=torch.float32, device=dev)
        sq.sq_fold_norm_weight(torch.from_numpy(wk.norm_gamma(K, wl.seed)).to(dev), s, gamma_s)
    if static:
        static_scale = torch.empty(1, dtype=torch.float32, device=dev)
        sq.sq_static_act_scale(act_absmax, s, static_scale)
        clip_count = torch.zeros(1, dtype=torch.int64, device=dev)

    decode = M <= DECODE_MAX_M and not raw

    def step(Xb=X, Yb=Y, Wqb=Wq, wsb=w_scale, lorab=lora):
        if norm:
            sq.sq_rmsnorm_quant_act(Xb, gamma_s, 1e-6, Xq, x_scale)
        elif static:
            sq.sq_quant_act_static(Xb, s, static_scale, Xq, x_scale, clip_count)
        else:
            sq.sq_quant_act(Xb, s, Xq, x_scale)
        if raw:
            sq.sq_lora_shrink_raw(Xb, lorab, seg_offsets, seg_adapter, ws)
            sq.sq_linear_lora_from_t(Xq, x_scale, Wqb, wsb, lorab, Yb, ws)
        else:
            sq.sq_linear_lora(Xq, x_scale, Wqb, wsb, lorab, seg_offsets, seg_adapter, Yb, ws)

    launches_per_step = 3  # quantize, LoRA shrink, fused GEMM (or the decode pair)

    sampler = ClockSampler(local_rank)
    sampler.start()
    for _ in range(args.warmup):
        flush_l2(1)
        step()
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    n = args.steps
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(n)]
    for e in ev:  # create the event handles before the library records them
        for x in e:
            x.record()
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    # the layer call's own event pair sits between the quantizer and the
    # shrink, and between the shrink and the GEMM; recorded on every
    # GEMM_EVENT_EVERY-th timed step only (all K steps count towards the step
    # time)
    gemm_steps = [i for i in range(n) if i % GEMM_EVENT_EVERY == GEMM_EVENT_EVERY // 2]
    gemm_steps = gemm_steps or [n // 2]
    for i in range(n):
        flush_l2(i & 0x7f)
        ev[i][0].record()
        if i in gemm_steps:
            sq.sq_set_gemm_events(ev[i][2], ev[i][3])
        step()
        sq.sq_set_gemm_events(None, None)
        ev[i][1].record()
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    clocks = sampler.stop()
    step_ms = [e[0].elapsed_time(e[1]) for e in ev]
    gemm_ms = [ev[i][2].elapsed_time(ev[i][3]) for i in gemm_steps]
    t_step_total, t_gemm_total = reduce_max([sum(step_ms), sum(gemm_ms)], dev)
    err = sq.sq_get_device_error(clear=True)
    if err:
        raise SystemExit(f"device error {err}: {sq.sq_status_string(err)}")

    # decode: 1000 steps back to back in a CUDA graph, cycling through copies
    # of Wq, w_scale and the adapters so that none is still in L2 when it is
    # used again (copies x bytes >= 4 x L2)
    repeated = None
    if decode:
        l2 = torch.cuda.get_device_properties(dev).L2_cache_size
        copies = max(2, math.ceil(4 * l2 / decode_layer_bytes(wl)))
        reps = [(Wq, w_scale, lora)]
        for _ in range(copies - 1):
            lp = sq.LoraPack(lora.A_pack.clone(), lora.B_pack.clone(), lora.offset.clone(),
                             lora.rank.clone(), lora.R, lora.n_adapters)
            reps.append((Wq.clone(), w_scale.clone(), lp))
        g_stream = torch.cuda.Stream(dev)
        g_stream.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(g_stream):
            for r in reps:  # warm: the library's first call per device does its set-up
                step(Wqb=r[0], wsb=r[1], lorab=r[2])
        g_stream.synchronize()
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph, stream=g_stream):
            for r in reps:
                step(Wqb=r[0], wsb=r[1], lorab=r[2])
        replays = math.ceil(DECODE_REPEAT / copies)
        for _ in range(2):
            graph.replay()
        torch.cuda.synchronize()
        a = torch.cuda.Event(enable_timing=True)
        b = torch.cuda.Event(enable_timing=True)
        a.record()
        for _ in range(replays):
            graph.replay()
        b.record()
        torch.cuda.synchronize()
        t_rep = reduce_max([a.elapsed_time(b)], dev)[0]
        steps_rep = replays * copies
        us = 1e3 * t_rep / steps_rep
        step_bytes = decode_layer_bytes(wl) + quant_bytes(wl)
        repeated = {"steps": steps_rep, "us_per_step": us,
                    "tokens_per_s": M * steps_rep * world / (t_rep * 1e-3),
                    "step_bytes": step_bytes, "gbs": step_bytes / (us * 1e-6) / 1e9,
                    "form": f"CUDA graph of {copies} steps (one per copy of Wq, w_scale and the "
                            f"adapters, {copies} x {decode_layer_bytes(wl) / 1e6:.1f} MB), "
                            f"replayed {replays} times; inputs not flushed between steps"}
        del graph, reps
        err = sq.sq_get_device_error(clear=True)
        if err:
            raise SystemExit(f"device error {err}: {sq.sq_status_string(err)}")

    # end to end through the public API with host buffers: every step copies
    # its X in from pinned host memory and its Y out to pinned host memory.
    # Serial form: copy in, kernels, copy out on one stream, one step at a
    # time.  Pipelined form (the reported value), as a serving loop runs:
    # three streams, so that step i's copy in, step i-1's kernels and step
    # i-2's copy out overlap, with two device buffers for X and for Y.
    X_host = torch.from_numpy(np.ascontiguousarray(wl.X)).view(torch.bfloat16) \
        if wl.x_is_bf16 else torch.from_numpy(np.ascontiguousarray(wl.X))
    X_host = X_host.pin_memory()
    Y_host = torch.empty((M, N), dtype=torch.bfloat16).pin_memory()

    def e2e_serial(nsteps):
        ms = []
        for _ in range(nsteps):
            flush_l2(3)
            a = torch.cuda.Event(enable_timing=True)
            b = torch.cuda.Event(enable_timing=True)
            a.record()
            X.copy_(X_host, non_blocking=True)
            step()
            Y_host.copy_(Y, non_blocking=True)
            b.record()
            torch.cuda.synchronize()
            ms.append(a.elapsed_time(b))
        return sum(ms)

    X_dev = [X, torch.empty_like(X)]
    Y_dev = [Y, torch.empty_like(Y)]
    s_h2d, s_cmp, s_d2h = (torch.cuda.Stream(dev) for _ in range(3))

    def e2e_pipelined(nsteps):
        ev_h2d = [torch.cuda.Event() for _ in range(nsteps)]
        ev_cmp = [torch.cuda.Event() for _ in range(nsteps)]
        ev_d2h = [torch.cuda.Event() for _ in range(nsteps)]
        a = torch.cuda.Event(enable_timing=True)
        b = torch.cuda.Event(enable_timing=True)
        torch.cuda.synchronize()
        a.record(s_h2d)
        s_cmp.wait_event(a)
        s_d2h.wait_event(a)
        for i in range(nsteps):
            j = i % 2
            with torch.cuda.stream(s_h2d):
                if i >= 2:
                    s_h2d.wait_event(ev_cmp[i - 2])  # the kernels of step i-2 read X_dev[j]
                X_dev[j].copy_(X_host, non_blocking=True)
                ev_h2d[i].record(s_h2d)
            with torch.cuda.stream(s_cmp):
                s_cmp.wait_event(ev_h2d[i])
                if i >= 2:
                    s_cmp.wait_event(ev_d2h[i - 2])  # Y_dev[j] of step i-2 is copied out
                flush_l2(3)  # untimed elsewhere; here it overlaps the copies
                step(X_dev[j], Y_dev[j])
                ev_cmp[i].record(s_cmp)
            with torch.cuda.stream(s_d2h):
                s_d2h.wait_event(ev_cmp[i])
                Y_host.copy_(Y_dev[j], non_blocking=True)
                ev_d2h[i].record(s_d2h)
        b.record(s_d2h)  # after the last copy out, which follows every other step
        torch.cuda.synchronize()
        return a.elapsed_time(b)

    e2e = None
    n_e2e = args.e2e_steps
    ops_step = 2 * M * N * K
    if n_e2e > 0:
        e2e_serial(min(args.warmup, 3))
        t_serial = reduce_max([e2e_serial(n_e2e)], dev)[0]
        e2e_pipelined(max(min(args.warmup, 3), 2))
        t_e2e = reduce_max([e2e_pipelined(n_e2e)], dev)[0]
        e2e = {"value": job_tops(ops_step, n_e2e, world, t_e2e), "unit": "TOPS",
               "h2d_bytes_per_step": int(X_host.numel() * X_host.element_size()),
               "d2h_bytes_per_step": int(Y_host.numel() * Y_host.element_size()),
               "ms_per_step": t_e2e / n_e2e,
               "tokens_per_s": M * n_e2e * world / (t_e2e * 1e-3),
               "form": "pipelined: copy in, kernels and copy out of consecutive steps "
                       "on three streams (two device buffers for X and Y)",
               "serial": {"value": job_tops(ops_step, n_e2e, world, t_serial),
                          "ms_per_step": t_serial / n_e2e}}

    value = job_tops(ops_step, n, world, t_step_total)
    tok_s = M * n * world / (t_step_total * 1e-3)
    gemm_avg_s = t_gemm_total * 1e-3 / max(1, len(gemm_steps))
    gemm_tops = ops_step / gemm_avg_s / 1e12
    peaks, peak_kind = measured_peaks()
    int8_peak = 2.0 * float(peaks["bf16_tflops"])  # dense int8 = 2x dense bf16 (nominal ratio)
    if decode:
        # decode form: bound by streaming Wq and the adapters from HBM; the
        # timed region is the whole layer call (shrink + GEMM kernels)
        nbytes = decode_layer_bytes(wl)
        gbs = nbytes / gemm_avg_s / 1e9
        hbm = float(peaks["hbm_gbs"])
        roofline = {"bound": "hbm", "kernel": "decode_shrink_kernel + decode_gemm_kernel",
                    "achieved": gbs, "peak": hbm, "unit": "GB/s", "frac": gbs / hbm,
                    "peak_source": f"{peak_kind}: copy bandwidth {hbm} GB/s",
                    "frac_of_nominal": gbs / NOMINAL_HBM_GBS,
                    "layer_us": gemm_avg_s * 1e6, "traffic": kernel_traffic(wl.spec.name),
                    "traffic_unit": "bytes per layer call (ncu dram read+write, both kernels)",
                    "algorithmic_bytes": nbytes}
    else:
        # context: the nominal dense int8 rate at the SM clock sampled under load
        sm_mhz = (clocks or {}).get("sm_mhz") or 0.0
        n_sm = torch.cuda.get_device_properties(dev).multi_processor_count
        clk_peak = n_sm * NOMINAL_INT8_OPS_PER_SM_CLK * sm_mhz * 1e6 / 1e12
        roofline = {"bound": "tensor", "kernel": "w8a8_lora_gemm_kernel", "achieved": gemm_tops,
                    "peak": int8_peak, "unit": "TOPS", "frac": gemm_tops / int8_peak,
                    "peak_source": f"{peak_kind}: 2 x bf16 burst {peaks['bf16_tflops']} TFLOP/s",
                    "clock_normalized_peak": clk_peak or None,
                    "frac_of_clock_normalized": (gemm_tops / clk_peak) if clk_peak else None,
                    "gemm_us": gemm_avg_s * 1e6, "traffic": kernel_traffic(wl.spec.name),
                    "traffic_unit": "bytes per launch (ncu dram read+write)",
                    "algorithmic_ops": ops_step}
    entry = {
        "value": value,
        "unit": "TOPS",
        "ms_per_step": t_step_total / n,
        "tokens_per_s": tok_s,
        "config": {"workload": wl.spec.name, "M": M, "K": K, "N": N,
                   "adapters": len(wl.adapters), "ranks": sorted(set(a.r for a in wl.adapters)),
                   "segments": int(len(wl.seg_adapter)), "alpha": wl.alpha,
                   "step": (("sq_rmsnorm_quant_act" if norm else
                             "sq_quant_act_static" if static else "sq_quant_act") +
                            (" + sq_lora_shrink_raw + sq_linear_lora_from_t "
                             "(LoRA on the raw bf16 activations)" if raw else
                             " + sq_linear_lora (shrink + fused GEMM)")),
                   "act_quant": args.act_quant,
                   "l2": "flushed between timed steps (256 MiB write + 256 MiB read, untimed)",
                   "parallelism": f"replicas x{world}"},
        "lora_flops_per_step": lora_flops(wl),
        "roofline": roofline,
        "cpu_baseline": cpu,
        "e2e": e2e,
        "clocks": clocks,
        "gpu_launches": launches_per_step * n * world,
    }
    if repeated is not None:
        entry["repeated"] = repeated
    return entry


def run_ours(args):
    import torch
    import torch.distributed as dist

    import w8a8_smoothquant_int8_b200 as sq

    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    if world > 1:
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                device_id=dev)
    if sq.sq_device_supported(local_rank) != 0:
        raise SystemExit("device is not compute capability 10.0")

    with_cpu = rank == 0 and world == 1 and not args.no_cpu_baseline
    if args.workload == "all":
        head, beside = HEADLINE, BESIDE
    else:
        head, beside = args.workload, []

    entries = {}
    for name in [head] + beside:
        secs = (CPU_SECONDS_HEADLINE if name == head else CPU_SECONDS_BESIDE) if with_cpu else 0.0
        entries[name] = measure(name, args, dev, world, local_rank, secs)
        torch.cuda.empty_cache()

    h = entries[head]
    line = {
        "metric": METRIC,
        "value": h["value"],
        "unit": "TOPS",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": h["ms_per_step"],
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "int8",
        "data": "synthetic",
        "config": h["config"],
        "tokens_per_s": h["tokens_per_s"],
        "lora_flops_per_step": h["lora_flops_per_step"],
        "roofline": h["roofline"],
        "cpu_baseline": h["cpu_baseline"],
        "e2e": h["e2e"],
        "clocks": h["clocks"],
        "gpu_launches": h["gpu_launches"],
    }
    if "repeated" in h:
        line["repeated"] = h["repeated"]
    if beside:
        line["workloads"] = {name: entries[name] for name in beside}
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    if rank == 0:
        print(json.dumps(line), flush=True)
    return 0


def main():
    args = parse()
    if args.impl == "reference":
        return run_reference(args)
    return run_ours(args)


if __name__ == "__main__":
    sys.exit(main())
