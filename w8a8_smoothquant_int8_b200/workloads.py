"""Seeded synthetic workloads for the SmoothQuant W8A8 + per-request LoRA linear.

This module only draws random numbers and lays them out. It holds none of the
method's arithmetic (no smoothing, no quantization, no GEMM): both the CPU
oracle and the CUDA library are fed the bytes produced here.

Workload recipe (one entry per named workload, sizes from the Llama-3-8B layer
shapes the benchmark is quoted on):

* activations X: ``normal`` = N(0, 1); ``heavy`` = sign(z)·|z|^1.5 with
  z ~ N(0, 1).  A fixed set of outlier channels (the same for every token and
  for the calibration batch) is multiplied either by a constant or by a
  per-channel factor drawn once from U(lo, hi).  X is drawn in fp32 and, for
  bf16 workloads, rounded to bf16 (round-to-nearest-even).
* calibration batch: a separate batch from the same distribution, same
  outlier channels and multipliers.
* weights W [N, K] (torch ``Linear`` layout: output channels by input
  channels): N(0, 0.02), rounded to bf16.
* LoRA adapter a of rank r: A [r, K] ~ N(0, (1/r)^2), B [N, r] ~ N(0, 0.01^2),
  both bf16, lora_alpha = 2r (so the scaling alpha/r is 2).
* request segments: ``single`` (one segment, adapter 0); ``random`` (S-1
  distinct cut points drawn uniformly from [1, M-1], sorted, adapter drawn
  uniformly, or -1 = no adapter with probability p_none); ``per_token``
  (segment i = token i, adapter i).

The draw order is fixed (outlier channels, multipliers, W, calibration X, X,
adapters, segments), so a (spec, seed) pair always yields the same bytes.
"""

from __future__ import annotations

import dataclasses
from typing import List, Optional

import numpy as np


def f32_to_bf16_bits(a: np.ndarray) -> np.ndarray:
    """Round fp32 values to bf16 (nearest, ties to even); returns uint16 bit patterns."""
    a = np.ascontiguousarray(a, dtype=np.float32)
    u = a.view(np.uint32)
    bias = ((u >> 16) & np.uint32(1)) + np.uint32(0x7FFF)
    return ((u + bias) >> 16).astype(np.uint16)


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    """Widen bf16 bit patterns (uint16) to fp32 values (exact)."""
    b = np.ascontiguousarray(b, dtype=np.uint16)
    return (b.astype(np.uint32) << 16).view(np.float32)


@dataclasses.dataclass(frozen=True)
class WorkloadSpec:
    name: str
    M: int
    K: int
    N: int
    x_dtype: str            # "f32" or "bf16"
    x_dist: str             # "normal" or "heavy"
    n_outliers: int
    outlier_lo: float       # multiplier drawn from U(lo, hi); lo == hi -> constant
    outlier_hi: float
    alpha: float
    calib_tokens: int
    ranks: tuple            # one entry per adapter
    segments: str           # "single", "random" or "per_token"
    n_segments: int = 1
    p_none: float = 0.0

    @property
    def ops(self) -> int:
        """Integer ops of the base GEMM (2*M*N*K), the unit of the TOPS figure."""
        return 2 * self.M * self.N * self.K


# The five benchmark workloads (sizes and distributions as stated with the
# benchmark) plus small parity workloads that span several GEMM tiles with
# ragged tails and finish in seconds on the CPU oracle.
SPECS = {
    "tiny_m16_k256_n256": WorkloadSpec(
        "tiny_m16_k256_n256", 16, 256, 256, "f32", "normal", 4, 50.0, 50.0,
        0.5, 128, (8,), "single"),
    "llama3_8b_qkv_m2048_k4096_n6144": WorkloadSpec(
        "llama3_8b_qkv_m2048_k4096_n6144", 2048, 4096, 6144, "bf16", "normal",
        20, 20.0, 100.0, 0.5, 512, (16,), "single"),
    "llama3_8b_gateup_m8192_k4096_n28672": WorkloadSpec(
        "llama3_8b_gateup_m8192_k4096_n28672", 8192, 4096, 28672, "bf16",
        "normal", 20, 20.0, 100.0, 0.8, 512, (8, 16, 32, 64, 8, 16, 32, 64),
        "random", 32, 0.1),
    "llama3_8b_down_m16384_k14336_n4096": WorkloadSpec(
        "llama3_8b_down_m16384_k14336_n4096", 16384, 14336, 4096, "bf16",
        "heavy", 143, 80.0, 80.0, 0.5, 512, (32, 32, 32, 32), "random", 64, 0.0),
    "llama3_8b_oproj_decode_m64_k4096_n4096": WorkloadSpec(
        "llama3_8b_oproj_decode_m64_k4096_n4096", 64, 4096, 4096, "bf16",
        "normal", 20, 50.0, 50.0, 0.5, 512, (16,) * 64, "per_token", 64),
    # parity-sized: several 128-row and 256-column tiles, ragged M/N/K tails,
    # several adapters of different ranks, segments with no adapter.
    "parity_ragged": WorkloadSpec(
        "parity_ragged", 333, 1040, 784, "bf16", "normal", 8, 20.0, 100.0,
        0.5, 200, (8, 16, 64), "random", 7, 0.25),
    "parity_heavy_f32": WorkloadSpec(
        "parity_heavy_f32", 257, 528, 272, "f32", "heavy", 6, 80.0, 80.0,
        0.8, 64, (32, 16), "random", 5, 0.2),
    "parity_decode": WorkloadSpec(
        "parity_decode", 64, 1024, 512, "bf16", "normal", 5, 50.0, 50.0,
        0.5, 128, (16,) * 64, "per_token", 64),
    # more than four waves of 256x256 output tiles on 74 CTA pairs (9 x 36 =
    # 324 tiles, the last row and column ragged), a ragged K tail, four
    # adapters of different ranks and segments without an adapter: the
    # persistent schedule, the double-buffered accumulators and the deferred
    # LoRA MMAs all run, and the oracle still checks every element in seconds
    "parity_waves": WorkloadSpec(
        "parity_waves", 2300, 272, 9200, "bf16", "normal", 6, 20.0, 100.0,
        0.5, 256, (8, 16, 64, 32), "random", 9, 0.2),
    # short segments (a few tokens each: many 16-token groups with three to
    # five adapters, so the shrink makes several passes over a group), an
    # adapter of rank 80 (two 64-column blocks), a ragged K tail.  The first
    # is small enough for the warp-MMA form of the shrink; the second runs
    # its tensor-memory form (several sweeps over K where a 128-token block
    # uses more than five 32-column slots), the raw-input form's two-group
    # blocks, and 65 GEMM row tiles
    "parity_segments": WorkloadSpec(
        "parity_segments", 3300, 272, 320, "bf16", "normal", 6, 20.0, 100.0,
        0.5, 256, (8, 16, 64, 32, 80), "random", 700, 0.2),
    "parity_segments_large": WorkloadSpec(
        "parity_segments_large", 16500, 272, 320, "bf16", "normal", 6, 20.0, 100.0,
        0.5, 256, (8, 16, 64, 32, 80), "random", 2000, 0.2),
}

# benchmark workloads in the order they are listed with the benchmark
BENCH_ORDER = [
    "tiny_m16_k256_n256",
    "llama3_8b_qkv_m2048_k4096_n6144",
    "llama3_8b_gateup_m8192_k4096_n28672",
    "llama3_8b_down_m16384_k14336_n4096",
    "llama3_8b_oproj_decode_m64_k4096_n4096",
]


def default_seed(name: str) -> int:
    if name in BENCH_ORDER:
        return 1000 + BENCH_ORDER.index(name)
    return 2000 + sorted(SPECS).index(name)


@dataclasses.dataclass
class Adapter:
    A: np.ndarray            # uint16 bf16 bits [r, K]
    B: np.ndarray            # uint16 bf16 bits [N, r]
    r: int
    lora_alpha: float


@dataclasses.dataclass
class Workload:
    spec: WorkloadSpec
    seed: int
    X: np.ndarray            # [M, K] float32, or uint16 bf16 bits
    X_cal: np.ndarray        # [calib, K], same dtype as X
    W: np.ndarray            # [N, K] uint16 bf16 bits
    adapters: List[Adapter]
    seg_offsets: np.ndarray  # int32 [S+1]
    seg_adapter: np.ndarray  # int32 [S]
    alpha: float

    @property
    def M(self):
        return self.spec.M

    @property
    def K(self):
        return self.spec.K

    @property
    def N(self):
        return self.spec.N

    @property
    def x_is_bf16(self) -> bool:
        return self.spec.x_dtype == "bf16"


def _base_draw(rng: np.random.Generator, shape, dist: str) -> np.ndarray:
    z = rng.standard_normal(shape, dtype=np.float32)
    if dist == "normal":
        return z
    if dist == "heavy":
        return (np.sign(z) * np.abs(z) ** np.float32(1.5)).astype(np.float32)
    raise ValueError(dist)


def _segments(rng, spec: WorkloadSpec, n_adapters: int):
    M = spec.M
    if spec.segments == "single":
        return np.array([0, M], np.int32), np.array([0], np.int32)
    if spec.segments == "per_token":
        return np.arange(M + 1, dtype=np.int32), (np.arange(M) % n_adapters).astype(np.int32)
    if spec.segments == "random":
        S = spec.n_segments
        cuts = np.sort(rng.choice(np.arange(1, M), size=S - 1, replace=False))
        offs = np.concatenate([[0], cuts, [M]]).astype(np.int32)
        adapters = rng.integers(0, n_adapters, size=S).astype(np.int32)
        if spec.p_none > 0:
            none = rng.random(S) < spec.p_none
            adapters[none] = -1
        return offs, adapters
    raise ValueError(spec.segments)


def make_workload(spec, seed: Optional[int] = None, M: Optional[int] = None) -> Workload:
    """Draw the workload ``spec`` (a WorkloadSpec or a name in SPECS).

    ``M`` overrides the token count (used to draw a bounded sample of a large
    workload with the same distribution).
    """
    if isinstance(spec, str):
        spec = SPECS[spec]
    if M is not None and M != spec.M:
        spec = dataclasses.replace(spec, M=M, name=f"{spec.name}[M={M}]")
    if seed is None:
        seed = default_seed(spec.name.split("[")[0])
    rng = np.random.default_rng(np.random.PCG64(seed))
    K, N = spec.K, spec.N
    out_ch = np.sort(rng.choice(K, size=spec.n_outliers, replace=False))
    if spec.outlier_lo == spec.outlier_hi:
        mult = np.full(spec.n_outliers, spec.outlier_lo, np.float32)
    else:
        mult = rng.uniform(spec.outlier_lo, spec.outlier_hi, spec.n_outliers).astype(np.float32)
    W = f32_to_bf16_bits(rng.standard_normal((N, K), dtype=np.float32) * np.float32(0.02))

    def draw_x(rows):
        x = _base_draw(rng, (rows, K), spec.x_dist)
        x[:, out_ch] *= mult
        return x if spec.x_dtype == "f32" else f32_to_bf16_bits(x)

    X_cal = draw_x(spec.calib_tokens)
    X = draw_x(spec.M)
    adapters = []
    for r in spec.ranks:
        A = f32_to_bf16_bits(rng.standard_normal((r, K), dtype=np.float32) * np.float32(1.0 / r))
        B = f32_to_bf16_bits(rng.standard_normal((N, r), dtype=np.float32) * np.float32(0.01))
        adapters.append(Adapter(A, B, r, float(2 * r)))
    seg_offsets, seg_adapter = _segments(rng, spec, len(adapters))
    return Workload(spec, seed, X, X_cal, W, adapters, seg_offsets, seg_adapter, spec.alpha)


def norm_gamma(K: int, seed: int) -> np.ndarray:
    """Weight of an RMS normalization in front of the layer, f32 [K]:
    1 + 0.1 * N(0, 1), drawn from its own seeded stream."""
    rng = np.random.default_rng(np.random.PCG64(seed + 7777))
    return (1.0 + 0.1 * rng.standard_normal(K)).astype(np.float32)


def row_adapter(seg_offsets: np.ndarray, seg_adapter: np.ndarray, M: int, n_adapters: int) -> np.ndarray:
    """Adapter index per token (-1 = none) implied by a segment table (layout helper)."""
    out = np.full(M, -1, np.int64)
    for s in reversed(range(len(seg_adapter))):  # the first segment that holds a row wins
        a = int(seg_adapter[s])
        lo, hi = max(0, int(seg_offsets[s])), min(M, int(seg_offsets[s + 1]))
        if hi > lo:
            out[lo:hi] = a if 0 <= a < n_adapters else -1
    return out
