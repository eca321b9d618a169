"""GPU parity of the folded norm weight and the fused RMS norm + per-token
quantization with the oracle ("SmoothQuant" explainer, Steps 5 and 6).

Everything is bit-exact: the fold, and the fused kernel's codes and scales.
The norm factor r_i depends on the sum of the squares of the row, which the
oracle defines as the exact sum rounded once to fp64.  The kernel sums in
fp64 as a tree and keeps that result only when the tree's error bound cannot
change r_i; other rows take an exact integer sum.  Rows built so that r_i
hangs on the last bit of the sum (an exact fp64 tie, a tie plus a sticky
term, just below a tie; squares spanning some 2^72) check that exact sum.
"""

import math

import numpy as np
import pytest

import oracle
from w8a8_smoothquant_int8_b200 import workloads as wk

pytestmark = pytest.mark.gpu

EPS = 1e-6


def _gpu_norm_quant(H, gamma, s, eps=EPS):
    import torch
    import w8a8_smoothquant_int8_b200 as sq
    from tests.gpu_pipeline import to_dev
    Hd, g, sd = to_dev(H), to_dev(gamma), to_dev(s)
    gs = torch.empty_like(g)
    sq.sq_fold_norm_weight(g, sd, gs)
    M, K = H.shape
    Xq = torch.empty((M, K), dtype=torch.int8, device="cuda")
    xs = torch.empty(M, dtype=torch.float32, device="cuda")
    sq.sq_rmsnorm_quant_act(Hd, gs, eps, Xq, xs)
    return gs.cpu().numpy(), Xq.cpu().numpy(), xs.cpu().numpy()


@pytest.mark.parametrize("name", ["parity_ragged", "parity_decode",
                                  "llama3_8b_qkv_m2048_k4096_n6144",
                                  "llama3_8b_down_m16384_k14336_n4096"])
def test_norm_fold_and_quant(name):
    wl = wk.make_workload(name)
    a = oracle.act_absmax_update(wl.X_cal)
    s = oracle.compute_smoothing(a, oracle.weight_absmax(wl.W), wl.alpha)
    gamma = wk.norm_gamma(wl.K, wl.seed)
    gs_ref = oracle.fold_norm_weight(gamma, s)
    Xq_ref, xs_ref = oracle.rmsnorm_quant_act(wl.X, gs_ref, EPS)
    gs, Xq, xs = _gpu_norm_quant(wl.X, gamma, s)
    assert np.array_equal(gs.view(np.uint32), gs_ref.view(np.uint32))
    bad = np.nonzero((xs.view(np.uint32) != xs_ref.view(np.uint32)) | (Xq != Xq_ref).any(1))[0]
    assert len(bad) == 0, bad[:10]


def test_norm_quant_constant_and_zero_rows():
    # a constant row (every code 127, scale RN(1/127) with eps = 0) and a zero
    # row (scale 0, codes 0)
    K = 256
    H = wk.f32_to_bf16_bits(np.stack([np.full(K, 3.0), np.zeros(K)]).astype(np.float32))
    gamma = np.ones(K, np.float32)
    s = np.ones(K, np.float32)
    _, Xq, xs = _gpu_norm_quant(H, gamma, s, eps=0.0)
    assert (Xq[0] == 127).all() and xs[0] == np.float32(1.0 / 127.0)
    assert not Xq[1].any() and xs[1] == 0.0


def test_norm_fold_through_the_linear_layer():
    from tests.gpu_pipeline import GpuRun, rel_err, to_dev
    import torch
    import w8a8_smoothquant_int8_b200 as sq
    wl = wk.make_workload("llama3_8b_qkv_m2048_k4096_n6144")
    P = oracle.Prepared(wl)
    g = GpuRun(wl, s_host=P.s)
    gamma = wk.norm_gamma(wl.K, wl.seed)
    gs = torch.empty(wl.K, dtype=torch.float32, device="cuda")
    sq.sq_fold_norm_weight(to_dev(gamma), g.s, gs)
    sq.sq_rmsnorm_quant_act(g.X, gs, EPS, g.Xq, g.x_scale)
    g.linear()
    Xq, xs = oracle.rmsnorm_quant_act(wl.X, oracle.fold_norm_weight(gamma, P.s), EPS)
    rows = np.unique(np.concatenate([[0, wl.M - 1], np.random.default_rng(8).choice(wl.M, 24)]))
    ref = oracle.linear_lora_rows(Xq, xs, P.Wq, P.w_scale, P.A_s, P.B_s, wl.seg_offsets,
                                  wl.seg_adapter, rows, want=("Y",))["Y"]
    assert rel_err(g.Y_f32()[rows], ref) <= 1e-2


def _assert_parity(H, gamma_s_host, eps, gs_dev=None):
    """Codes and scales of the GPU kernel against the oracle, bit for bit."""
    import torch
    import w8a8_smoothquant_int8_b200 as sq
    from tests.gpu_pipeline import to_dev
    M, K = H.shape
    Xq = torch.empty((M, K), dtype=torch.int8, device="cuda")
    xs = torch.empty(M, dtype=torch.float32, device="cuda")
    sq.sq_rmsnorm_quant_act(to_dev(H), to_dev(gamma_s_host), eps, Xq, xs)
    Xq, xs = Xq.cpu().numpy(), xs.cpu().numpy()
    Xq_ref, xs_ref = oracle.rmsnorm_quant_act(H, gamma_s_host, eps)
    bad = np.nonzero((xs.view(np.uint32) != xs_ref.view(np.uint32)) | (Xq != Xq_ref).any(1))[0]
    assert len(bad) == 0, (bad[:10], xs[bad[:3]], xs_ref[bad[:3]])
    return xs_ref


def _rows(M, K, seed, scale_exp=0.0):
    # N(0, 1) entries, a log-normal magnitude per row and a few outlier
    # channels (x20), as bf16
    rng = np.random.default_rng(seed)
    X = rng.standard_normal((M, K)) * np.exp(rng.standard_normal((M, 1)))
    X[:, rng.choice(K, max(1, K // 256), replace=False)] *= 20.0
    return wk.f32_to_bf16_bits((X * 2.0 ** scale_exp).astype(np.float32))


# every team shape of the streaming kernel (rows of 2 to 2048 16-byte
# vectors), the block-per-row kernel beyond, ragged row counts and grids with
# fewer rows than blocks
@pytest.mark.parametrize("K,M", [(16, 37), (1024, 300), (1040, 129), (2048, 300), (4096, 1),
                                 (4096, 517), (8192, 300), (14336, 3), (14336, 261),
                                 (16384, 200), (16400, 70), (32768, 40)])
def test_norm_quant_shapes(K, M):
    H = _rows(M, K, seed=K + M)
    gs = wk.norm_gamma(K, K) / np.float32(1.5)
    _assert_parity(H, gs.astype(np.float32), EPS)


@pytest.mark.parametrize("K", [256, 4096, 14336])
def test_norm_quant_range_edges(K):
    # rows whose mean square leaves [2^-100, 2^100] (tiny and huge values
    # with eps = 0) take the correctly rounded square root and division; a
    # huge eps puts the row maximum below 2^-60 (IEEE divisions per element);
    # single-element rows give codes of +-127; an all-zero row with eps = 0
    # gives r = inf, xt = NaN and codes 0
    gs = wk.norm_gamma(K, 3).astype(np.float32)
    for exp, eps in [(-60.0, 0.0), (60.0, 0.0), (0.0, 2.0 ** 126), (-20.0, 2.0 ** 126),
                     (-30.0, 1e-6)]:
        _assert_parity(_rows(9, K, seed=int(exp) + 100, scale_exp=exp), gs, eps)
    H = np.zeros((3, K), np.uint16)
    H[0, 5] = wk.f32_to_bf16_bits(np.array([-3.0], np.float32))[0]
    H[1, K - 1] = wk.f32_to_bf16_bits(np.array([2.0 ** -70], np.float32))[0]
    _assert_parity(H, gs, 0.0)


def _bf16_floor_sqrt(R):
    """Largest bf16 value h with h*h <= R (R a positive Fraction), as
    (significand m in [128, 255], exponent e): h = m * 2^e."""
    from fractions import Fraction
    e = (R.numerator.bit_length() - R.denominator.bit_length()) // 2 - 8
    while True:
        x = R / Fraction(2) ** (2 * e)
        m = math.isqrt(x.numerator // x.denominator)
        if m < 128:
            e -= 1
        elif m > 255:
            e += 1
        else:
            return m, e


def _midpoint_row(K, f, delta_exp, sign):
    """A bf16 row and an eps whose r = 1/sqrt(t) lies at (1 + sign*2^delta_exp)
    times the point halfway between the float f and the next float up (t
    from the oracle's fp64 steps).  eps carries t's leading bits; a few
    squares whose fp64 sum is exact in any order supply the rest."""
    from fractions import Fraction
    f32 = np.float32(f)
    mid = (Fraction(float(f32)) + Fraction(float(np.nextafter(f32, np.float32(np.inf))))) / 2
    target = mid * (1 + sign * Fraction(2) ** delta_exp) if delta_exp is not None else mid
    T = 1 / (target * target)
    eps = np.float32(float(T))
    while Fraction(float(eps)) > T:
        eps = np.nextafter(eps, np.float32(0))
    R = (T - Fraction(float(eps))) * K
    terms = []
    for _ in range(4):
        if R <= 0:
            break
        m, e = _bf16_floor_sqrt(R)
        # keep the squares' sum within 53 bits from the smallest's last bit
        trial = terms + [(m, e)]
        emin = min(2 * ee for _, ee in trial)
        total = sum(mm * mm << (2 * ee - emin) for mm, ee in trial)
        if total.bit_length() > 53:
            break
        terms = trial
        R -= Fraction(m * m) * Fraction(2) ** (2 * e)
    vals = np.array([m * 2.0 ** e for m, e in terms], np.float32)
    H = np.zeros(K, np.uint16)
    H[np.arange(len(vals)) * (K // max(1, len(vals))) % K] = wk.f32_to_bf16_bits(vals)
    # the oracle's t and the distance of 1/sqrt(t) from the midpoint
    ss = 0.0
    for v in wk.bf16_bits_to_f32(H).astype(np.float64):
        ss += v * v
    t = ss / K + float(eps)
    q = 1 / (Fraction(t) * mid * mid)  # (r / mid)^2
    return H, float(eps), abs(float(q - 1)) / 2


def test_norm_factor_near_float_midpoints():
    # r_i = RN32(RN64(1/RN64(sqrt(t)))) when 1/sqrt(t) sits almost exactly
    # halfway between two floats: within 2^-46 the kernel takes the correctly
    # rounded square root and division; at 2^-44 its Newton estimate decides
    # (it is within 2^-51 of the double-rounded value)
    for K in (16, 4096, 14336):
        gs = np.ones(K, np.float32)
        rows, epss = [], []
        for f in (1.0 + 2.0 ** -20, 1.2345, 0.777, 3.5, 0.0123):
            for delta_exp, sign in [(None, 0), (-50, 1), (-50, -1), (-44, 1), (-44, -1)]:
                H, eps, dist = _midpoint_row(K, f, delta_exp, sign)
                if delta_exp is None or delta_exp <= -48:
                    assert dist < 2.0 ** -47, (K, f, delta_exp, dist)
                else:
                    assert 2.0 ** -45 < dist < 2.0 ** -43, (K, f, delta_exp, dist)
                rows.append(H)
                epss.append(eps)
        # one call per eps (eps is a scalar of the call)
        for H, eps in zip(rows, epss):
            _assert_parity(H[None, :], gs, eps)


# ---------------------------------------------------------------------------
# rows whose r_i hangs on the rounding of the exact sum of squares
# ---------------------------------------------------------------------------
def _rn64(x):
    from fractions import Fraction
    return Fraction(x.numerator / x.denominator)  # int / int is correctly rounded


def _sqrt_rn64(x):
    """Correctly rounded fp64 square root of a positive fp64 value (exact
    rational in, exact rational out): a 300-bit integer square root, then one
    rounding (an fp64 value's root is never an fp64 midpoint)."""
    from fractions import Fraction
    P = 300
    y = math.isqrt(x.numerator * (1 << (2 * P)) // x.denominator)
    return _rn64(Fraction(y, 1 << P))


def _r_of(ss, K):
    """The oracle's chain with eps = 0: RN32(1 / sqrt(ss / K)), fp64 steps."""
    from fractions import Fraction
    t = _rn64(ss / K)
    return np.float32(float(_rn64(1 / _sqrt_rn64(t))))


def _bits_as_squares(D):
    """bf16 values whose squares add up to the dyadic D exactly: one power of
    two per set bit at an even position, two at an odd one."""
    from fractions import Fraction
    out = []
    num, den = D.numerator, D.denominator
    shift = den.bit_length() - 1  # den is a power of two
    k = 0
    while num:
        if num & 1:
            e = k - shift
            out += [2.0 ** (e // 2)] if e % 2 == 0 else [2.0 ** ((e - 1) // 2)] * 2
        num >>= 1
        k += 1
    return out


def _tie_rows(K, f):
    """Three rows whose exact sums of squares are A + u/2 (an fp64 tie), that
    plus a square of 2^-100 (rounds up) and that less its lowest bit (rounds
    down), with A < K/mid^2 < A + u for the midpoint `mid` above the float f,
    so that r differs between A and A + u.  None when f does not give that."""
    from fractions import Fraction
    f32 = np.float32(f)
    mid = (Fraction(float(f32)) + Fraction(float(np.nextafter(f32, np.float32(np.inf))))) / 2
    target = Fraction(K) / (mid * mid)
    A = _rn64(target)
    if A > target:
        A = Fraction(float(np.nextafter(float(A), 0.0)))
    u = Fraction(float(np.nextafter(float(A), np.inf))) - A
    if _r_of(A, K) == _r_of(A + u, K):
        return None
    # bf16 squares approaching A - 2u from below, to within u / 2^10
    X, terms = A - 2 * u, []
    R = X
    while R > u / 1024:
        m, e = _bf16_floor_sqrt(R)
        terms.append(m * 2.0 ** e)
        R -= Fraction(m * m) * Fraction(2) ** (2 * e)
    D = A + u / 2 - (X - R)
    low = Fraction(1, D.denominator)  # D's lowest set bit
    rows = []
    for vals in (terms + _bits_as_squares(D),
                 terms + _bits_as_squares(D) + [2.0 ** -100],
                 terms + _bits_as_squares(D - low)):
        assert len(vals) <= K
        H = np.zeros(K, np.uint16)
        pos = np.random.default_rng(len(vals)).permutation(K)[:len(vals)]
        H[pos] = wk.f32_to_bf16_bits(np.array(vals, np.float32))
        assert np.array_equal(wk.bf16_bits_to_f32(H[pos]), np.array(vals, np.float32))
        rows.append(H)
    even = A if (A / u).numerator % 2 == 0 else A + u
    expect = [even, A + u, A]
    for H, e in zip(rows, expect):
        assert oracle.sum_squares_bf16(H) == float(e)
    return rows, [_r_of(e, K) for e in expect]


@pytest.mark.parametrize("K", [256, 4096, 16384, 32768])
def test_norm_factor_from_exact_sum_at_fp64_ties(K):
    gs = np.ones(K, np.float32)
    found = 0
    for f in (1.0 + 2.0 ** -20, 1.2345, 0.777, 3.5, 0.0123, 0.301, 1.9, 0.66, 2.71, 0.05,
              1.111, 0.4142, 1.7320508, 0.9, 0.123, 6.25):
        got = _tie_rows(K, f)
        if got is None:
            continue
        rows, rs = got
        assert rs[1] != rs[2]  # the rounding of the sum decides r
        for H in rows:
            _assert_parity(H[None, :], gs, 0.0)
        found += 1
        if found == 3:
            break
    assert found >= 2
