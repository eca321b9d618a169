"""Parity of the small-M (decode) form of the linear layer with the oracle.

Calls with at most 64 tokens take the streaming form (a shrink grid and CTA
pairs that split K, with the pair's int32 halves added through distributed
shared memory).  These cases walk its shapes and tables: one token to 64;
N from one 16-channel group to several tiles per pair; K of one stage, a
ragged last stage and the shrink's K slices up to their cap; adapters used
by most tokens (whole B' rows copied into shared memory during the K loop)
and by few (each thread's B' words copied for ranks up to 16, read from
global memory above); ranks 8 to 256; segments with no adapter, segment tables that are
not sorted or overlap (the first segment holding a token wins), more
segments than threads, and more adapters than the staged table holds.
Bars: int32 accumulators bit-exact, Y within 1e-2 and the delta within 5e-3
(max-norm relative), as for the other forms.
"""

import numpy as np
import pytest

import oracle
from w8a8_smoothquant_int8_b200 import workloads as wk

pytestmark = pytest.mark.gpu

Y_TOL = 1e-2
DELTA_TOL = 5e-3


def _case(M, N, K, ranks, seg, ad, seed=0, pack=None):
    """Quantized operands from the oracle, the adapters packed on the GPU;
    `pack` = (offsets, R, slot) packs adapter a into column block offsets[a]
    of a width-R pack from the base adapter slot[a] (aliases share columns)."""
    import torch
    import w8a8_smoothquant_int8_b200 as sq
    from tests.gpu_pipeline import to_dev
    rng = np.random.default_rng(seed + 31 * M + 7 * N + K)
    X = wk.f32_to_bf16_bits(rng.standard_normal((M, K)).astype(np.float32))
    X[:, rng.choice(K, max(1, K // 200), replace=False)] = wk.f32_to_bf16_bits(
        np.full(1, 40.0, np.float32))[0]
    W = wk.f32_to_bf16_bits(rng.standard_normal((N, K)).astype(np.float32) * 0.02)
    s = rng.uniform(0.5, 2, K).astype(np.float32)
    Wq, ws = oracle.quantize_weight(W, s)
    Xq, xs = oracle.quant_act(X, s)
    base = list(ranks)
    As = [wk.f32_to_bf16_bits(rng.standard_normal((r, K)).astype(np.float32) / r) for r in base]
    Bs = [wk.f32_to_bf16_bits(rng.standard_normal((N, r)).astype(np.float32) * 0.01) for r in base]
    if pack is None:
        lora = sq.LoraPack.build([to_dev(a) for a in As], [to_dev(b) for b in Bs],
                                 [2.0 * r for r in base], to_dev(s))
        slot = list(range(len(base)))
        n_ad = len(base)
    else:
        offsets, R, slot = pack
        n_ad = len(slot)
        A_pack = torch.zeros((R, K), dtype=torch.bfloat16, device="cuda")
        B_pack = torch.zeros((N, R), dtype=torch.bfloat16, device="cuda")
        for b in sorted(set(slot)):
            a = slot.index(b)
            sq.sq_prepare_lora(to_dev(As[b]), to_dev(Bs[b]), to_dev(s), 2.0 * base[b], R,
                               offsets[a], A_pack, B_pack)
        lora = sq.LoraPack(A_pack, B_pack, to_dev(np.array(offsets, np.int32)),
                           to_dev(np.array([base[b] for b in slot], np.int32)), R, n_ad)
    seg = np.array(seg, np.int32)
    ad = np.array(ad, np.int32)
    ws_buf = torch.empty(max(sq.sq_linear_lora_workspace_size(M, lora.R), 256),
                         dtype=torch.uint8, device="cuda")
    Xq_d, xs_d, Wq_d, wsc_d = to_dev(Xq), to_dev(xs), to_dev(Wq), to_dev(ws)
    seg_d, ad_d = to_dev(seg), to_dev(ad)
    Y = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
    sq.sq_linear_lora(Xq_d, xs_d, Wq_d, wsc_d, lora, seg_d, ad_d, Y, ws_buf)
    delta = torch.empty((M, N), dtype=torch.float32, device="cuda")
    sq.sq_lora_delta(Xq_d, xs_d, N, lora, seg_d, ad_d, delta, ws_buf)
    acc = torch.empty((M, N), dtype=torch.int32, device="cuda")
    sq.sq_gemm_i32(Xq_d, Wq_d, acc)
    torch.cuda.synchronize()
    A_s, B_s = [], []
    for b in slot:
        x, y = oracle.prepare_lora(As[b], Bs[b], s, 2.0 * base[b])
        A_s.append(x)
        B_s.append(y)
    ref = oracle.linear_lora_rows(Xq, xs, Wq, ws, A_s, B_s, seg, ad,
                                  want=("Y", "delta", "acc"))
    return (Y.float().cpu().numpy(), delta.cpu().numpy(), acc.cpu().numpy(), ref,
            wk.row_adapter(seg, ad, M, n_ad))


def _check(M, N, K, ranks, seg, ad, **kw):
    import w8a8_smoothquant_int8_b200 as sq
    from tests.gpu_pipeline import rel_err
    sq.sq_get_device_error(clear=True)
    Y, d, acc, ref, row_ad = _case(M, N, K, ranks, seg, ad, **kw)
    assert np.array_equal(acc.astype(np.int64), ref["acc"])
    assert rel_err(Y, ref["Y"]) <= Y_TOL
    if np.abs(ref["delta"]).max() > 0:
        assert rel_err(d, ref["delta"]) <= DELTA_TOL
    assert not d[row_ad < 0].any()
    assert sq.sq_get_device_error(clear=True) == 0


def _per_token(M, n_ad):
    return list(range(M + 1)), [i % n_ad for i in range(M)]


# (M, N, K): one token to 64; N = one 16-channel group, a few groups, one
# tile per pair, several tiles per pair; K = one stage, a ragged stage, the
# shrink's K slices (K / 2048 of them, at most 8)
@pytest.mark.parametrize("M,N,K", [(1, 16, 16), (7, 48, 144), (33, 784, 1040), (64, 512, 1024),
                                   (64, 4096, 4096), (17, 9216, 2064), (64, 256, 14336),
                                   (5, 160, 20000)])
def test_decode_shapes_per_token_adapters(M, N, K):
    seg, ad = _per_token(M, min(M, 8))
    _check(M, N, K, [16] * min(M, 8), seg, ad)


def test_decode_dense_pack_of_64_adapters():
    # every token its own rank-16 adapter: the B' rows of each CTA's channels
    # are copied into shared memory during the K loop
    seg, ad = _per_token(64, 64)
    _check(64, 1024, 2048, [16] * 64, seg, ad, pack=([16 * a for a in range(64)], 1024,
                                                     list(range(64))))


def test_decode_sparse_use_reads_b_from_global():
    # a 1024-column pack of which the tokens use one 16-column block
    seg, ad = [0, 64], [37]
    _check(64, 512, 1024, [16] * 64, seg, ad, pack=([16 * a for a in range(64)], 1024,
                                                    list(range(64))))


def test_decode_sparse_use_of_a_wide_adapter_reads_b_from_global():
    # a 1024-column pack of sixteen rank-64 adapters of which the tokens use
    # two: too few columns for whole rows, ranks too wide for the copied words
    seg, ad = [0, 20, 64], [5, 11]
    _check(64, 400, 1040, [64] * 16, seg, ad, pack=([64 * a for a in range(16)], 1024,
                                                    list(range(16))))


def test_decode_mixed_ranks_and_none():
    # ranks 8 .. 256 (the largest), tokens without an adapter
    ranks = [8, 64, 256, 32]
    seg = [0, 3, 10, 11, 20, 33, 40]
    ad = [0, -1, 2, 1, 3, -1]
    _check(40, 304, 528, ranks, seg, ad)


def test_decode_unsorted_overlapping_and_many_segments():
    # the first segment that holds a token decides; overlapping and reversed
    # ranges; more segments than a block has threads
    ranks = [16, 32, 8]
    seg = [10, 20, 0, 15, 64, 5, 12]
    ad = [1, 0, 2, 1, -1, 2]
    _check(64, 400, 1040, ranks, seg, ad)
    n = 700  # 699 empty segments around one that covers tokens 3..9
    seg2 = [3] * 300 + [10] + [10] * (n - 301)
    ad2 = [2] * (n - 1)
    _check(12, 64, 256, ranks, seg2, ad2)


def test_decode_more_adapters_than_the_staged_table():
    # 300 adapter indices aliasing 4 column blocks: the offsets and ranks are
    # read from global memory
    slot = [a % 4 for a in range(300)]
    offsets = [16 * (a % 4) for a in range(300)]
    seg = list(range(0, 64, 2)) + [64]
    ad = [(7 * j) % 300 for j in range(32)]
    _check(64, 208, 512, [16] * 4, seg, ad, pack=(offsets, 64, slot))
