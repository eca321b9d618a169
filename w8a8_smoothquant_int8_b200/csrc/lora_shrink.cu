// LoRA shrink: the low-rank projection of the dequantized activations,
//   T[i, j] = x_scale_i * sum_k Xq[i,k] * A_pack[off_a + j, k]   (j < r_a)
// for the adapter a of token i ("[Feature]: LoRA support for W8A8
// SmoothQuant", Pitch: the LoRA path runs after the INT8 GEMM in BF16; A_pack
// carries the smoothing scale so that Xq*x_scale*diag(s) ~ X).
//
// T is written as two bf16 planes over the packed width R, T_hi = bf16(T) and
// T_lo = bf16(T - T_hi), with zeros outside the token's adapter columns, so
// that the GEMM epilogue can apply every adapter of a 128-token tile with
// dense bf16 tensor-core MMAs and still carry ~16 significant bits of T.
// mask[g] holds, per group of 16 tokens, the 16-column groups of R that some
// token of the group uses (each word written once, by the block of the group).
//
// The contraction is a skinny GEMM (N = rank <= 64 per pass) done with
// warp-level bf16 tensor-core MMAs (m16n8k16, fp32 accumulation): the int8
// codes are exact in bf16, so converting them in registers loses nothing.
// Each thread loads 16 contiguous K values of its two rows per 64-wide K
// chunk; within a chunk the K order seen by the MMA is a permutation that
// both operands share, which leaves the dot products unchanged.
//
// Raw-input form (the issue's Pitch read on the layer's own activations):
// T[i, j] = sum_k X[i,k] * A_pack[off_a + j, k] from the bf16 activations,
// with A_pack holding the adapters as given (packed without the smoothing
// fold); the bf16 values are the MMA operands directly.
#include <cuda_bf16.h>

#include "common.cuh"
#include "ptx_sm100.cuh"
#include "tmap.cuh"

namespace sq {

constexpr int kShrinkWarps = 8;
constexpr int kShrinkThreads = 32 * kShrinkWarps;

// Two signed bytes of w (bytes `first_byte`, `first_byte`+1) -> packed bf16
// pair, exactly.  The byte, biased by 128 (xor 0x80), is placed in the low
// mantissa bits of 2^23 and 2^23 + 128 is subtracted; the result is a small
// integer whose low 16 float bits are zero, so its bf16 pattern is the high
// half of the float.  Needs only byte permutes and adds.
__device__ __forceinline__ uint32_t bf16x2_of_s8(uint32_t w, int first_byte) {
  const uint32_t wb = w ^ 0x80808080u;
  const uint32_t magic = 0x4B000000u;
  const uint32_t sel0 = 0x7650u | static_cast<uint32_t>(first_byte);
  const uint32_t sel1 = 0x7650u | static_cast<uint32_t>(first_byte + 1);
  const float f0 = __fsub_rn(__uint_as_float(__byte_perm(wb, magic, sel0)), 8388736.0f);
  const float f1 = __fsub_rn(__uint_as_float(__byte_perm(wb, magic, sel1)), 8388736.0f);
  return __byte_perm(__float_as_uint(f0), __float_as_uint(f1), 0x7632);
}

__device__ __forceinline__ void mma_bf16_16816(float (&d)[4], const uint32_t (&a)[4],
                                               uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 "
      "{%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, {%0, %1, %2, %3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// Partial products of 16 rows [row0, row0+16) with 8*kNT consecutive rows of
// A_pack starting at `arow0`, over the 64-wide K chunks c = c_begin,
// c_begin + c_step, ...  acc[nt][.] is the m16n8 fragment of columns
// [8nt, 8nt+8).  Two chunks are loaded before either is used, so that each
// warp keeps twice the bytes in flight.
template <int kNT, bool kRaw>
__device__ __forceinline__ void shrink_warp_tile(const void *__restrict__ Xsrc, int64_t M,
                                                 int64_t K, int64_t row0,
                                                 const uint16_t *__restrict__ A_pack, int64_t arow0,
                                                 int c_begin, int c_step, float (&acc)[8][4]) {
  const int lane = threadIdx.x & 31, g = lane >> 2, tig = lane & 3;
  const int64_t ra = row0 + g, rb = row0 + g + 8;
  const int nchunks = static_cast<int>((K + 63) / 64);
#pragma unroll
  for (int nt = 0; nt < 8; ++nt)
#pragma unroll
    for (int t = 0; t < 4; ++t) acc[nt][t] = 0.f;
  // chunks loaded ahead; the raw form's rows are twice as many bytes
  constexpr int kDepth0 = (kNT <= 2) ? 4 : ((kNT <= 4) ? 2 : 1);
  constexpr int kDepth = kRaw ? (kDepth0 > 1 ? kDepth0 / 2 : 1) : kDepth0;
  constexpr int kXW = kRaw ? 2 : 1;  // 16-byte words per row and chunk
  const int8_t *Xq = static_cast<const int8_t *>(Xsrc);
  const uint16_t *Xr = static_cast<const uint16_t *>(Xsrc);
  for (int c0 = c_begin; c0 < nchunks; c0 += kDepth * c_step) {
    uint4 xa[kDepth][kXW], xb[kDepth][kXW], bv[kDepth][kNT][2];
#pragma unroll
    for (int d = 0; d < kDepth; ++d) {
      const int c = c0 + d * c_step;
      const int64_t k = static_cast<int64_t>(c) * 64 + 16 * tig;
      const bool kin = c < nchunks && k < K;  // K % 16 == 0: a 16-slice is all in or out
#pragma unroll
      for (int w = 0; w < kXW; ++w) {
        xa[d][w] = make_uint4(0, 0, 0, 0);
        xb[d][w] = make_uint4(0, 0, 0, 0);
      }
      if constexpr (kRaw) {
        if (kin && ra < M) {
          xa[d][0] = __ldg(reinterpret_cast<const uint4 *>(Xr + ra * K + k));
          xa[d][1] = __ldg(reinterpret_cast<const uint4 *>(Xr + ra * K + k + 8));
        }
        if (kin && rb < M) {
          xb[d][0] = __ldg(reinterpret_cast<const uint4 *>(Xr + rb * K + k));
          xb[d][1] = __ldg(reinterpret_cast<const uint4 *>(Xr + rb * K + k + 8));
        }
      } else {
        if (kin && ra < M) xa[d][0] = __ldg(reinterpret_cast<const uint4 *>(Xq + ra * K + k));
        if (kin && rb < M) xb[d][0] = __ldg(reinterpret_cast<const uint4 *>(Xq + rb * K + k));
      }
#pragma unroll
      for (int nt = 0; nt < kNT; ++nt) {
        bv[d][nt][0] = make_uint4(0, 0, 0, 0);
        bv[d][nt][1] = make_uint4(0, 0, 0, 0);
        if (kin) {
          const uint16_t *ap = A_pack + (arow0 + nt * 8 + g) * K + k;
          bv[d][nt][0] = __ldg(reinterpret_cast<const uint4 *>(ap));
          bv[d][nt][1] = __ldg(reinterpret_cast<const uint4 *>(ap + 8));
        }
      }
    }
#pragma unroll
    for (int d = 0; d < kDepth; ++d) {
      uint32_t afrag[4][4];  // [k16 step][a0..a3]
      if constexpr (kRaw) {
        // elements (4st, 4st+1) and (4st+2, 4st+3) of the 16 are words 2st, 2st+1
        const uint32_t wa[8] = {xa[d][0].x, xa[d][0].y, xa[d][0].z, xa[d][0].w,
                                xa[d][1].x, xa[d][1].y, xa[d][1].z, xa[d][1].w};
        const uint32_t wb[8] = {xb[d][0].x, xb[d][0].y, xb[d][0].z, xb[d][0].w,
                                xb[d][1].x, xb[d][1].y, xb[d][1].z, xb[d][1].w};
#pragma unroll
        for (int st = 0; st < 4; ++st) {
          afrag[st][0] = wa[2 * st];
          afrag[st][1] = wb[2 * st];
          afrag[st][2] = wa[2 * st + 1];
          afrag[st][3] = wb[2 * st + 1];
        }
      } else {
        const uint32_t wa[4] = {xa[d][0].x, xa[d][0].y, xa[d][0].z, xa[d][0].w};
        const uint32_t wb[4] = {xb[d][0].x, xb[d][0].y, xb[d][0].z, xb[d][0].w};
#pragma unroll
        for (int st = 0; st < 4; ++st) {
          afrag[st][0] = bf16x2_of_s8(wa[st], 0);
          afrag[st][1] = bf16x2_of_s8(wb[st], 0);
          afrag[st][2] = bf16x2_of_s8(wa[st], 2);
          afrag[st][3] = bf16x2_of_s8(wb[st], 2);
        }
      }
#pragma unroll
      for (int nt = 0; nt < kNT; ++nt) {
        const uint32_t bw[8] = {bv[d][nt][0].x, bv[d][nt][0].y, bv[d][nt][0].z, bv[d][nt][0].w,
                                bv[d][nt][1].x, bv[d][nt][1].y, bv[d][nt][1].z, bv[d][nt][1].w};
#pragma unroll
        for (int st = 0; st < 4; ++st)
          mma_bf16_16816(acc[nt], afrag[st], bw[2 * st], bw[2 * st + 1]);
      }
    }
  }
}

__device__ __forceinline__ void store_t_pair(uint16_t *T_hi, uint16_t *T_lo, int64_t idx, float v0,
                                             float v1) {
  __nv_bfloat16 h0 = __float2bfloat16_rn(v0), h1 = __float2bfloat16_rn(v1);
  __nv_bfloat16 l0 = __float2bfloat16_rn(v0 - __bfloat162float(h0));
  __nv_bfloat16 l1 = __float2bfloat16_rn(v1 - __bfloat162float(h1));
  *reinterpret_cast<uint32_t *>(T_hi + idx) =
      static_cast<uint32_t>(__bfloat16_as_ushort(h0)) |
      (static_cast<uint32_t>(__bfloat16_as_ushort(h1)) << 16);
  *reinterpret_cast<uint32_t *>(T_lo + idx) =
      static_cast<uint32_t>(__bfloat16_as_ushort(l0)) |
      (static_cast<uint32_t>(__bfloat16_as_ushort(l1)) << 16);
}

// A block of 8 warps covers kRG groups of 16 rows; the kKS = 8/kRG warps of a
// row group split K between them and add their partial sums in a fixed order
// through shared memory.  More row groups per block means more reuse of the
// adapter rows through L1; more K splits means more blocks for small M.
__device__ __forceinline__ void group_sync(int rg, int nwarps) {
  if (nwarps == 1)
    __syncwarp();
  else
    asm volatile("bar.sync %0, %1;" ::"r"(1 + rg), "r"(nwarps * 32) : "memory");
}

template <int kRG, bool kRaw>
__global__ void __launch_bounds__(kShrinkThreads) lora_shrink_kernel(
    const void *__restrict__ Xq, const float *__restrict__ x_scale, int64_t M, int64_t K,
    const uint16_t *__restrict__ A_pack, const int32_t *__restrict__ lora_offset,
    const int32_t *__restrict__ lora_rank, int n_adapters, int64_t R,
    const int32_t *__restrict__ seg_offsets, const int32_t *__restrict__ seg_adapter, int64_t S,
    uint16_t *__restrict__ T_hi, uint16_t *__restrict__ T_lo,
    unsigned long long *__restrict__ mask) {
  constexpr int kKS = kShrinkWarps / kRG;
  __shared__ float red[kShrinkWarps][16][64 + 1];
  __shared__ int s_ad[kRG][16];
  __shared__ int s_off[kRG][16];
  __shared__ int s_rank[kRG][16];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, g = lane >> 2, tig = lane & 3;
  const int rg = warp / kKS, ks = warp % kKS;
  const int64_t row0 = (static_cast<int64_t>(blockIdx.x) * kRG + rg) * 16;
  // everything this grid reads may come from the preceding kernel (a no-op
  // unless the grid is launched as a programmatic dependent)
  asm volatile("griddepcontrol.wait;" ::: "memory");

  // adapter, column offset and rank of each of the 16 rows of the group
  if (ks == 0 && lane < 16) {
    const int64_t i = row0 + lane;
    int a = (i < M) ? token_adapter(seg_offsets, seg_adapter, S, n_adapters, i) : -1;
    int off = 0, r = 0;
    if (a >= 0) {
      off = lora_offset[a];
      r = lora_rank[a];
      if (off < 0 || (off & 15) || r <= 0 || off + ((r + 15) & ~15) > R) {
        record_device_error(SQ_ERR_BAD_SEGMENTS);
        a = -1;
      }
    }
    s_ad[rg][lane] = a;
    s_off[rg][lane] = off;
    s_rank[rg][lane] = r;
  }
  __syncthreads();
  if (row0 >= M) return;  // whole row group; only group barriers follow

  // zero both planes where the group's rows get no value below (outside the
  // row's adapter columns [off, off + rank rounded up to 16); the whole row
  // for a token without adapter), and write the group's mask word
  {
    const int nrows = static_cast<int>((M - row0 < 16) ? (M - row0) : 16);
    const int wpr = static_cast<int>(R / 8);  // 16-byte words per row (R % 16 == 0)
    const int tid = ks * 32 + lane;
    for (int w = tid; w < nrows * wpr; w += kKS * 32) {
      const int r = w / wpr, col = (w - r * wpr) * 8;
      const int a = s_ad[rg][r], off = s_off[rg][r], rpad = (s_rank[rg][r] + 15) & ~15;
      if (a >= 0 && col >= off && col < off + rpad) continue;
      reinterpret_cast<uint4 *>(T_hi + row0 * R)[w] = make_uint4(0, 0, 0, 0);
      reinterpret_cast<uint4 *>(T_lo + row0 * R)[w] = make_uint4(0, 0, 0, 0);
    }
    if (tid == 0) {
      unsigned long long bits = 0;
      for (int r = 0; r < 16; ++r) {
        if (s_ad[rg][r] < 0) continue;
        const int off = s_off[rg][r], rpad = (s_rank[rg][r] + 15) & ~15;
        for (int gi = off / 16; gi < (off + rpad) / 16; ++gi) bits |= 1ull << gi;
      }
      mask[row0 >> 4] = bits;
    }
  }
  group_sync(rg, kKS);

  // one pass per distinct adapter among the 16 rows (usually one)
  unsigned done = 0;  // bit r: row r handled
  for (int r = 0; r < 16; ++r)
    if (s_ad[rg][r] < 0) done |= 1u << r;
  while (done != 0xffffu) {
    const int first = __ffs(~done) - 1;
    const int a = s_ad[rg][first], off = s_off[rg][first], rank = s_rank[rg][first];
    unsigned rows_a = 0;
    for (int r = 0; r < 16; ++r)
      if (s_ad[rg][r] == a) rows_a |= 1u << r;
    const int rpad = (rank + 15) & ~15;
    for (int cb = 0; cb < rpad; cb += 64) {
      const int ncols = min(64, rpad - cb);
      float acc[8][4];
      if (ncols <= 16)
        shrink_warp_tile<2, kRaw>(Xq, M, K, row0, A_pack, off + cb, ks, kKS, acc);
      else if (ncols <= 32)
        shrink_warp_tile<4, kRaw>(Xq, M, K, row0, A_pack, off + cb, ks, kKS, acc);
      else
        shrink_warp_tile<8, kRaw>(Xq, M, K, row0, A_pack, off + cb, ks, kKS, acc);
      if (kKS > 1) {
        // fixed-order sum of the group's K parts through shared memory
#pragma unroll
        for (int nt = 0; nt < 8; ++nt) {
          if (nt * 8 >= ncols) break;
          red[warp][g][nt * 8 + 2 * tig] = acc[nt][0];
          red[warp][g][nt * 8 + 2 * tig + 1] = acc[nt][1];
          red[warp][g + 8][nt * 8 + 2 * tig] = acc[nt][2];
          red[warp][g + 8][nt * 8 + 2 * tig + 1] = acc[nt][3];
        }
        group_sync(rg, kKS);
        if (ks == 0) {
#pragma unroll
          for (int nt = 0; nt < 8; ++nt) {
            if (nt * 8 >= ncols) break;
#pragma unroll
            for (int h = 0; h < 4; ++h) {
              const int rr = g + ((h & 2) ? 8 : 0), cc = nt * 8 + 2 * tig + (h & 1);
              float t = red[rg * kKS][rr][cc];
#pragma unroll
              for (int w = 1; w < kKS; ++w) t += red[rg * kKS + w][rr][cc];
              acc[nt][h] = t;
            }
          }
        }
      }
      if (ks == 0) {
#pragma unroll
        for (int nt = 0; nt < 8; ++nt) {
          if (nt * 8 >= ncols) break;
          const int col = cb + nt * 8 + 2 * tig;  // column within the adapter
#pragma unroll
          for (int half = 0; half < 2; ++half) {
            const int rr = g + 8 * half;
            const int64_t i = row0 + rr;
            if (!((rows_a >> rr) & 1u) || i >= M) continue;
            const float xs = kRaw ? 1.0f : x_scale[i];
            const float v0 = (col < rank) ? xs * acc[nt][2 * half] : 0.f;
            const float v1 = (col + 1 < rank) ? xs * acc[nt][2 * half + 1] : 0.f;
            store_t_pair(T_hi, T_lo, i * R + off + col, v0, v1);
          }
        }
      }
      if (kKS > 1) group_sync(rg, kKS);
    }
    done |= rows_a;
  }
  // the following kernel may start its set-up once every block is here (not
  // earlier, so that it does not hold SMs that later blocks of this one need)
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

// ---------------------------------------------------------------------------
// Tensor-memory form (large M; codes, or raw bf16 input).  The warp-level MMAs above
// run on the legacy tensor path, which on this GPU sustains only a few
// hundred multiply-adds per clock per SM: at the largest workloads the form
// above is bound by it (measured: the same ~1 us per 64-wide K slice per warp
// whatever the loading scheme).  Here one CTA takes 128 tokens and a range of
// K in 128-wide slices:
//  - one producer warp loads the Xq slices (int8, 128-byte rows, 128-byte
//    swizzle) into a ring of shared-memory stages with TMA, two adjacent
//    slices per stage so that each row is read as 256 contiguous bytes
//    (measured: 126 -> 122 us at the down shape); another loads the
//    slice's A_pack rows of every adapter the 128 tokens use (two 64-wide
//    halves, one box per lane) into a ring of its own.  An Xq stage is free
//    again once it is converted, an A_pack stage once the MMAs that read it
//    complete, so the HBM-bound Xq ring does not wait for the MMAs;
//  - eight converter warps (half a row per thread) turn the int8 slice into
//    bf16 (exact: |q| <= 128) in the K-major 128-byte-swizzled layout that
//    tcgen05.mma reads, into one of two slice buffers;
//  - one thread issues tcgen05.mma kind::f16 (M = 128 tokens, K = 16) with
//    fp32 accumulators in tensor memory, one 32-column slot per (adapter, 32
//    columns of it): a single sweep over K serves every adapter of the block
//    (up to kTSlots slots per sweep), and one MMA of N = 32 x slots covers
//    all of them (the slots' A_pack rows are contiguous in the stage).  The
//    eight K steps of a slice accumulate into separate banks (when tensor
//    memory allows), so that the small MMAs do not wait on one another; the
//    banks are added when a slot is read back;
//  - four of the converter warps read the accumulators back (tcgen05.ld);
//    all of them keep the rows that use each slot's adapter and scale by
//    x_scale.
// K is split over the `nsplit` CTAs of a thread-block cluster that share 128
// tokens: each leaves its fp32 sums in its own shared memory, and each CTA
// then adds, for its share of the rows, the sums of all CTAs of the cluster
// in rank order (distributed shared memory), so the result does not depend
// on timing.  Output as in the form above.
// ---------------------------------------------------------------------------
constexpr int kTRows = 128;                     // tokens per CTA (the MMA's M)
constexpr int kTK = 128;                        // K per slice (128 bytes of an Xq row)
constexpr int kTSlotCols = 32;                  // TMEM columns per slot
constexpr int kTSlots = 5;                      // slots per sweep over K
constexpr int kTTmemCols = 256;                 // >= kTSlots * kTSlotCols, a power of 2
constexpr int kTXBytes = kTRows * kTK;          // int8 slice: 16 KB
constexpr int kTSlotBytes = kTSlotCols * kTK * 2;  // A_pack slice of one slot: 8 KB (two 64-wide halves)
constexpr int kTABytes = kTRows * kTK * 2;      // bf16 slice: 32 KB (two 64-wide halves)
constexpr int kTABufs = 2;
constexpr int kTXSub = 2;                       // K slices per Xq stage (256 contiguous bytes of a row)
constexpr int kTMaxXStages = 8;                 // Xq ring
constexpr int kTMaxPStages = 4;                 // A_pack ring
constexpr int kTSmem = 220 * 1024;              // dynamic shared memory (one CTA per SM)
constexpr int kTConvWarps = 8;                  // two per row quarter of the slice
// Xq producer, MMA, converter/epilogue warps, A_pack producer
constexpr int kTThreads = (3 + kTConvWarps) * 32;
constexpr int kTMaxPasses = kTRows * (SQ_MAX_LORA_RANK / kTSlotCols);
constexpr int kTTargetCtas = 148;               // split K until about this many CTAs
constexpr int kTMaxSplit = 8;                   // CTAs of a cluster (portable size)
constexpr int kTMinSlicesPerSplit = 8;
constexpr int kTTab = 1024;                     // segment / adapter tables staged in smem

// two converter threads per token row, and the four epilogue warps cover the
// four 32-lane quarters of tensor memory
static_assert(kTConvWarps * 32 == 2 * kTRows, "converter threads: two per row");
// the accumulator banks: 4 x 2 slots, 2 x 4 slots, 1 x kTSlots slots
static_assert(4 * 2 * kTSlotCols <= kTTmemCols && 2 * 4 * kTSlotCols <= kTTmemCols &&
                  kTSlots * kTSlotCols <= kTTmemCols,
              "accumulator banks exceed the tensor-memory allocation");
// one A_pack box per lane of its producer warp: two halves x two 16-row groups
static_assert(4 * kTSlots <= 32, "A_pack boxes of a stage exceed a warp");
// the widest sweep still fits two bf16 slices, two A_pack stages and one Xq
// stage; the slots' sums (16 KB each) and the staged tables fit as well
static_assert(kTABufs * kTABytes + 2 * kTSlots * kTSlotBytes + kTXSub * kTXBytes <=
                  kTSmem - 1024,
              "shared-memory layout of the widest sweep");
static_assert(kTSlots * kTRows * 128 <= kTSmem - 1024 &&
                  static_cast<int>(sizeof(int32_t)) * (4 * kTTab + 1) <= kTSmem - 1024,
              "sums or tables exceed shared memory");

// K splits for M tokens: about kTTargetCtas CTAs in all, at most a portable
// cluster, and at least kTMinSlicesPerSplit K slices per split.
static inline int tc_shrink_splits(int64_t M) {
  const int64_t nrb = (M + kTRows - 1) / kTRows;
  int64_t n = kTTargetCtas / (nrb > 0 ? nrb : 1);
  return static_cast<int>(n < 1 ? 1 : (n > kTMaxSplit ? kTMaxSplit : n));
}

struct ShrinkPass {
  int16_t row;  // first row of the block with the pass's adapter
  int16_t cb;   // first adapter column of the pass
};

struct ShrinkCtl {
  uint64_t xfull[kTMaxXStages], xempty[kTMaxXStages];  // Xq ring: TMA -> converters
  uint64_t pfull[kTMaxPStages], pempty[kTMaxPStages];  // A_pack ring: TMA -> MMAs
  uint64_t afull[kTABufs], aempty[kTABufs];            // bf16 slices: converters <-> MMAs
  uint64_t done, drain;                            // accumulators ready / MMAs retired
  uint32_t tmem_base;
  int abort, npass;
  int ad[kTRows], off[kTRows], rank[kTRows], groups[kTRows];
  ShrinkPass pass[kTMaxPasses];
};

// 8 consecutive T values of a row -> the 16-byte words of both planes.
__device__ __forceinline__ void store_t8(uint16_t *T_hi, uint16_t *T_lo, int64_t idx,
                                         const float (&v)[8]) {
  uint32_t hi[4], lo[4];
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    const __nv_bfloat16 h0 = __float2bfloat16_rn(v[2 * j]), h1 = __float2bfloat16_rn(v[2 * j + 1]);
    const __nv_bfloat16 l0 = __float2bfloat16_rn(v[2 * j] - __bfloat162float(h0));
    const __nv_bfloat16 l1 = __float2bfloat16_rn(v[2 * j + 1] - __bfloat162float(h1));
    hi[j] = static_cast<uint32_t>(__bfloat16_as_ushort(h0)) |
            (static_cast<uint32_t>(__bfloat16_as_ushort(h1)) << 16);
    lo[j] = static_cast<uint32_t>(__bfloat16_as_ushort(l0)) |
            (static_cast<uint32_t>(__bfloat16_as_ushort(l1)) << 16);
  }
  *reinterpret_cast<uint4 *>(T_hi + idx) = make_uint4(hi[0], hi[1], hi[2], hi[3]);
  *reinterpret_cast<uint4 *>(T_lo + idx) = make_uint4(lo[0], lo[1], lo[2], lo[3]);
}


// Rows of the 128-token block handled by cluster rank q in the reduction.
__device__ __forceinline__ void share_rows(int q, int ns, int &lo, int &hi) {
  lo = q * kTRows / ns;
  hi = (q + 1) * kTRows / ns;
}

// kRaw: T = X·A'ᵀ from the bf16 activations themselves (x_scale unused): each
// X slice is already the MMA's bf16 operand, so there is no conversion; an X
// stage is one slice (two 64-wide halves of 128 rows, 256 bytes of a row) and
// is released by the MMAs that read it.
template <bool kRaw>
__global__ void __launch_bounds__(kTThreads, 1) lora_shrink_tc_kernel(
    const __grid_constant__ CUtensorMap tm_xq, const __grid_constant__ CUtensorMap tm_a,
    const float *__restrict__ x_scale, int64_t M, int64_t K,
    const int32_t *__restrict__ lora_offset, const int32_t *__restrict__ lora_rank,
    int n_adapters, int64_t R, const int32_t *__restrict__ seg_offsets,
    const int32_t *__restrict__ seg_adapter, int64_t S, int nsplit, uint16_t *__restrict__ T_hi,
    uint16_t *__restrict__ T_lo, unsigned long long *__restrict__ mask, uint64_t timeout_ns) {
  extern __shared__ uint8_t sh_raw[];
  uint8_t *base = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(sh_raw) + 1023) &
                                              ~static_cast<uintptr_t>(1023));
  __shared__ ShrinkCtl ctl;
  volatile int *abort_flag = &ctl.abort;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int rb = blockIdx.x / nsplit, sp = blockIdx.x - rb * nsplit;  // sp: rank in the cluster
  const int64_t row0 = static_cast<int64_t>(rb) * kTRows;
  const int nslices = static_cast<int>((K + kTK - 1) / kTK);
  const int c0 = static_cast<int>(static_cast<int64_t>(sp) * nslices / nsplit);
  const int c1 = static_cast<int>(static_cast<int64_t>(sp + 1) * nslices / nsplit);

  // ---- segment and adapter tables into shared memory (the stage area is
  //      not in use yet), then each row's adapter, column offset and rank
  int32_t *t_seg = reinterpret_cast<int32_t *>(base);  // S + 1 offsets
  int32_t *t_sad = t_seg + kTTab + 1;                  // S adapters
  int32_t *t_off = t_sad + kTTab;                      // lora_offset
  int32_t *t_rnk = t_off + kTTab;                      // lora_rank
  const bool seg_tab = S <= kTTab, ad_tab = n_adapters <= kTTab;
  if (seg_tab)
    for (int i = threadIdx.x; i <= static_cast<int>(S); i += kTThreads) {
      t_seg[i] = seg_offsets[i];
      if (i < S) t_sad[i] = seg_adapter[i];
    }
  if (ad_tab)
    for (int i = threadIdx.x; i < n_adapters; i += kTThreads) {
      t_off[i] = lora_offset[i];
      t_rnk[i] = lora_rank[i];
    }
  if (threadIdx.x == 0) {
    for (int i = 0; i < kTMaxXStages; ++i) {
      mbar_init(&ctl.xfull[i], 1);
      // every converter warp has read the slice (raw: the MMAs that read it)
      mbar_init(&ctl.xempty[i], kRaw ? 1 : kTConvWarps);
    }
    for (int i = 0; i < kTMaxPStages; ++i) {
      mbar_init(&ctl.pfull[i], 1);
      mbar_init(&ctl.pempty[i], 1);  // the MMAs that read the rows have completed
    }
    for (int i = 0; i < kTABufs; ++i) {
      mbar_init(&ctl.afull[i], kTConvWarps);
      mbar_init(&ctl.aempty[i], 1);
    }
    mbar_init(&ctl.done, 1);
    mbar_init(&ctl.drain, 1);
    ctl.abort = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(&ctl.tmem_base, kTTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (threadIdx.x < kTRows) {
    const int64_t i = row0 + threadIdx.x;
    int a = (i < M) ? token_adapter(seg_tab ? t_seg : seg_offsets, seg_tab ? t_sad : seg_adapter,
                                    S, n_adapters, i)
                    : -1;
    int off = 0, r = 0;
    if (a >= 0) {
      off = ad_tab ? t_off[a] : lora_offset[a];
      r = ad_tab ? t_rnk[a] : lora_rank[a];
      if (off < 0 || (off & 15) || r <= 0 || r > SQ_MAX_LORA_RANK || off + ((r + 15) & ~15) > R) {
        record_device_error(SQ_ERR_BAD_SEGMENTS);
        a = -1;
        off = 0;
        r = 0;
      }
    }
    ctl.ad[threadIdx.x] = a;
    ctl.off[threadIdx.x] = off;
    ctl.rank[threadIdx.x] = r;
  }
  __syncthreads();
  // passes: one per (adapter, 32 columns of it), adapters in order of first
  // appearance among the rows (the same in every CTA of the cluster)
  if (threadIdx.x < kTRows) {
    const int a = ctl.ad[threadIdx.x];
    bool first = a >= 0;
    for (int j = 0; j < static_cast<int>(threadIdx.x) && first; ++j) first = ctl.ad[j] != a;
    const int rpad = (ctl.rank[threadIdx.x] + 15) & ~15;
    ctl.groups[threadIdx.x] = first ? (rpad + kTSlotCols - 1) / kTSlotCols : 0;
  }
  __syncthreads();
  {
    // pass indices: an exclusive prefix sum of the groups over the rows
    __shared__ int wsum[kTRows / 32];
    const int g = (threadIdx.x < kTRows) ? ctl.groups[threadIdx.x] : 0;
    int incl = g;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int v = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += v;
    }
    if (threadIdx.x < kTRows && lane == 31) wsum[warp] = incl;
    __syncthreads();
    if (threadIdx.x < kTRows) {
      int excl = incl - g;
      for (int w = 0; w < warp; ++w) excl += wsum[w];
      for (int gi = 0; gi < g; ++gi)
        ctl.pass[excl + gi] = ShrinkPass{static_cast<int16_t>(threadIdx.x),
                                         static_cast<int16_t>(gi * kTSlotCols)};
      if (threadIdx.x == kTRows - 1) ctl.npass = excl + g;
    }
  }
  __syncthreads();
  // the tokens' codes and scales (raw: activations) may come from the
  // preceding kernel (programmatic dependent launch: everything above
  // overlapped its tail)
  asm volatile("griddepcontrol.wait;" ::: "memory");
  const int npass = ctl.npass;
  const int nsweep = (npass + kTSlots - 1) / kTSlots;
  const int slots_max = npass < kTSlots ? npass : kTSlots;
  // bf16 slices in flight between the converters and the MMAs, then the
  // A_pack ring (released when the MMAs that read it complete), then the Xq
  // ring (released as soon as a slice is converted, so more of its stages
  // are in flight than in one ring of both)
  constexpr int kXSlices = kRaw ? 1 : kTXSub;        // K slices per X stage
  constexpr int kXStageBytes = kRaw ? kTABytes : kTXSub * kTXBytes;
  const int nab = kRaw ? 0 : kTABufs;
  const int pstage_bytes = slots_max * kTSlotBytes;
  const int pstages = slots_max <= 2 ? 3 : 2;
  int xstages = (kTSmem - 1024 - nab * kTABytes - pstages * pstage_bytes) / kXStageBytes;
  xstages = xstages > kTMaxXStages ? kTMaxXStages : xstages;
  uint8_t *abuf = base;                                 // nab bf16 slices
  uint8_t *pring = base + nab * kTABytes;               // A_pack slots of each stage
  uint8_t *xring = pring + pstages * pstage_bytes;      // int8 (raw: bf16) slices
  // independent accumulator banks: the K steps of a slice go to different
  // banks, so consecutive MMAs do not wait on each other; summed at the end
  const int nbank = (slots_max <= 2) ? 4 : ((slots_max <= 4) ? 2 : 1);
  const uint32_t tmem = ctl.tmem_base;

  if (warp == 0) {
    // ---------------------------------------------------------- Xq producer
    int st = 0;
    uint32_t ph = 0;
    int64_t issued = 0;
    for (int sw = 0; sw < nsweep; ++sw) {
      if (lane == 0) {
        if (sw == 0) prefetch_tmap(&tm_xq);
        for (int c = c0; c < c1; c += kXSlices) {
          if (*abort_flag || !mbar_wait(&ctl.xempty[st], ph ^ 1u, timeout_ns, abort_flag)) {
            *abort_flag = 1;
            record_device_error(SQ_ERR_DEVICE_TIMEOUT);
            break;
          }
          // 16 KB boxes back to back: adjacent 128-byte pieces of each row
          // (int8: whole slices; raw: the two 64-wide halves of one slice)
          const int nbox = kRaw ? 2 : min(kTXSub, c1 - c);
          mbar_arrive_expect_tx(&ctl.xfull[st], static_cast<uint32_t>(nbox * kTXBytes));
          for (int u = 0; u < nbox; ++u)
            tma_load_2d(xring + st * kXStageBytes + u * kTXBytes, &tm_xq, &ctl.xfull[st],
                        kRaw ? c * kTK + 64 * u : (c + u) * kTK, static_cast<int32_t>(row0));
          ++issued;
          if (++st == xstages) { st = 0; ph ^= 1u; }
        }
      }
      __syncwarp();
      // the sweep's sums are exchanged through the stage area, which is
      // refilled only after both cluster barriers
      cluster_sync();
      cluster_sync();
    }
    if (lane == 0) {
      // every copy issued must land before the block exits
      volatile int never = 0;
      for (int s2 = 0; s2 < xstages && s2 < issued; ++s2) {
        const int64_t last = issued - 1 - ((issued - 1 - s2) % xstages);
        mbar_wait(&ctl.xfull[s2], static_cast<uint32_t>((last / xstages) & 1), 1000000000ull,
                  &never);
      }
    }
  } else if (warp == 2 + kTConvWarps) {
    // ------------------------------------------------------ A_pack producer
    int st = 0;
    uint32_t ph = 0;
    int64_t issued = 0;
    for (int sw = 0; sw < nsweep; ++sw) {
      const int p0 = sw * kTSlots, np = min(kTSlots, npass - p0);
      if (sw == 0 && lane == 0) prefetch_tmap(&tm_a);
      // the boxes of a stage, one per lane: (slot q, half h, 16-row group g)
      int ncopy = 0;
      uint32_t bytes = 0;
      for (int q = 0; q < np; ++q) {
        const int i = ctl.pass[p0 + q].row, cb = ctl.pass[p0 + q].cb;
        const int w = min(kTSlotCols, ((ctl.rank[i] + 15) & ~15) - cb);
        ncopy += 2 * (w / 16);
        bytes += static_cast<uint32_t>(w) * kTK * 2;
      }
      int my_q = -1, my_h = 0, my_g = 0;
      if (lane < ncopy) {
        int k = lane;
        for (int q = 0; q < np && my_q < 0; ++q) {
          const int i = ctl.pass[p0 + q].row, cb = ctl.pass[p0 + q].cb;
          const int n2 = 2 * (min(kTSlotCols, ((ctl.rank[i] + 15) & ~15) - cb) / 16);
          if (k < n2) {
            my_q = q;
            my_h = k / (n2 / 2);
            my_g = k % (n2 / 2);
          } else {
            k -= n2;
          }
        }
      }
      for (int c = c0; c < c1; ++c) {
        bool go = false;
        if (lane == 0) {
          go = !*abort_flag && mbar_wait(&ctl.pempty[st], ph ^ 1u, timeout_ns, abort_flag);
          if (!go) {
            *abort_flag = 1;
            record_device_error(SQ_ERR_DEVICE_TIMEOUT);
          } else {
            mbar_arrive_expect_tx(&ctl.pfull[st], bytes);
          }
        }
        if (!__shfl_sync(0xffffffffu, go, 0)) break;
        if (my_q >= 0) {
          const int i = ctl.pass[p0 + my_q].row, cb = ctl.pass[p0 + my_q].cb;
          tma_load_2d(pring + st * pstage_bytes + my_h * (slots_max * kTSlotCols * 128) +
                          my_q * (kTSlotCols * 128) + my_g * 2048,
                      &tm_a, &ctl.pfull[st], c * kTK + 64 * my_h, ctl.off[i] + cb + 16 * my_g);
        }
        ++issued;
        if (++st == pstages) { st = 0; ph ^= 1u; }
      }
      __syncwarp();
      cluster_sync();
      cluster_sync();
    }
    if (lane == 0) {
      volatile int never = 0;
      for (int s2 = 0; s2 < pstages && s2 < issued; ++s2) {
        const int64_t last = issued - 1 - ((issued - 1 - s2) % pstages);
        mbar_wait(&ctl.pfull[s2], static_cast<uint32_t>((last / pstages) & 1), 1000000000ull,
                  &never);
      }
    }
  } else if (warp == 1) {
    // ----------------------------------------------------------------- MMA
    int st = 0, b = 0;
    uint32_t ph = 0, bph = 0;
    for (int sw = 0; sw < nsweep; ++sw) {
      const int p0 = sw * kTSlots, np = min(kTSlots, npass - p0);
      if (lane == 0) {
        tc_fence_after();  // the previous sweep's accumulators have been read
        bool ok = !*abort_flag;
        for (int c = c0; c < c1 && ok; ++c) {
          // the bf16 slice: converted (b counts them) or, raw, the X stage
          // itself (b counts the X ring's stages)
          if (!mbar_wait(kRaw ? &ctl.xfull[b] : &ctl.afull[b], bph, timeout_ns, abort_flag) ||
              !mbar_wait(&ctl.pfull[st], ph, timeout_ns, abort_flag)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t a_addr = smem_u32(kRaw ? xring + b * kXStageBytes : abuf + b * kTABytes);
          const uint32_t s_addr = smem_u32(pring + st * pstage_bytes);
          // one MMA per K step for all slots of the sweep: their A_pack rows
          // are contiguous within each 64-wide half (a slot narrower than 32
          // columns leaves rows that only its own unused columns read)
          const uint32_t idesc = idesc_bf16_f32(kTRows, static_cast<uint32_t>(np * kTSlotCols));
#pragma unroll
          for (int kk = 0; kk < kTK / 16; ++kk) {
            const int h = kk >> 2, k16 = kk & 3;  // 64-wide half, K step inside it
            const int bank = kk % nbank;
            mma_f16(tmem + static_cast<uint32_t>(bank * slots_max * kTSlotCols),
                    sdesc_kmajor_sw128(a_addr + h * (kTRows * 128) + 32 * k16),
                    sdesc_kmajor_sw128(s_addr + h * (slots_max * kTSlotCols * 128) + 32 * k16),
                    idesc, (c > c0 || kk >= nbank) ? 1u : 0u);
          }
          mma_commit(kRaw ? &ctl.xempty[b] : &ctl.aempty[b]);
          mma_commit(&ctl.pempty[st]);
          if (++st == pstages) { st = 0; ph ^= 1u; }
          if (++b == (kRaw ? xstages : nab)) { b = 0; bph ^= 1u; }
        }
        if (ok) {
          mma_commit(&ctl.done);
        } else if (!*abort_flag) {
          *abort_flag = 1;
          record_device_error(SQ_ERR_DEVICE_TIMEOUT);
        }
      }
      __syncwarp();
      cluster_sync();
      cluster_sync();
    }
    if (lane == 0 && nsweep > 0) {
      // every MMA issued must retire before TMEM is freed
      mma_commit(&ctl.drain);
      volatile int never = 0;
      mbar_wait(&ctl.drain, 0, 1000000000ull, &never);
    }
  } else {
    // ------------------------------------------- converters, then epilogue
    const int ctid = threadIdx.x - 64;     // 0..255 among the converter threads
    const int r = ctid & (kTRows - 1);     // row converted by this thread
    const int hq = ctid >> 7;              // its half of the row: int8 chunks 4hq .. 4hq+3
    const int quarter = warp & 3;          // TMEM lanes of this warp
    const int re = quarter * 32 + lane;    // row read back by this thread
    int st = 0, b = 0;
    uint32_t ph = 0, bph = 0;
    int lo_row, hi_row;
    share_rows(sp, nsplit, lo_row, hi_row);
    for (int sw = 0; sw < nsweep; ++sw) {
      const int p0 = sw * kTSlots, np = min(kTSlots, npass - p0);
      bool ok = !*abort_flag;
      for (int c = c0; c < c1 && ok && !kRaw; ++c) {
        const int u = (c - c0) % kTXSub;  // slice of the Xq stage
        ok = (u != 0 ||
              __all_sync(0xffffffffu, mbar_wait(&ctl.xfull[st], ph, timeout_ns, abort_flag))) &&
             __all_sync(0xffffffffu, mbar_wait(&ctl.aempty[b], bph ^ 1u, timeout_ns, abort_flag));
        if (!ok) break;
        // row r: 128 int8 codes (128-byte swizzle: chunk q at q ^ (r & 7));
        // this thread's chunks 4hq .. 4hq+3 are the codes of the slice's
        // 64-wide half hq, written as that half's bf16 row
        const uint8_t *src = xring + (st * kTXSub + u) * kTXBytes + r * 128;
        uint8_t *dst = abuf + b * kTABytes + hq * (kTRows * 128) + r * 128;
        uint4 v[4];
#pragma unroll
        for (int qq = 0; qq < 4; ++qq)
          v[qq] = *reinterpret_cast<const uint4 *>(src + (((4 * hq + qq) ^ (r & 7)) * 16));
#pragma unroll
        for (int qq = 0; qq < 4; ++qq) {
          const uint32_t w4[4] = {v[qq].x, v[qq].y, v[qq].z, v[qq].w};
          // bf16 chunks 2qq (codes 16qq..16qq+7 of the half) and 2qq+1
          const uint4 c_lo = make_uint4(bf16x2_of_s8(w4[0], 0), bf16x2_of_s8(w4[0], 2),
                                        bf16x2_of_s8(w4[1], 0), bf16x2_of_s8(w4[1], 2));
          const uint4 c_hi = make_uint4(bf16x2_of_s8(w4[2], 0), bf16x2_of_s8(w4[2], 2),
                                        bf16x2_of_s8(w4[3], 0), bf16x2_of_s8(w4[3], 2));
          *reinterpret_cast<uint4 *>(dst + (((2 * qq) ^ (r & 7)) * 16)) = c_lo;
          *reinterpret_cast<uint4 *>(dst + (((2 * qq + 1) ^ (r & 7)) * 16)) = c_hi;
        }
        fence_proxy_async_shared();  // the tensor core reads the slice
        __syncwarp();
        const bool stage_done = u == kTXSub - 1 || c == c1 - 1;
        if (lane == 0) {
          mbar_arrive(&ctl.afull[b]);
          if (stage_done) mbar_arrive(&ctl.xempty[st]);
        }
        if (stage_done && ++st == xstages) { st = 0; ph ^= 1u; }
        if (++b == nab) { b = 0; bph ^= 1u; }
      }
      // this CTA's sums -> its shared memory, slot q at base + q * 16 KB,
      // row-major 128-byte rows (16-byte chunk c of row x at c ^ (x & 7))
      if (ok) ok = __all_sync(0xffffffffu, mbar_wait(&ctl.done, static_cast<uint32_t>(sw & 1),
                                                     timeout_ns, abort_flag));
      if (!ok) {
        if (!*abort_flag) {
          *abort_flag = 1;
          record_device_error(SQ_ERR_DEVICE_TIMEOUT);
        }
      } else if (ctid < kTRows) {  // warps 2-5 cover the four lane quarters
        tc_fence_after();
        for (int q = 0; q < np; ++q) {
          uint8_t *prow = base + q * (kTRows * 128) + re * 128;
#pragma unroll
          for (int h = 0; h < 2; ++h) {
            float acc16[16];
            for (int bank = 0; bank < nbank; ++bank) {
              uint32_t v[16];
              tmem_ld_32x32b_x16(tmem + (static_cast<uint32_t>(quarter * 32) << 16) +
                                     static_cast<uint32_t>((bank * slots_max + q) * kTSlotCols + 16 * h),
                                 v);
              tmem_ld_wait();
#pragma unroll
              for (int j = 0; j < 16; ++j)
                acc16[j] = (bank == 0) ? __uint_as_float(v[j]) : acc16[j] + __uint_as_float(v[j]);
            }
#pragma unroll
            for (int c = 0; c < 4; ++c)
              *reinterpret_cast<uint4 *>(prow + (((4 * h + c) ^ (re & 7)) * 16)) =
                  make_uint4(__float_as_uint(acc16[4 * c]), __float_as_uint(acc16[4 * c + 1]),
                             __float_as_uint(acc16[4 * c + 2]), __float_as_uint(acc16[4 * c + 3]));
          }
        }
        tc_fence_before();
      }
      __syncwarp();
      cluster_sync();  // every CTA's sums are in place
      // rows [lo_row, hi_row): sum over the cluster's CTAs in rank order
      const int nrow = hi_row - lo_row;
      for (int e = ctid; e < nrow * np * 4; e += 32 * kTConvWarps) {
        const int q = e / (nrow * 4), rem = e - q * nrow * 4;
        const int x = lo_row + rem / 4, c8 = rem % 4;  // row, 8-column group of the slot
        const int i = ctl.pass[p0 + q].row, cb = ctl.pass[p0 + q].cb;
        const int a = ctl.ad[i], off = ctl.off[i], rank = ctl.rank[i];
        const int w = min(kTSlotCols, ((rank + 15) & ~15) - cb);
        const int64_t row = row0 + x;
        if (8 * c8 >= w || row >= M || ctl.ad[x] != a || *abort_flag) continue;
        const uint32_t local = smem_u32(base + q * (kTRows * 128) + x * 128);
        float s8[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
        for (int p0 = 0; p0 < nsplit; p0 += 4) {  // rank order, four loads pairs in flight
          float4 pv[4][2];
#pragma unroll
          for (int u = 0; u < 4; ++u)
            if (p0 + u < nsplit) {
              const uint32_t ra = map_to_rank(local, static_cast<uint32_t>(p0 + u));
              pv[u][0] = ld_cluster_f4(ra + (((2 * c8) ^ (x & 7)) * 16));
              pv[u][1] = ld_cluster_f4(ra + (((2 * c8 + 1) ^ (x & 7)) * 16));
            }
#pragma unroll
          for (int u = 0; u < 4; ++u)
            if (p0 + u < nsplit) {
              s8[0] += pv[u][0].x; s8[1] += pv[u][0].y; s8[2] += pv[u][0].z; s8[3] += pv[u][0].w;
              s8[4] += pv[u][1].x; s8[5] += pv[u][1].y; s8[6] += pv[u][1].z; s8[7] += pv[u][1].w;
            }
        }
        const float xs = kRaw ? 1.0f : x_scale[row];
#pragma unroll
        for (int j = 0; j < 8; ++j) s8[j] = (cb + 8 * c8 + j < rank) ? xs * s8[j] : 0.f;
        store_t8(T_hi, T_lo, row * R + off + cb + 8 * c8, s8);
      }
      __syncwarp();
      cluster_sync();  // the peers are done reading this CTA's sums
    }
    // zeros outside each row's adapter columns, for this CTA's share of rows
    const int words = static_cast<int>(R / 8);  // 8 columns: 16 bytes of a plane
    for (int e = ctid; e < (hi_row - lo_row) * words; e += 32 * kTConvWarps) {
      const int x = lo_row + e / words, wcol = (e % words) * 8;
      const int64_t row = row0 + x;
      if (row >= M) continue;
      const int a = ctl.ad[x], off = ctl.off[x], rpad = (ctl.rank[x] + 15) & ~15;
      if (a >= 0 && wcol >= off && wcol < off + rpad) continue;
      *reinterpret_cast<uint4 *>(T_hi + row * R + wcol) = make_uint4(0, 0, 0, 0);
      *reinterpret_cast<uint4 *>(T_lo + row * R + wcol) = make_uint4(0, 0, 0, 0);
    }
    if (sp == 0 && ctid < kTRows / 16 && row0 + 16 * ctid < M) {
      // the 16-column groups that each group of 16 tokens uses (one word each)
      unsigned long long bits = 0;
      for (int x = 16 * ctid; x < 16 * ctid + 16; ++x) {
        if (ctl.ad[x] < 0) continue;
        const int off = ctl.off[x], rpad = (ctl.rank[x] + 15) & ~15;
        for (int gi = off / 16; gi < (off + rpad) / 16; ++gi) bits |= 1ull << gi;
      }
      mask[(row0 >> 4) + ctid] = bits;
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, kTTmemCols);
  }
}


// Clusters of `size` CTAs of the tensor-memory form that are resident at
// once on the current device (asked of the runtime once per device and size).
template <bool kRaw>
static cudaError_t tc_clusters_resident(int size, int *out) {
  static std::atomic<int> cache[kMaxDevices][kTMaxSplit + 1];
  const int dev = current_device_index();
  if (dev < 0 || size < 1 || size > kTMaxSplit) return cudaErrorInvalidValue;
  int n = cache[dev][size].load(std::memory_order_relaxed);
  if (n == 0) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(static_cast<unsigned>(size), 1, 1);
    cfg.blockDim = dim3(kTThreads, 1, 1);
    cfg.dynamicSmemBytes = kTSmem;
    cudaLaunchAttribute attr;
    attr.id = cudaLaunchAttributeClusterDimension;
    attr.val.clusterDim.x = static_cast<unsigned>(size);
    attr.val.clusterDim.y = 1;
    attr.val.clusterDim.z = 1;
    cfg.attrs = &attr;
    cfg.numAttrs = 1;
    const cudaError_t e = cudaOccupancyMaxActiveClusters(&n, lora_shrink_tc_kernel<kRaw>, &cfg);
    if (e != cudaSuccess) return e;
    n = n > 0 ? n + 1 : 1;  // stored plus one: 0 means not asked yet
    cache[dev][size].store(n, std::memory_order_relaxed);
  }
  *out = n - 1;
  return cudaSuccess;
}

// Launch of the tensor-memory form: 128-token blocks, K split over a cluster
// of up to eight CTAs so that about one CTA per SM runs, all clusters at once.
// X: Xq (int8) or, kRaw, the bf16 activations (x_scale unused).
template <bool kRaw>
static cudaError_t launch_lora_shrink_tc(const void *X, const float *x_scale, int64_t M,
                                         int64_t K, const uint16_t *A_pack,
                                         const int32_t *lora_offset, const int32_t *lora_rank,
                                         int n_adapters, int64_t R, const int32_t *seg_offsets,
                                         const int32_t *seg_adapter, int64_t S, uint16_t *T_hi,
                                         uint16_t *T_lo, unsigned long long *mask,
                                         cudaStream_t st) {
  const int64_t nrb = (M + kTRows - 1) / kTRows;
  const int nslices = static_cast<int>((K + kTK - 1) / kTK);
  int nsplit = tc_shrink_splits(M);
  const int most = nslices / kTMinSlicesPerSplit;  // keep at least a few slices per split
  if (nsplit > most) nsplit = most > 1 ? most : 1;
  static std::atomic<int> attr_set[kMaxDevices];
  cudaError_t e = ensure_smem_optin(lora_shrink_tc_kernel<kRaw>, kTSmem, attr_set);
  if (e != cudaSuccess) return e;
  // the widest split whose clusters are all resident at once (one CTA per
  // SM: clusters of 3 or more CTAs leave SMs of a GPC unused, so fewer of
  // them fit than SMs / size)
  while (nsplit > 1) {
    int fit = 0;
    e = tc_clusters_resident<kRaw>(nsplit, &fit);
    if (e != cudaSuccess) return e;
    if (fit >= nrb) break;
    --nsplit;
  }
  CUtensorMap tm_xq, tm_a;
  memset(&tm_xq, 0, sizeof tm_xq);
  memset(&tm_a, 0, sizeof tm_a);
  const bool x_ok =
      kRaw ? make_tmap(&tm_xq, X, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, K, M, 64, kTRows,
                       CU_TENSOR_MAP_SWIZZLE_128B)
           : make_tmap(&tm_xq, X, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, K, M, kTK, kTRows,
                       CU_TENSOR_MAP_SWIZZLE_128B);
  if (!x_ok ||
      !make_tmap(&tm_a, A_pack, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, K, R, 64, 16))
    return cudaErrorInvalidValue;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(nrb * nsplit), 1, 1);
  cfg.blockDim = dim3(kTThreads, 1, 1);
  cfg.dynamicSmemBytes = kTSmem;
  cfg.stream = st;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = static_cast<unsigned>(nsplit);
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  return cudaLaunchKernelEx(&cfg, lora_shrink_tc_kernel<kRaw>, tm_xq, tm_a, x_scale, M, K, lora_offset,
                            lora_rank, n_adapters, R, seg_offsets, seg_adapter, S, nsplit, T_hi,
                            T_lo, mask, wait_timeout_ns());
}

template <bool kRaw>
static cudaError_t launch_lora_shrink_t(const void *X, const float *x_scale, int64_t M, int64_t K,
                                        const uint16_t *A_pack, const int32_t *lora_offset,
                                        const int32_t *lora_rank, int n_adapters, int64_t R,
                                        const int32_t *seg_offsets, const int32_t *seg_adapter,
                                        int64_t S, uint16_t *T_hi, uint16_t *T_lo,
                                        unsigned long long *mask, cudaStream_t st) {
  const int64_t row_tiles = (M + 15) / 16;
  // widest row grouping that still leaves about two blocks per SM.  A grid
  // of one wave is launched as a programmatic dependent of the preceding
  // kernel (its blocks wait at the start for that kernel's results, so the
  // launch gap overlaps the quantizer's tail); larger grids in plain stream
  // order: as dependents their blocks were placed worse on the large
  // workloads (measured).  The fused GEMM that follows is launched as the
  // shrink's dependent.
  const unsigned g1 = static_cast<unsigned>(row_tiles);
  cudaLaunchConfig_t cfg = {};
  cfg.blockDim = dim3(kShrinkThreads, 1, 1);
  cfg.dynamicSmemBytes = 0;
  cfg.stream = st;
  cfg.attrs = nullptr;
  cfg.numAttrs = 0;
  if (row_tiles >= 8 * 2 * 148) {
    cfg.gridDim = dim3((g1 + 7) / 8, 1, 1);
    return cudaLaunchKernelEx(&cfg, lora_shrink_kernel<8, kRaw>, X, x_scale, M, K, A_pack,
                              lora_offset, lora_rank, n_adapters, R, seg_offsets, seg_adapter, S,
                              T_hi, T_lo, mask);
  }
  if (row_tiles >= 4 * 2 * 148) {
    cfg.gridDim = dim3((g1 + 3) / 4, 1, 1);
    return cudaLaunchKernelEx(&cfg, lora_shrink_kernel<4, kRaw>, X, x_scale, M, K, A_pack,
                              lora_offset, lora_rank, n_adapters, R, seg_offsets, seg_adapter, S,
                              T_hi, T_lo, mask);
  }
  if (row_tiles >= 2 * 2 * 148) {
    cfg.gridDim = dim3((g1 + 1) / 2, 1, 1);
    return cudaLaunchKernelEx(&cfg, lora_shrink_kernel<2, kRaw>, X, x_scale, M, K, A_pack,
                              lora_offset, lora_rank, n_adapters, R, seg_offsets, seg_adapter, S,
                              T_hi, T_lo, mask);
  }
  cfg.gridDim = dim3(g1, 1, 1);
  cudaLaunchAttribute attr[1];
  if (g1 <= static_cast<unsigned>(sm_count_of_current_device())) {
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
  }
  return cudaLaunchKernelEx(&cfg, lora_shrink_kernel<1, kRaw>, X, x_scale, M, K, A_pack,
                            lora_offset, lora_rank, n_adapters, R, seg_offsets, seg_adapter, S,
                            T_hi, T_lo, mask);
}

cudaError_t launch_lora_shrink(const int8_t *Xq, const float *x_scale, int64_t M, int64_t K,
                               const uint16_t *A_pack, const int32_t *lora_offset,
                               const int32_t *lora_rank, int n_adapters, int64_t R,
                               const int32_t *seg_offsets, const int32_t *seg_adapter, int64_t S,
                               uint16_t *T_hi, uint16_t *T_lo, unsigned long long *mask,
                               cudaStream_t st) {
  if (M == 0) return cudaSuccess;
  // the tensor-memory form once there are 128-token blocks for a fifth of the
  // SMs (measured: at 2048 tokens the form above is faster, from 4096 on
  // this one; K split over clusters fills the remaining SMs)
  const int nsm = sm_count_of_current_device();
  if (nsm > 0 && M >= static_cast<int64_t>(kTRows) * (nsm / 5))
    return launch_lora_shrink_tc<false>(Xq, x_scale, M, K, A_pack, lora_offset, lora_rank,
                                        n_adapters, R, seg_offsets, seg_adapter, S, T_hi, T_lo,
                                        mask, st);
  return launch_lora_shrink_t<false>(Xq, x_scale, M, K, A_pack, lora_offset, lora_rank,
                                     n_adapters, R, seg_offsets, seg_adapter, S, T_hi, T_lo, mask,
                                     st);
}

cudaError_t launch_lora_shrink_raw(const uint16_t *X, int64_t M, int64_t K,
                                   const uint16_t *A_pack, const int32_t *lora_offset,
                                   const int32_t *lora_rank, int n_adapters, int64_t R,
                                   const int32_t *seg_offsets, const int32_t *seg_adapter,
                                   int64_t S, uint16_t *T_hi, uint16_t *T_lo,
                                   unsigned long long *mask, cudaStream_t st) {
  if (M == 0) return cudaSuccess;
  // the tensor-memory form from the same number of tokens as above
  const int nsm = sm_count_of_current_device();
  if (nsm > 0 && M >= static_cast<int64_t>(kTRows) * (nsm / 5))
    return launch_lora_shrink_tc<true>(X, nullptr, M, K, A_pack, lora_offset, lora_rank,
                                       n_adapters, R, seg_offsets, seg_adapter, S, T_hi, T_lo,
                                       mask, st);
  return launch_lora_shrink_t<true>(X, nullptr, M, K, A_pack, lora_offset, lora_rank, n_adapters,
                                    R, seg_offsets, seg_adapter, S, T_hi, T_lo, mask, st);
}

}  // namespace sq
