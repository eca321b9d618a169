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
  return launch_lora_shrink_t<true>(X, nullptr, M, K, A_pack, lora_offset, lora_rank, n_adapters,
                                    R, seg_offsets, seg_adapter, S, T_hi, T_lo, mask, st);
}

}  // namespace sq
