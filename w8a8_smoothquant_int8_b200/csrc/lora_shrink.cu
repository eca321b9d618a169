// LoRA shrink: the low-rank projection of the dequantized activations,
//   T[i, j] = x_scale_i * sum_k Xq[i,k] * A_pack[off_a + j, k]   (j < r_a)
// for the adapter a of token i ("[Feature]: LoRA support for W8A8
// SmoothQuant", Pitch: the LoRA path runs after the INT8 GEMM in BF16; A_pack
// carries the smoothing scale so Xq*x_scale*diag(s) ~ X).
//
// T is written as two bf16 planes over the packed width R, T_hi = bf16(T) and
// T_lo = bf16(T - T_hi), with zeros outside the token's adapter columns, so
// that the GEMM epilogue can apply every adapter of a 128-token tile with
// dense bf16 tensor-core MMAs and still carry ~16 significant bits of T.
// mask[tile] collects, per 128-token tile, the 16-column groups of R that
// some token of the tile uses.
#include <cuda_bf16.h>

#include "common.cuh"

namespace sq {

constexpr int kShrinkThreads = 128;

__global__ void __launch_bounds__(kShrinkThreads) lora_shrink_kernel(
    const int8_t *__restrict__ Xq, const float *__restrict__ x_scale, int64_t K,
    const uint16_t *__restrict__ A_pack, const int32_t *__restrict__ lora_offset,
    const int32_t *__restrict__ lora_rank, int n_adapters, int64_t R,
    const int32_t *__restrict__ seg_offsets, const int32_t *__restrict__ seg_adapter, int64_t S,
    uint16_t *__restrict__ T_hi, uint16_t *__restrict__ T_lo,
    unsigned long long *__restrict__ mask) {
  __shared__ float tv[SQ_MAX_LORA_COLS];
  __shared__ float part[kShrinkThreads / 32][16];
  __shared__ int s_off, s_rank;
  const int64_t i = blockIdx.x;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  if (tid == 0) {
    int a = token_adapter(seg_offsets, seg_adapter, S, n_adapters, i);
    int off = -1, r = 0;
    if (a >= 0) {
      off = lora_offset[a];
      r = lora_rank[a];
      const int rpad = (r + 15) & ~15;
      if (off < 0 || (off & 15) || r <= 0 || off + rpad > R) {
        record_device_error(SQ_ERR_BAD_SEGMENTS);
        off = -1;
        r = 0;
      } else {
        unsigned long long bits = 0;
        for (int g = off / 16; g < (off + rpad) / 16; ++g) bits |= 1ull << g;
        atomicOr(mask + (i >> 7), bits);
      }
    }
    s_off = off;
    s_rank = r;
  }
  __syncthreads();
  const int off = s_off, r = s_rank;
  const float xs = x_scale[i];
  const int8_t *xrow = Xq + i * K;
  for (int g0 = 0; g0 < r; g0 += 16) {
    float acc[16];
#pragma unroll
    for (int j = 0; j < 16; ++j) acc[j] = 0.f;
    const int jn = min(16, r - g0);
    for (int64_t k0 = static_cast<int64_t>(tid) * 16; k0 < K; k0 += kShrinkThreads * 16) {
      uint4 xr = *reinterpret_cast<const uint4 *>(xrow + k0);
      float xv[16];
      const uint32_t w4[4] = {xr.x, xr.y, xr.z, xr.w};
#pragma unroll
      for (int t = 0; t < 16; ++t)
        xv[t] = static_cast<float>(static_cast<int8_t>((w4[t >> 2] >> (8 * (t & 3))) & 0xff));
      for (int j = 0; j < jn; ++j) {
        const uint16_t *arow = A_pack + static_cast<int64_t>(off + g0 + j) * K + k0;
        uint4 a0 = *reinterpret_cast<const uint4 *>(arow);
        uint4 a1 = *reinterpret_cast<const uint4 *>(arow + 8);
        const uint32_t av[8] = {a0.x, a0.y, a0.z, a0.w, a1.x, a1.y, a1.z, a1.w};
        float s = 0.f;
#pragma unroll
        for (int t = 0; t < 8; ++t) {
          s = fmaf(xv[2 * t], __uint_as_float(av[t] << 16), s);
          s = fmaf(xv[2 * t + 1], __uint_as_float(av[t] & 0xffff0000u), s);
        }
        acc[j] += s;
      }
    }
#pragma unroll
    for (int j = 0; j < 16; ++j) {
      float v = acc[j];
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
      if (lane == 0) part[warp][j] = v;
    }
    __syncthreads();
    if (tid < 16) {
      float v = 0.f;
#pragma unroll
      for (int w = 0; w < kShrinkThreads / 32; ++w) v += part[w][tid];
      tv[g0 + tid] = (g0 + tid < r) ? xs * v : 0.f;
    }
    __syncthreads();
  }
  // write the full row of both planes: own columns from tv, zeros elsewhere
  const int rpad = (r + 15) & ~15;
  for (int64_t c0 = static_cast<int64_t>(tid) * 8; c0 < R; c0 += kShrinkThreads * 8) {
    uint32_t hi[4] = {0, 0, 0, 0}, lo[4] = {0, 0, 0, 0};
    if (off >= 0 && c0 >= off && c0 < off + rpad) {
#pragma unroll
      for (int t = 0; t < 8; ++t) {
        float v = tv[c0 - off + t];
        __nv_bfloat16 h = __float2bfloat16_rn(v);
        __nv_bfloat16 l = __float2bfloat16_rn(v - __bfloat162float(h));
        hi[t >> 1] |= static_cast<uint32_t>(__bfloat16_as_ushort(h)) << (16 * (t & 1));
        lo[t >> 1] |= static_cast<uint32_t>(__bfloat16_as_ushort(l)) << (16 * (t & 1));
      }
    }
    *reinterpret_cast<uint4 *>(T_hi + i * R + c0) = make_uint4(hi[0], hi[1], hi[2], hi[3]);
    *reinterpret_cast<uint4 *>(T_lo + i * R + c0) = make_uint4(lo[0], lo[1], lo[2], lo[3]);
  }
}

cudaError_t launch_lora_shrink(const int8_t *Xq, const float *x_scale, int64_t M, int64_t K,
                               const uint16_t *A_pack, const int32_t *lora_offset,
                               const int32_t *lora_rank, int n_adapters, int64_t R,
                               const int32_t *seg_offsets, const int32_t *seg_adapter, int64_t S,
                               uint16_t *T_hi, uint16_t *T_lo, unsigned long long *mask,
                               cudaStream_t st) {
  if (M == 0) return cudaSuccess;
  cudaError_t e = cudaMemsetAsync(mask, 0, static_cast<size_t>((M + 127) / 128) * 8, st);
  if (e != cudaSuccess) return e;
  lora_shrink_kernel<<<static_cast<unsigned>(M), kShrinkThreads, 0, st>>>(
      Xq, x_scale, K, A_pack, lora_offset, lora_rank, n_adapters, R, seg_offsets, seg_adapter, S,
      T_hi, T_lo, mask);
  return cudaGetLastError();
}

}  // namespace sq
