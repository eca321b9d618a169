// Layer-wise output error of the W8A8 layer for one migration strength alpha
// ("SmoothQuant" explainer, "Reading the diagnostics": compare layer-wise
// output error across alpha values; "Variants and related ideas": per-layer
// alpha chosen by calibration error).  On the calibration tokens X:
//   a = max_i |X[i,:]|, w = max_n |W[n,:]|, s = smoothing(a, w, alpha),
//   Wq, w_scale = weight quantization; Xq, x_scale = activation quantization;
//   Y = bf16(f32(acc) * x_scale * w_scale) (the fused GEMM, no adapters);
//   err[0] = sum (Y - X W^T)^2,  err[1] = sum (X W^T)^2
// with X W^T from the unquantized operands, fp32 products and sums, and the
// two sums in fp64.  An offline diagnostic, not on the hot path.
#include <cuda_bf16.h>

#include "common.cuh"

namespace sq {

constexpr int kRefTile = 64;
constexpr int kRefK = 32;

template <typename T>
__device__ __forceinline__ float ref_value(const T *p, int64_t idx) {
  if constexpr (sizeof(T) == 2)
    return __uint_as_float(static_cast<uint32_t>(p[idx]) << 16);
  else
    return p[idx];
}

// 64x64 outputs per block, 4x4 per thread, fp32 FMAs on CUDA cores.
template <typename T>
__global__ void __launch_bounds__(256) ref_error_kernel(const T *__restrict__ X,
                                                        const uint16_t *__restrict__ W,
                                                        const uint16_t *__restrict__ Y, int64_t M,
                                                        int64_t N, int64_t K,
                                                        double *__restrict__ err) {
  __shared__ float xs[kRefK][kRefTile + 4];
  __shared__ float ws[kRefK][kRefTile + 4];
  __shared__ double part[2][8];
  const int tid = threadIdx.x, tx = tid & 15, ty = tid >> 4;
  const int64_t m0 = static_cast<int64_t>(blockIdx.y) * kRefTile;
  const int64_t n0 = static_cast<int64_t>(blockIdx.x) * kRefTile;
  float acc[4][4];
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int j = 0; j < 4; ++j) acc[i][j] = 0.f;
  for (int64_t k0 = 0; k0 < K; k0 += kRefK) {
    // 64 rows x 32 K of each operand: element e = tid + 256 * t, row e / 32, k e % 32
#pragma unroll
    for (int t = 0; t < 8; ++t) {
      const int e = tid + 256 * t, r = e >> 5, kk = e & 31;
      const int64_t k = k0 + kk;
      xs[kk][r] = (m0 + r < M && k < K) ? ref_value(X, (m0 + r) * K + k) : 0.f;
      ws[kk][r] = (n0 + r < N && k < K) ? ref_value(W, (n0 + r) * K + k) : 0.f;
    }
    __syncthreads();
#pragma unroll 8
    for (int kk = 0; kk < kRefK; ++kk) {
      float a[4], b[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) a[i] = xs[kk][ty * 4 + i];
#pragma unroll
      for (int j = 0; j < 4; ++j) b[j] = ws[kk][tx * 4 + j];
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(a[i], b[j], acc[i][j]);
    }
    __syncthreads();
  }
  double e = 0.0, r = 0.0;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int64_t m = m0 + ty * 4 + i;
    if (m >= M) continue;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int64_t n = n0 + tx * 4 + j;
      if (n >= N) continue;
      const double ref = acc[i][j];
      const double y = __uint_as_float(static_cast<uint32_t>(Y[m * N + n]) << 16);
      e += (y - ref) * (y - ref);
      r += ref * ref;
    }
  }
  for (int o = 16; o > 0; o >>= 1) {
    e += __shfl_xor_sync(0xffffffffu, e, o);
    r += __shfl_xor_sync(0xffffffffu, r, o);
  }
  if ((tid & 31) == 0) {
    part[0][tid >> 5] = e;
    part[1][tid >> 5] = r;
  }
  __syncthreads();
  if (tid == 0) {
    double te = 0.0, tr = 0.0;
    for (int w = 0; w < 8; ++w) {
      te += part[0][w];
      tr += part[1][w];
    }
    atomicAdd(err, te);
    atomicAdd(err + 1, tr);
  }
}

static size_t align256_ae(size_t x) { return (x + 255) & ~static_cast<size_t>(255); }

size_t alpha_error_workspace_bytes(int64_t M, int64_t N, int64_t K) {
  if (M <= 0 || N <= 0 || K <= 0) return 0;
  return 3 * align256_ae(4 * static_cast<size_t>(K)) + align256_ae(4 * static_cast<size_t>(N)) +
         align256_ae(4 * static_cast<size_t>(M)) + align256_ae(static_cast<size_t>(N) * K) +
         align256_ae(static_cast<size_t>(M) * K) + align256_ae(2 * static_cast<size_t>(M) * N);
}

cudaError_t launch_alpha_error(const void *X, int dtype, const uint16_t *W, int64_t M, int64_t N,
                               int64_t K, float alpha, double *err, void *workspace,
                               cudaStream_t st) {
  uint8_t *p = static_cast<uint8_t *>(workspace);
  auto take = [&](size_t bytes) {
    uint8_t *q = p;
    p += align256_ae(bytes);
    return q;
  };
  float *a = reinterpret_cast<float *>(take(4 * K));
  float *w = reinterpret_cast<float *>(take(4 * K));
  float *s = reinterpret_cast<float *>(take(4 * K));
  float *w_scale = reinterpret_cast<float *>(take(4 * N));
  float *x_scale = reinterpret_cast<float *>(take(4 * M));
  int8_t *Wq = reinterpret_cast<int8_t *>(take(static_cast<size_t>(N) * K));
  int8_t *Xq = reinterpret_cast<int8_t *>(take(static_cast<size_t>(M) * K));
  uint16_t *Y = reinterpret_cast<uint16_t *>(take(2 * static_cast<size_t>(M) * N));
  cudaError_t e;
  if ((e = cudaMemsetAsync(a, 0, 4 * K, st)) != cudaSuccess) return e;
  if ((e = launch_act_absmax_update(X, dtype, M, K, a, st)) != cudaSuccess) return e;
  if ((e = launch_weight_absmax(W, N, K, w, st)) != cudaSuccess) return e;
  if ((e = launch_compute_smoothing(a, w, K, alpha, s, st)) != cudaSuccess) return e;
  if ((e = launch_quantize_weight(W, s, N, K, Wq, w_scale, st)) != cudaSuccess) return e;
  if ((e = launch_quant_act(X, dtype, s, M, K, Xq, x_scale, st)) != cudaSuccess) return e;
  if ((e = launch_w8a8_gemm(Xq, Wq, x_scale, w_scale, M, N, K, 0, Y, nullptr, st)) != cudaSuccess)
    return e;
  if ((e = cudaMemsetAsync(err, 0, 2 * sizeof(double), st)) != cudaSuccess) return e;
  const dim3 grid(static_cast<unsigned>((N + kRefTile - 1) / kRefTile),
                  static_cast<unsigned>((M + kRefTile - 1) / kRefTile), 1);
  if (dtype == SQ_DTYPE_BF16)
    ref_error_kernel<uint16_t><<<grid, 256, 0, st>>>(static_cast<const uint16_t *>(X), W, Y, M,
                                                     N, K, err);
  else
    ref_error_kernel<float><<<grid, 256, 0, st>>>(static_cast<const float *>(X), W, Y, M, N, K,
                                                  err);
  return cudaGetLastError();
}

// The choice of alpha from the sweep's sums: rel[t] = err[t][0] / err[t][1]
// (IEEE fp64 division; 0 when the reference energy is 0) and *best = the
// alpha of the smallest rel, the first one on ties.  One thread: at most
// kAlphaSweepMax values.
struct AlphaList {
  float a[kAlphaSweepMax];
  int n;
};

__global__ void alpha_pick_kernel(const double *__restrict__ err, AlphaList al,
                                  double *__restrict__ rel, float *__restrict__ best) {
  if (threadIdx.x != 0 || blockIdx.x != 0) return;
  int bi = 0;
  double bv = 0.0;
  for (int t = 0; t < al.n; ++t) {
    const double den = err[2 * t + 1];
    const double r = den > 0.0 ? __ddiv_rn(err[2 * t], den) : 0.0;
    rel[t] = r;
    if (t == 0 || r < bv) {
      bv = r;
      bi = t;
    }
  }
  *best = al.a[bi];
}

cudaError_t launch_alpha_sweep(const void *X, int dtype, const uint16_t *W, int64_t M, int64_t N,
                               int64_t K, const float *alphas, int n, double *err, double *rel,
                               float *best, void *workspace, cudaStream_t st) {
  AlphaList al;
  al.n = n;
  for (int t = 0; t < n; ++t) {
    al.a[t] = alphas[t];
    const cudaError_t e = launch_alpha_error(X, dtype, W, M, N, K, alphas[t], err + 2 * t, workspace, st);
    if (e != cudaSuccess) return e;
  }
  alpha_pick_kernel<<<1, 32, 0, st>>>(err, al, rel, best);
  return cudaGetLastError();
}

}  // namespace sq
