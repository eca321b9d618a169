// Shared definitions of the CUDA library (not part of the public ABI).
#pragma once

#include <atomic>
#include <cstdint>
#include <cuda_runtime.h>

#include "../../include/sq_w8a8.h"

namespace sq {

// Device-side error record: the first sq_status code a kernel hits.  The
// library is built as one translation unit (sq_lib.cu), so this is one object.
__device__ unsigned int g_device_error = 0;

__device__ __forceinline__ void record_device_error(unsigned int code) {
  atomicCAS(&g_device_error, 0u, code);
}

// Default bound of every device-side spin-wait (ns), settable from the host.
uint64_t wait_timeout_ns();

// Launch facts are kept per device: a process may drive several GPUs, and
// kernel attributes and occupancies belong to a device.  The caches are
// atomics, so host threads may launch concurrently (two threads that find a
// slot empty both compute the same value).  They hold for the life of the
// process: after cudaDeviceReset of a device the library must not be used on
// that device again.
constexpr int kMaxDevices = 64;

// The current device, or -1 when it cannot be queried or is beyond the caches.
static inline int current_device_index() {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return -1;
  return dev;
}

// Number of SMs of the current device (cached per device).
static inline int sm_count_of_current_device() {
  static std::atomic<int> cached[kMaxDevices];
  const int dev = current_device_index();
  if (dev < 0) return 148;
  int n = cached[dev].load(std::memory_order_relaxed);
  if (n == 0) {
    cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
    n = n > 0 ? n : 148;
    cached[dev].store(n, std::memory_order_relaxed);
  }
  return n;
}

// Sets the dynamic shared-memory opt-in of `kern` to `bytes` once per device;
// `done` holds one flag per device (one array per kernel).
template <class Kern>
static inline cudaError_t ensure_smem_optin(Kern kern, int bytes,
                                            std::atomic<int> (&done)[kMaxDevices]) {
  const int dev = current_device_index();
  if (dev < 0) return cudaErrorInvalidDevice;
  if (done[dev].load(std::memory_order_acquire)) return cudaSuccess;
  const cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
  if (e == cudaSuccess) done[dev].store(1, std::memory_order_release);
  return e;
}

// Resident blocks per SM of `kern` with `threads` threads and `smem` bytes of
// dynamic shared memory on the current device, cached per device in
// cache[dev][slot] (the caller's slot stands for its shared-memory size).
template <class Kern, int kSlots>
static inline cudaError_t blocks_per_sm(Kern kern, int threads, size_t smem, int slot,
                                        std::atomic<int> (&cache)[kMaxDevices][kSlots], int *out) {
  const int dev = current_device_index();
  if (dev < 0 || slot < 0 || slot >= kSlots) return cudaErrorInvalidValue;
  int bps = cache[dev][slot].load(std::memory_order_relaxed);
  if (bps == 0) {
    const cudaError_t e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&bps, kern, threads, smem);
    if (e != cudaSuccess) return e;
    bps = bps > 0 ? bps : 1;
    cache[dev][slot].store(bps, std::memory_order_relaxed);
  }
  *out = bps;
  return cudaSuccess;
}

// LoRA operands of the fused GEMM: T planes [M,R] bf16 (written by the
// shrink kernel), the packed B [N,R] bf16 and one mask of used 16-column
// groups per 16 tokens.
struct LoraOperands {
  const uint16_t *T_hi, *T_lo, *B_pack;
  const unsigned long long *mask;
  int64_t R;
};

// launchers (one per kernel family); they only enqueue work on `st`
cudaError_t launch_act_absmax_update(const void *X, int dtype, int64_t M, int64_t K, float *out,
                                     cudaStream_t st);
cudaError_t launch_weight_absmax(const uint16_t *W, int64_t N, int64_t K, float *out,
                                 cudaStream_t st);
cudaError_t launch_compute_smoothing(const float *a, const float *w, int64_t K, float alpha,
                                     float *s, cudaStream_t st);
cudaError_t launch_quant_act(const void *X, int dtype, const float *s, int64_t M, int64_t K,
                             int8_t *Xq, float *x_scale, cudaStream_t st);
cudaError_t launch_static_act_scale(const float *a, const float *s, int64_t K, float *scale,
                                    cudaStream_t st);
cudaError_t launch_quant_act_static(const void *X, int dtype, const float *s, const float *scale,
                                    int64_t M, int64_t K, int8_t *Xq, float *x_scale,
                                    unsigned long long *clip_count, cudaStream_t st);
cudaError_t launch_fold_norm_weight(const float *gamma, const float *s, int64_t K, float *gamma_s,
                                    cudaStream_t st);
bool rmsnorm_quant_supported(int64_t K);
cudaError_t launch_rmsnorm_quant(const uint16_t *H, const float *gamma_s, float eps, int64_t M,
                                 int64_t K, int8_t *Xq, float *x_scale, cudaStream_t st);
cudaError_t launch_quantize_weight(const uint16_t *W, const float *s, int64_t N, int64_t K,
                                   int8_t *Wq, float *w_scale, cudaStream_t st);
cudaError_t launch_prepare_lora(const uint16_t *A, const uint16_t *B, const float *s, int64_t r,
                                int64_t K, int64_t N, float scale, int64_t R, int64_t off,
                                uint16_t *A_pack, uint16_t *B_pack, cudaStream_t st);
cudaError_t launch_write_lora_table(const int32_t *offs, const int32_t *ranks, int n,
                                    int32_t *off_dev, int32_t *rank_dev, cudaStream_t st);
cudaError_t launch_lora_shrink(const int8_t *Xq, const float *x_scale, int64_t M, int64_t K,
                               const uint16_t *A_pack, const int32_t *lora_offset,
                               const int32_t *lora_rank, int n_adapters, int64_t R,
                               const int32_t *seg_offsets, const int32_t *seg_adapter, int64_t S,
                               uint16_t *T_hi, uint16_t *T_lo, unsigned long long *mask,
                               cudaStream_t st);
cudaError_t launch_lora_shrink_raw(const uint16_t *X, int64_t M, int64_t K,
                                   const uint16_t *A_pack, const int32_t *lora_offset,
                                   const int32_t *lora_rank, int n_adapters, int64_t R,
                                   const int32_t *seg_offsets, const int32_t *seg_adapter,
                                   int64_t S, uint16_t *T_hi, uint16_t *T_lo,
                                   unsigned long long *mask, cudaStream_t st);
size_t decode_workspace_bytes(int64_t M);
bool decode_applicable(int64_t M);
cudaError_t launch_decode(const int8_t *Xq, const float *x_scale, const int8_t *Wq,
                          const float *w_scale, int64_t M, int64_t N, int64_t K, int mode,
                          const uint16_t *A_pack, const uint16_t *B_pack,
                          const int32_t *lora_offset, const int32_t *lora_rank, int n_adapters,
                          int64_t R, const int32_t *seg_offsets, const int32_t *seg_adapter,
                          int64_t S, float *part, void *out, cudaStream_t st);
cudaError_t launch_w8a8_gemm(const int8_t *Xq, const int8_t *Wq, const float *x_scale,
                             const float *w_scale, int64_t M, int64_t N, int64_t K, int mode,
                             void *out, const LoraOperands *lora, cudaStream_t st);

size_t alpha_error_workspace_bytes(int64_t M, int64_t N, int64_t K);
constexpr int kAlphaSweepMax = SQ_ALPHA_SWEEP_MAX;
cudaError_t launch_alpha_sweep(const void *X, int dtype, const uint16_t *W, int64_t M, int64_t N,
                               int64_t K, const float *alphas, int n, double *err, double *rel,
                               float *best, void *workspace, cudaStream_t st);
cudaError_t launch_alpha_error(const void *X, int dtype, const uint16_t *W, int64_t M, int64_t N,
                               int64_t K, float alpha, double *err, void *workspace,
                               cudaStream_t st);

// Adapter of token `i` for a segment table: the first segment s with
// off[s] <= i < off[s+1].  Segments are assumed sorted (off non-decreasing);
// the binary search finds the last segment starting at or before i and then
// checks that it covers i.  Returns -1 when no segment covers the token; an
// adapter index outside [-1, n_adapters) is reported and treated as -1.
__device__ __forceinline__ int token_adapter(const int32_t *__restrict__ seg_offsets,
                                             const int32_t *__restrict__ seg_adapter,
                                             int64_t S, int n_adapters, int64_t i) {
  if (S <= 0) return -1;
  int64_t lo = 0, hi = S - 1, s = -1;
  while (lo <= hi) {
    int64_t mid = (lo + hi) >> 1;
    if (seg_offsets[mid] <= i) {
      s = mid;
      lo = mid + 1;
    } else {
      hi = mid - 1;
    }
  }
  // several empty segments may start at the same offset: step back to the
  // first segment whose range is non-empty and holds i
  while (s >= 0 && !(seg_offsets[s] <= i && i < seg_offsets[s + 1])) {
    if (seg_offsets[s] < i) return -1;
    --s;
  }
  if (s < 0) return -1;
  int a = seg_adapter[s];
  if (a < -1 || a >= n_adapters) {
    record_device_error(SQ_ERR_BAD_SEGMENTS);
    return -1;
  }
  return a;
}

}  // namespace sq
