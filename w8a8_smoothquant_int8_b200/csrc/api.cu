// C ABI entry points (include/sq_w8a8.h): argument validation on the host,
// then launches.  Nothing here allocates device memory.
#include <cstdio>
#include <cstring>

#include "common.cuh"
#include "ptx_sm100.cuh"

namespace sq {

static std::atomic<uint64_t> g_wait_timeout_ns{2000000000ull};
static cudaEvent_t g_gemm_ev_before = nullptr, g_gemm_ev_after = nullptr;
uint64_t wait_timeout_ns() { return g_wait_timeout_ns; }

// ---------------------------------------------------------------------------
// validation helpers
// ---------------------------------------------------------------------------
static bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
static bool ptr_ok(const void *p) { return p != nullptr && aligned16(p); }
static bool aligned_to(const void *p, uintptr_t a) {
  return p != nullptr && (reinterpret_cast<uintptr_t>(p) & (a - 1)) == 0;
}

// Result of sq_device_supported per device, cached: querying the device
// properties takes far longer than a launch.
static int check_device() {
  static std::atomic<int> cached[kMaxDevices];  // 0 = unknown, else status + 1
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return SQ_ERR_CUDA;
  if (dev < 0 || dev >= kMaxDevices) return sq_device_supported(dev);
  int c = cached[dev].load(std::memory_order_relaxed);
  if (c == 0) {
    const int st = sq_device_supported(dev);
    if (st == SQ_ERR_CUDA) return st;
    c = st + 1;
    cached[dev].store(c, std::memory_order_relaxed);
  }
  return c - 1;
}

static int check_mk(int64_t M, int64_t K) {
  if (M < 0 || K < 0) return SQ_ERR_INVALID_ARG;
  if (K % 16 != 0 || K > SQ_MAX_K) return SQ_ERR_UNSUPPORTED_SHAPE;
  if (M > 0x7fffffffLL) return SQ_ERR_UNSUPPORTED_SHAPE;
  return SQ_OK;
}

static int cuda_status(cudaError_t e) { return e == cudaSuccess ? SQ_OK : SQ_ERR_CUDA; }

static size_t align256(size_t x) { return (x + 255) & ~static_cast<size_t>(255); }

struct Workspace {
  uint16_t *T_hi, *T_lo;
  unsigned long long *mask;
};

// The large-M form needs the two T planes and one mask word per 16 tokens; the small-M
// (decode) form needs its shrink partials.
static size_t workspace_bytes(int64_t M, int64_t R) {
  if (R <= 0 || M <= 0) return 0;
  if (decode_applicable(M)) return align256(decode_workspace_bytes(M));
  const size_t plane = align256(static_cast<size_t>(M) * static_cast<size_t>(R) * 2);
  return 2 * plane + align256(static_cast<size_t>((M + 15) / 16) * 8);
}

// T planes and mask words alone (the raw-input entry points, any M)
static size_t t_workspace_bytes(int64_t M, int64_t R) {
  if (R <= 0 || M <= 0) return 0;
  const size_t plane = align256(static_cast<size_t>(M) * static_cast<size_t>(R) * 2);
  return 2 * plane + align256(static_cast<size_t>((M + 15) / 16) * 8);
}

static Workspace carve(void *ws, int64_t M, int64_t R) {
  const size_t plane = align256(static_cast<size_t>(M) * static_cast<size_t>(R) * 2);
  uint8_t *p = static_cast<uint8_t *>(ws);
  return Workspace{reinterpret_cast<uint16_t *>(p), reinterpret_cast<uint16_t *>(p + plane),
                   reinterpret_cast<unsigned long long *>(p + 2 * plane)};
}

// checks shared by sq_linear_lora and sq_lora_delta
static int check_lora_args(int64_t M, int64_t K, const uint16_t *A_pack, const uint16_t *B_pack,
                           const int32_t *lora_offset, const int32_t *lora_rank, int n_adapters,
                           int64_t R, const int32_t *seg_offsets, const int32_t *seg_adapter,
                           int64_t S, void *workspace, size_t workspace_size, bool *active) {
  if (n_adapters < 0 || R < 0 || S < 0) return SQ_ERR_INVALID_ARG;
  *active = (R > 0 && n_adapters > 0 && S > 0 && M > 0);
  if (!*active) return SQ_OK;
  if (R % 16 != 0 || R > SQ_MAX_LORA_COLS) return SQ_ERR_UNSUPPORTED_SHAPE;
  if (!ptr_ok(A_pack) || !ptr_ok(B_pack) || !lora_offset || !lora_rank || !seg_offsets ||
      !seg_adapter)
    return SQ_ERR_INVALID_ARG;
  if (!workspace || (reinterpret_cast<uintptr_t>(workspace) & 255u) ||
      workspace_size < workspace_bytes(M, R))
    return SQ_ERR_WORKSPACE;
  (void)K;
  return SQ_OK;
}

}  // namespace sq

namespace sq {
// A wait on an mbarrier that nothing ever arrives on: the bounded wait used
// by every kernel must give up and record SQ_ERR_DEVICE_TIMEOUT.
__global__ void selftest_wait_kernel(uint64_t timeout_ns) {
  __shared__ uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    abort_flag = 0;
    fence_mbar_init();
  }
  __syncthreads();
  if (threadIdx.x == 0 && !mbar_wait(&bar, 0, timeout_ns, &abort_flag))
    record_device_error(SQ_ERR_DEVICE_TIMEOUT);
}
}  // namespace sq

using namespace sq;

// capability of the current device (cached), for the entry points below
static int sq_device_supported_current() { return check_device(); }

extern "C" {

const char *sq_status_string(int status) {
  switch (status) {
    case SQ_OK: return "ok";
    case SQ_ERR_INVALID_ARG: return "invalid argument";
    case SQ_ERR_UNSUPPORTED_SHAPE: return "unsupported shape";
    case SQ_ERR_UNSUPPORTED_DEVICE: return "unsupported device (needs compute capability 10.0)";
    case SQ_ERR_CUDA: return "CUDA runtime error";
    case SQ_ERR_DEVICE_TIMEOUT: return "device-side wait timed out";
    case SQ_ERR_WORKSPACE: return "workspace missing, misaligned or too small";
    case SQ_ERR_BAD_SEGMENTS: return "segment table names an adapter that does not exist";
    default: return "unknown status";
  }
}

int sq_version(void) { return 100; }

int sq_device_supported(int device) {
  int major = 0, minor = 0;
  if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, device) != cudaSuccess ||
      cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, device) != cudaSuccess)
    return SQ_ERR_CUDA;
  return (major == 10 && minor == 0) ? SQ_OK : SQ_ERR_UNSUPPORTED_DEVICE;
}

int sq_get_device_error(int *code, int clear) {
  if (!code) return SQ_ERR_INVALID_ARG;
  if (cudaDeviceSynchronize() != cudaSuccess) return SQ_ERR_CUDA;
  unsigned int v = 0;
  if (cudaMemcpyFromSymbol(&v, g_device_error, sizeof v) != cudaSuccess) return SQ_ERR_CUDA;
  *code = static_cast<int>(v);
  if (clear) {
    unsigned int z = 0;
    if (cudaMemcpyToSymbol(g_device_error, &z, sizeof z) != cudaSuccess) return SQ_ERR_CUDA;
  }
  return SQ_OK;
}

int sq_set_wait_timeout_ns(uint64_t ns) {
  if (ns == 0) return SQ_ERR_INVALID_ARG;
  g_wait_timeout_ns = ns;
  return SQ_OK;
}

int sq_set_gemm_events(void *before, void *after) {
  if ((before == nullptr) != (after == nullptr)) return SQ_ERR_INVALID_ARG;
  g_gemm_ev_before = static_cast<cudaEvent_t>(before);
  g_gemm_ev_after = static_cast<cudaEvent_t>(after);
  return SQ_OK;
}

int sq_selftest_wait_timeout(uint64_t timeout_ns, void *stream) {
  if (timeout_ns == 0 || timeout_ns > 100000000ull) return SQ_ERR_INVALID_ARG;
  int st = check_device();
  if (st) return st;
  selftest_wait_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>(timeout_ns);
  return cuda_status(cudaGetLastError());
}

int sq_act_absmax_update(const void *X, int x_dtype, int64_t M, int64_t K, float *act_absmax,
                         void *stream) {
  int st = check_mk(M, K);
  if (st) return st;
  if (x_dtype != SQ_DTYPE_BF16 && x_dtype != SQ_DTYPE_F32) return SQ_ERR_INVALID_ARG;
  if ((M > 0 && K > 0) && (!ptr_ok(X) || !ptr_ok(act_absmax))) return SQ_ERR_INVALID_ARG;
  if ((st = check_device())) return st;
  return cuda_status(launch_act_absmax_update(X, x_dtype, M, K, act_absmax,
                                              static_cast<cudaStream_t>(stream)));
}

int sq_weight_absmax(const uint16_t *W, int64_t N, int64_t K, float *w_absmax, void *stream) {
  int st = check_mk(N, K);
  if (st) return st;
  if (K > 0 && (!ptr_ok(w_absmax) || (N > 0 && !ptr_ok(W)))) return SQ_ERR_INVALID_ARG;
  if ((st = check_device())) return st;
  if (K == 0) return SQ_OK;
  return cuda_status(launch_weight_absmax(W, N, K, w_absmax, static_cast<cudaStream_t>(stream)));
}

int sq_compute_smoothing(const float *act_absmax, const float *w_absmax, int64_t K, float alpha,
                         float *s, void *stream) {
  if (K < 0) return SQ_ERR_INVALID_ARG;
  if (!(alpha >= 0.f && alpha <= 1.f)) return SQ_ERR_INVALID_ARG;
  if (K > 0 && (!ptr_ok(act_absmax) || !ptr_ok(w_absmax) || !ptr_ok(s))) return SQ_ERR_INVALID_ARG;
  int st = check_device();
  if (st) return st;
  return cuda_status(
      launch_compute_smoothing(act_absmax, w_absmax, K, alpha, s, static_cast<cudaStream_t>(stream)));
}

int sq_quantize_weight(const uint16_t *W, const float *s, int64_t N, int64_t K, int8_t *Wq,
                       float *w_scale, void *stream) {
  int st = check_mk(N, K);
  if (st) return st;
  if (N > 0 && (!ptr_ok(w_scale) || (K > 0 && (!ptr_ok(W) || !ptr_ok(s) || !ptr_ok(Wq)))))
    return SQ_ERR_INVALID_ARG;
  if ((st = check_device())) return st;
  return cuda_status(launch_quantize_weight(W, s, N, K, Wq, w_scale, static_cast<cudaStream_t>(stream)));
}

int sq_prepare_lora(const uint16_t *A, const uint16_t *B, const float *s, int64_t r, int64_t K,
                    int64_t N, float lora_alpha, int64_t R, int64_t off, uint16_t *A_pack,
                    uint16_t *B_pack, void *stream) {
  if (r <= 0 || r > SQ_MAX_LORA_RANK || K < 0 || N < 0 || R <= 0 || off < 0)
    return SQ_ERR_INVALID_ARG;
  if (K % 16 != 0 || K > SQ_MAX_K || R % 16 != 0 || R > SQ_MAX_LORA_COLS || off % 16 != 0)
    return SQ_ERR_UNSUPPORTED_SHAPE;
  const int64_t rpad = (r + 15) / 16 * 16;
  if (off + rpad > R) return SQ_ERR_INVALID_ARG;
  // s == NULL packs A as given (raw-input reading of the LoRA path)
  if (!A || !B || (s && !ptr_ok(s)) || !ptr_ok(A_pack) || !ptr_ok(B_pack))
    return SQ_ERR_INVALID_ARG;
  int st = check_device();
  if (st) return st;
  const float scale = lora_alpha / static_cast<float>(r);  // IEEE fp32 division
  return cuda_status(launch_prepare_lora(A, B, s, r, K, N, scale, R, off, A_pack, B_pack,
                                         static_cast<cudaStream_t>(stream)));
}

int64_t sq_lora_pack_width(const int64_t *ranks, int n_adapters) {
  if (!ranks || n_adapters < 1) return -1;
  int64_t R = 0;
  for (int a = 0; a < n_adapters; ++a) {
    if (ranks[a] < 1 || ranks[a] > SQ_MAX_LORA_RANK) return -1;
    R += (ranks[a] + 15) / 16 * 16;
  }
  return R;
}

int sq_pack_lora(const uint16_t *const *A, const uint16_t *const *B, const int64_t *ranks,
                 const float *lora_alpha, int n_adapters, const float *s, int64_t K, int64_t N,
                 int64_t R, uint16_t *A_pack, uint16_t *B_pack, int32_t *lora_offset,
                 int32_t *lora_rank, void *stream) {
  if (!A || !B || !ranks || !lora_alpha || n_adapters < 1 || K < 0 || N < 0)
    return SQ_ERR_INVALID_ARG;
  if (K % 16 != 0 || K > SQ_MAX_K) return SQ_ERR_UNSUPPORTED_SHAPE;
  const int64_t width = sq_lora_pack_width(ranks, n_adapters);
  if (width < 0) return SQ_ERR_INVALID_ARG;
  if (width > SQ_MAX_LORA_COLS) return SQ_ERR_UNSUPPORTED_SHAPE;
  if (R != width) return SQ_ERR_INVALID_ARG;
  if ((s && !ptr_ok(s)) || !ptr_ok(A_pack) || !ptr_ok(B_pack) || !aligned_to(lora_offset, 4) ||
      !aligned_to(lora_rank, 4))
    return SQ_ERR_INVALID_ARG;
  for (int a = 0; a < n_adapters; ++a)
    if (!A[a] || !B[a]) return SQ_ERR_INVALID_ARG;
  int st = check_device();
  if (st) return st;
  cudaStream_t cs = static_cast<cudaStream_t>(stream);
  int32_t offs[SQ_MAX_LORA_COLS / 16], rks[SQ_MAX_LORA_COLS / 16];
  int64_t off = 0;
  for (int a = 0; a < n_adapters; ++a) {
    const float scale = lora_alpha[a] / static_cast<float>(ranks[a]);  // IEEE fp32 division
    cudaError_t e = launch_prepare_lora(A[a], B[a], s, ranks[a], K, N, scale, R, off, A_pack,
                                        B_pack, cs);
    if (e != cudaSuccess) return SQ_ERR_CUDA;
    offs[a] = static_cast<int32_t>(off);
    rks[a] = static_cast<int32_t>(ranks[a]);
    off += (ranks[a] + 15) / 16 * 16;
  }
  return cuda_status(launch_write_lora_table(offs, rks, n_adapters, lora_offset, lora_rank, cs));
}

int sq_quant_act(const void *X, int x_dtype, const float *s, int64_t M, int64_t K, int8_t *Xq,
                 float *x_scale, void *stream) {
  int st = check_mk(M, K);
  if (st) return st;
  if (x_dtype != SQ_DTYPE_BF16 && x_dtype != SQ_DTYPE_F32) return SQ_ERR_INVALID_ARG;
  if (M > 0 && (!ptr_ok(x_scale) || (K > 0 && (!ptr_ok(X) || !ptr_ok(s) || !ptr_ok(Xq)))))
    return SQ_ERR_INVALID_ARG;
  if ((st = check_device())) return st;
  return cuda_status(
      launch_quant_act(X, x_dtype, s, M, K, Xq, x_scale, static_cast<cudaStream_t>(stream)));
}


int sq_static_act_scale(const float *act_absmax, const float *s, int64_t K, float *scale,
                        void *stream) {
  int st = check_mk(1, K);
  if (st) return st;
  if (K == 0 || !ptr_ok(act_absmax) || !ptr_ok(s) || !aligned_to(scale, 4))
    return SQ_ERR_INVALID_ARG;
  if ((st = check_device())) return st;
  return cuda_status(
      launch_static_act_scale(act_absmax, s, K, scale, static_cast<cudaStream_t>(stream)));
}

int sq_quant_act_static(const void *X, int x_dtype, const float *s, const float *scale,
                        int64_t M, int64_t K, int8_t *Xq, float *x_scale,
                        unsigned long long *clip_count, void *stream) {
  int st = check_mk(M, K);
  if (st) return st;
  if (x_dtype != SQ_DTYPE_BF16 && x_dtype != SQ_DTYPE_F32) return SQ_ERR_INVALID_ARG;
  if (!aligned_to(scale, 4) || !aligned_to(clip_count, 8)) return SQ_ERR_INVALID_ARG;
  if (M > 0 && (!ptr_ok(x_scale) || (K > 0 && (!ptr_ok(X) || !ptr_ok(s) || !ptr_ok(Xq)))))
    return SQ_ERR_INVALID_ARG;
  if ((st = check_device())) return st;
  // (K == 0: no codes, the scale is still every token's scale)
  return cuda_status(launch_quant_act_static(X, x_dtype, s, scale, M, K, Xq, x_scale, clip_count,
                                             static_cast<cudaStream_t>(stream)));
}

int sq_fold_norm_weight(const float *gamma, const float *s, int64_t K, float *gamma_s,
                        void *stream) {
  int st = check_mk(1, K);
  if (st) return st;
  if (K > 0 && (!ptr_ok(gamma) || !ptr_ok(s) || !ptr_ok(gamma_s))) return SQ_ERR_INVALID_ARG;
  if ((st = check_device())) return st;
  if (K == 0) return SQ_OK;
  return cuda_status(
      launch_fold_norm_weight(gamma, s, K, gamma_s, static_cast<cudaStream_t>(stream)));
}

int sq_rmsnorm_quant_act(const uint16_t *H, const float *gamma_s, float eps, int64_t M, int64_t K,
                         int8_t *Xq, float *x_scale, void *stream) {
  int st = check_mk(M, K);
  if (st) return st;
  if (K == 0 || !rmsnorm_quant_supported(K)) return SQ_ERR_UNSUPPORTED_SHAPE;
  if (!(eps >= 0.0f) || !(eps < 3.4e38f)) return SQ_ERR_INVALID_ARG;
  if (M > 0 && (!ptr_ok(H) || !ptr_ok(gamma_s) || !ptr_ok(Xq) || !ptr_ok(x_scale)))
    return SQ_ERR_INVALID_ARG;
  if ((st = check_device())) return st;
  return cuda_status(launch_rmsnorm_quant(H, gamma_s, eps, M, K, Xq, x_scale,
                                          static_cast<cudaStream_t>(stream)));
}

size_t sq_linear_lora_workspace_size(int64_t M, int64_t R) { return workspace_bytes(M, R); }

static int linear_common(const int8_t *Xq, const float *x_scale, const int8_t *Wq,
                         const float *w_scale, int64_t M, int64_t N, int64_t K,
                         const uint16_t *A_pack, const uint16_t *B_pack,
                         const int32_t *lora_offset, const int32_t *lora_rank, int n_adapters,
                         int64_t R, const int32_t *seg_offsets, const int32_t *seg_adapter,
                         int64_t S, int mode, void *out, void *workspace, size_t workspace_size,
                         void *stream) {
  int st = check_mk(M, K);
  if (st) return st;
  if (N < 0) return SQ_ERR_INVALID_ARG;
  if (N % 16 != 0) return SQ_ERR_UNSUPPORTED_SHAPE;
  bool lora = false;
  if (mode != 1) {
    st = check_lora_args(M, K, A_pack, B_pack, lora_offset, lora_rank, n_adapters, R, seg_offsets,
                         seg_adapter, S, workspace, workspace_size, &lora);
    if (st) return st;
  }
  if (M == 0 || N == 0) return check_device();
  if (!ptr_ok(out)) return SQ_ERR_INVALID_ARG;
  if (K > 0 && (!ptr_ok(Xq) || (mode != 2 && !ptr_ok(Wq)))) return SQ_ERR_INVALID_ARG;
  if (mode != 1 && !ptr_ok(x_scale)) return SQ_ERR_INVALID_ARG;
  if (mode == 0 && !ptr_ok(w_scale)) return SQ_ERR_INVALID_ARG;
  if ((st = check_device())) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const size_t esize = (mode == 0) ? 2 : 4;
  if (K == 0 || (mode == 2 && !lora)) {
    // empty contraction (and no LoRA rows with K == 0 either: T = 0)
    return cuda_status(cudaMemsetAsync(out, 0, static_cast<size_t>(M) * N * esize, s));
  }
  if (decode_applicable(M)) {
    // few tokens: bound by streaming the weights, see decode.cu
    const bool timed = (mode == 0) && g_gemm_ev_before != nullptr;
    if (timed && cudaEventRecord(g_gemm_ev_before, s) != cudaSuccess) return SQ_ERR_CUDA;
    cudaError_t e = launch_decode(Xq, x_scale, Wq, w_scale, M, N, K, mode, A_pack, B_pack,
                                  lora_offset, lora_rank, n_adapters, R, seg_offsets, seg_adapter,
                                  S, lora ? static_cast<float *>(workspace) : nullptr, out, s);
    if (e != cudaSuccess) return SQ_ERR_CUDA;
    if (timed && cudaEventRecord(g_gemm_ev_after, s) != cudaSuccess) return SQ_ERR_CUDA;
    return SQ_OK;
  }
  LoraOperands lo;
  LoraOperands *lop = nullptr;
  if (lora) {
    Workspace w = carve(workspace, M, R);
    cudaError_t e = launch_lora_shrink(Xq, x_scale, M, K, A_pack, lora_offset, lora_rank,
                                       n_adapters, R, seg_offsets, seg_adapter, S, w.T_hi, w.T_lo,
                                       w.mask, s);
    if (e != cudaSuccess) return SQ_ERR_CUDA;
    lo = LoraOperands{w.T_hi, w.T_lo, B_pack, w.mask, R};
    lop = &lo;
  }
  const bool timed = (mode == 0) && g_gemm_ev_before != nullptr;
  if (timed && cudaEventRecord(g_gemm_ev_before, s) != cudaSuccess) return SQ_ERR_CUDA;
  cudaError_t e = launch_w8a8_gemm(Xq, Wq, x_scale, w_scale, M, N, K, mode, out, lop, s);
  if (e != cudaSuccess) return SQ_ERR_CUDA;
  if (timed && cudaEventRecord(g_gemm_ev_after, s) != cudaSuccess) return SQ_ERR_CUDA;
  return SQ_OK;
}

int sq_linear_lora(const int8_t *Xq, const float *x_scale, const int8_t *Wq, const float *w_scale,
                   int64_t M, int64_t N, int64_t K, const uint16_t *A_pack, const uint16_t *B_pack,
                   const int32_t *lora_offset, const int32_t *lora_rank, int n_adapters, int64_t R,
                   const int32_t *seg_offsets, const int32_t *seg_adapter, int64_t S, uint16_t *Y,
                   void *workspace, size_t workspace_size, void *stream) {
  return linear_common(Xq, x_scale, Wq, w_scale, M, N, K, A_pack, B_pack, lora_offset, lora_rank,
                       n_adapters, R, seg_offsets, seg_adapter, S, 0, Y, workspace, workspace_size,
                       stream);
}

int sq_gemm_i32(const int8_t *Xq, const int8_t *Wq, int64_t M, int64_t N, int64_t K, int32_t *acc,
                void *stream) {
  return linear_common(Xq, nullptr, Wq, nullptr, M, N, K, nullptr, nullptr, nullptr, nullptr, 0, 0,
                       nullptr, nullptr, 0, 1, acc, nullptr, 0, stream);
}

int sq_lora_delta(const int8_t *Xq, const float *x_scale, int64_t M, int64_t N, int64_t K,
                  const uint16_t *A_pack, const uint16_t *B_pack, const int32_t *lora_offset,
                  const int32_t *lora_rank, int n_adapters, int64_t R, const int32_t *seg_offsets,
                  const int32_t *seg_adapter, int64_t S, float *delta, void *workspace,
                  size_t workspace_size, void *stream) {
  return linear_common(Xq, x_scale, nullptr, nullptr, M, N, K, A_pack, B_pack, lora_offset,
                       lora_rank, n_adapters, R, seg_offsets, seg_adapter, S, 2, delta, workspace,
                       workspace_size, stream);
}

// ---- layer-wise output error for one alpha (offline diagnostic) ------------
size_t sq_alpha_error_workspace_size(int64_t M, int64_t N, int64_t K) {
  return alpha_error_workspace_bytes(M, N, K);
}

int sq_alpha_output_error(const void *X, int x_dtype, const uint16_t *W, int64_t M, int64_t N,
                          int64_t K, float alpha, double *err, void *workspace,
                          size_t workspace_size, void *stream) {
  int st = check_mk(M, K);
  if (st) return st;
  if (x_dtype != SQ_DTYPE_BF16 && x_dtype != SQ_DTYPE_F32) return SQ_ERR_INVALID_ARG;
  if (!(alpha >= 0.0f && alpha <= 1.0f) || M <= 0 || N <= 0 || K <= 0) return SQ_ERR_INVALID_ARG;
  if (N % 16 != 0) return SQ_ERR_UNSUPPORTED_SHAPE;
  if (!ptr_ok(X) || !ptr_ok(W) || !aligned_to(err, 8)) return SQ_ERR_INVALID_ARG;
  if (!workspace || (reinterpret_cast<uintptr_t>(workspace) & 255u) ||
      workspace_size < alpha_error_workspace_bytes(M, N, K))
    return SQ_ERR_WORKSPACE;
  if ((st = check_device())) return st;
  return cuda_status(launch_alpha_error(X, x_dtype, W, M, N, K, alpha, err, workspace,
                                        static_cast<cudaStream_t>(stream)));
}

int sq_alpha_sweep(const void *X, int x_dtype, const uint16_t *W, int64_t M, int64_t N, int64_t K,
                   const float *alphas, int n, double *err, double *rel, float *best,
                   void *workspace, size_t workspace_size, void *stream) {
  int st = check_mk(M, K);
  if (st) return st;
  if (x_dtype != SQ_DTYPE_BF16 && x_dtype != SQ_DTYPE_F32) return SQ_ERR_INVALID_ARG;
  if (M <= 0 || N <= 0 || K <= 0 || n < 1 || n > SQ_ALPHA_SWEEP_MAX || !alphas)
    return SQ_ERR_INVALID_ARG;
  for (int t = 0; t < n; ++t)
    if (!(alphas[t] >= 0.0f && alphas[t] <= 1.0f)) return SQ_ERR_INVALID_ARG;
  if (N % 16 != 0) return SQ_ERR_UNSUPPORTED_SHAPE;
  if (!ptr_ok(X) || !ptr_ok(W) || !aligned_to(err, 8) || !aligned_to(rel, 8) || !aligned_to(best, 4))
    return SQ_ERR_INVALID_ARG;
  if (!workspace || (reinterpret_cast<uintptr_t>(workspace) & 255u) ||
      workspace_size < alpha_error_workspace_bytes(M, N, K))
    return SQ_ERR_WORKSPACE;
  if ((st = check_device())) return st;
  return cuda_status(launch_alpha_sweep(X, x_dtype, W, M, N, K, alphas, n, err, rel, best,
                                        workspace, static_cast<cudaStream_t>(stream)));
}

// ---- raw-input reading of the LoRA path ------------------------------------
size_t sq_lora_t_workspace_size(int64_t M, int64_t R) { return t_workspace_bytes(M, R); }

int sq_lora_shrink_raw(const uint16_t *X, int64_t M, int64_t K, const uint16_t *A_pack,
                       const int32_t *lora_offset, const int32_t *lora_rank, int n_adapters,
                       int64_t R, const int32_t *seg_offsets, const int32_t *seg_adapter,
                       int64_t S, void *workspace, size_t workspace_size, void *stream) {
  int st = check_mk(M, K);
  if (st) return st;
  if (n_adapters < 0 || R <= 0 || S < 0) return SQ_ERR_INVALID_ARG;
  if (R % 16 != 0 || R > SQ_MAX_LORA_COLS) return SQ_ERR_UNSUPPORTED_SHAPE;
  if (M == 0) return check_device();
  if (!workspace || (reinterpret_cast<uintptr_t>(workspace) & 255u) ||
      workspace_size < t_workspace_bytes(M, R))
    return SQ_ERR_WORKSPACE;
  if (K > 0 && (!ptr_ok(X) || !ptr_ok(A_pack))) return SQ_ERR_INVALID_ARG;
  if (n_adapters > 0 && (!lora_offset || !lora_rank)) return SQ_ERR_INVALID_ARG;
  if (S > 0 && (!seg_offsets || !seg_adapter)) return SQ_ERR_INVALID_ARG;
  if ((st = check_device())) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  Workspace w = carve(workspace, M, R);
  if (K == 0 || n_adapters == 0 || S == 0)  // no adapter rows or no contraction: T = 0, masks 0
    return cuda_status(cudaMemsetAsync(workspace, 0, t_workspace_bytes(M, R), s));
  return cuda_status(launch_lora_shrink_raw(X, M, K, A_pack, lora_offset, lora_rank, n_adapters,
                                            R, seg_offsets, seg_adapter, S, w.T_hi, w.T_lo, w.mask,
                                            s));
}

// Y or the delta alone (mode 0 / 2) from the T planes in the workspace
static int from_t_common(const int8_t *Xq, const float *x_scale, const int8_t *Wq,
                         const float *w_scale, int64_t M, int64_t N, int64_t K,
                         const uint16_t *B_pack, int64_t R, int mode, void *out,
                         const void *workspace, size_t workspace_size, void *stream) {
  int st = check_mk(M, K);
  if (st) return st;
  if (N < 0 || R < 0) return SQ_ERR_INVALID_ARG;
  if (N % 16 != 0) return SQ_ERR_UNSUPPORTED_SHAPE;
  if (R % 16 != 0 || R > SQ_MAX_LORA_COLS) return SQ_ERR_UNSUPPORTED_SHAPE;
  if (M == 0 || N == 0) return check_device();
  if (!ptr_ok(out)) return SQ_ERR_INVALID_ARG;
  if (K > 0 && (!ptr_ok(Xq) || (mode == 0 && (!ptr_ok(Wq) || !ptr_ok(x_scale) || !ptr_ok(w_scale)))))
    return SQ_ERR_INVALID_ARG;
  const bool lora = R > 0;
  if (lora && !ptr_ok(B_pack)) return SQ_ERR_INVALID_ARG;
  if (lora && (!workspace || (reinterpret_cast<uintptr_t>(workspace) & 255u) ||
               workspace_size < t_workspace_bytes(M, R)))
    return SQ_ERR_WORKSPACE;
  if ((st = check_device())) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const size_t esize = (mode == 0) ? 2 : 4;
  // K == 0: no contraction and T = 0 (sq_lora_shrink_raw), so the output is 0
  if (K == 0 || (mode == 2 && !lora))
    return cuda_status(cudaMemsetAsync(out, 0, static_cast<size_t>(M) * N * esize, s));
  LoraOperands lo;
  LoraOperands *lop = nullptr;
  if (lora) {
    Workspace w = carve(const_cast<void *>(workspace), M, R);
    lo = LoraOperands{w.T_hi, w.T_lo, B_pack, w.mask, R};
    lop = &lo;
  }
  const bool timed = (mode == 0) && g_gemm_ev_before != nullptr;
  if (timed && cudaEventRecord(g_gemm_ev_before, s) != cudaSuccess) return SQ_ERR_CUDA;
  cudaError_t e = launch_w8a8_gemm(Xq, Wq, x_scale, w_scale, M, N, K, mode, out, lop, s);
  if (e != cudaSuccess) return SQ_ERR_CUDA;
  if (timed && cudaEventRecord(g_gemm_ev_after, s) != cudaSuccess) return SQ_ERR_CUDA;
  return SQ_OK;
}

int sq_linear_lora_from_t(const int8_t *Xq, const float *x_scale, const int8_t *Wq,
                          const float *w_scale, int64_t M, int64_t N, int64_t K,
                          const uint16_t *B_pack, int64_t R, uint16_t *Y, const void *workspace,
                          size_t workspace_size, void *stream) {
  return from_t_common(Xq, x_scale, Wq, w_scale, M, N, K, B_pack, R, 0, Y, workspace,
                       workspace_size, stream);
}

int sq_lora_delta_from_t(const int8_t *Xq, int64_t M, int64_t N, int64_t K,
                         const uint16_t *B_pack, int64_t R, float *delta, const void *workspace,
                         size_t workspace_size, void *stream) {
  return from_t_common(Xq, nullptr, nullptr, nullptr, M, N, K, B_pack, R, 2, delta, workspace,
                       workspace_size, stream);
}

}  // extern "C"
