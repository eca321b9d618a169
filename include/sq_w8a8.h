/*
 * sq_w8a8.h -- C ABI of the SmoothQuant W8A8 linear layer with a
 * per-request LoRA delta, for NVIDIA B200 (sm_100a).
 *
 * What it computes (sources named by page title and section):
 *  - "SmoothQuant" explainer (ozercemkelahmet.com/tools/smoothquant),
 *    How it works, Steps 2-7, and its Python sketch: per-channel smoothing
 *    s_j = max|X_j|^alpha / max|W_j|^(1-alpha), folded into the weights;
 *    per-token dynamic INT8 activations; per-output-channel INT8 weights;
 *    INT8 x INT8 GEMM with INT32 accumulation, dequantized with the stored
 *    scales.
 *  - "[Feature]: LoRA support for W8A8 SmoothQuant" (TensorRT-LLM issue
 *    #12703), Pitch: a BF16 low-rank LoRA path after the INT8 GEMM whose
 *    result is added to the dequantized output; Motivation: one adapter per
 *    request, many requests per batch.
 *
 * Conventions for every call:
 *  - All tensor pointers are DEVICE pointers owned by the caller, row-major,
 *    16-byte aligned.  The library never allocates device memory.
 *  - bf16 tensors are passed as uint16_t bit patterns.
 *  - `stream` is a cudaStream_t (NULL = the legacy default stream).  Calls
 *    only enqueue work: they return after validating arguments and
 *    launching, and the results are ready when the stream reaches them.
 *  - Return value: SQ_OK (0) or an sq_status code.  Argument errors are found
 *    on the host before anything is launched and leave the outputs untouched.
 *    Errors found on the device (a wait that ran out, a segment naming an
 *    adapter that does not exist) do not fault: the kernel records a code
 *    that sq_get_device_error() returns.
 *  - Only compute capability 10.0 (B200) is supported; other devices get
 *    SQ_ERR_UNSUPPORTED_DEVICE.  There is no fallback path.
 *
 * Shapes: M tokens, K input channels, N output channels.
 *   X  [M,K]  bf16 or f32        Xq [M,K] int8      x_scale [M] f32
 *   W  [N,K]  bf16 (torch Linear layout: output channels by input channels)
 *   Wq [N,K]  int8               w_scale [N] f32    s [K] f32
 *   Y  [M,N]  bf16
 * Constraints: K % 16 == 0, N % 16 == 0, K <= SQ_MAX_K (a row of K fp32
 * values is staged in shared memory; K*127^2 then also fits in int32).
 */
#ifndef SQ_W8A8_H
#define SQ_W8A8_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum sq_status {
  SQ_OK = 0,
  SQ_ERR_INVALID_ARG = 1,        /* null/misaligned pointer, negative size  */
  SQ_ERR_UNSUPPORTED_SHAPE = 2,  /* K or N not a multiple of 16, K too big  */
  SQ_ERR_UNSUPPORTED_DEVICE = 3, /* not compute capability 10.0             */
  SQ_ERR_CUDA = 4,               /* a CUDA runtime call failed              */
  SQ_ERR_DEVICE_TIMEOUT = 5,     /* a bounded device-side wait ran out      */
  SQ_ERR_WORKSPACE = 6,          /* workspace missing or too small          */
  SQ_ERR_BAD_SEGMENTS = 7        /* device: adapter index out of range      */
} sq_status;

typedef enum sq_dtype { SQ_DTYPE_F32 = 0, SQ_DTYPE_BF16 = 1 } sq_dtype;

/* Largest supported number of input channels. */
#define SQ_MAX_K 57344

/* Largest packed LoRA width (sum over adapters of the rank rounded up to 16). */
#define SQ_MAX_LORA_COLS 1024

/* Largest rank of one adapter. */
#define SQ_MAX_LORA_RANK 256

/* Human-readable name of a status code (static string, never NULL). */
const char *sq_status_string(int status);

/* Library version as 10000*major + 100*minor + patch. */
int sq_version(void);

/* SQ_OK if `device` is a compute capability 10.0 GPU, else
 * SQ_ERR_UNSUPPORTED_DEVICE (or SQ_ERR_CUDA if it cannot be queried). */
int sq_device_supported(int device);

/* Device-side error code recorded by earlier launches on the current device
 * (an sq_status value, 0 if none), after synchronizing the device.  If
 * `clear` is nonzero the record is reset to 0. */
int sq_get_device_error(int *code, int clear);

/* Upper bound, in nanoseconds, of every spin-wait inside the kernels
 * (default 2 s).  A wait that runs out makes the kernel stop, record
 * SQ_ERR_DEVICE_TIMEOUT and return.  Bounds below 1 us (finer than the
 * device timer) make a wait give up after one non-blocking probe.  Host-side
 * setting for later launches. */
int sq_set_wait_timeout_ns(uint64_t ns);

/* Test of failure detection: launches one block that waits, with the bound
 * `timeout_ns` (1 ns .. 100 ms), on a barrier nothing ever arrives on.  The
 * wait gives up and SQ_ERR_DEVICE_TIMEOUT is recorded for
 * sq_get_device_error(); the context stays usable.  Returns the launch
 * status. */
int sq_selftest_wait_timeout(uint64_t timeout_ns, void *stream);

/* Measurement aid: when both are non-NULL, sq_linear_lora (and
 * sq_linear_lora_from_t) records the cudaEvent_t `before` on its stream right
 * before it launches the fused GEMM kernel and `after` right after, so a
 * caller can time that kernel alone.
 * NULL disables.  Host-side setting for later calls. */
int sq_set_gemm_events(void *before, void *after);

/* ---------------------------------------------------------------------------
 * Offline preparation ("SmoothQuant" explainer, Steps 3-5 and the sketch)
 * ------------------------------------------------------------------------ */

/* Calibration ("Calibration in practice"): act_absmax[j] =
 * max(act_absmax[j], max_i |X[i,j]|).  X [M,K] of x_dtype; act_absmax [K]
 * f32, read and written (zero it before the first batch). */
int sq_act_absmax_update(const void *X, int x_dtype, int64_t M, int64_t K,
                         float *act_absmax, void *stream);

/* w_absmax[j] = max_n |W[n,j]| (the sketch's abs().max(dim=0) over the
 * output channels).  W [N,K] bf16; w_absmax [K] f32, written. */
int sq_weight_absmax(const uint16_t *W, int64_t N, int64_t K, float *w_absmax,
                     void *stream);

/* Step 3 and the sketch: s_j = max(max(a_j,1e-5)^alpha /
 * max(w_j,1e-5)^(1-alpha), 1e-5), evaluated in fp64 and rounded once to fp32.
 * act_absmax, w_absmax, s: [K] f32. alpha in [0,1]. */
int sq_compute_smoothing(const float *act_absmax, const float *w_absmax, int64_t K,
                         float alpha, float *s, void *stream);

/* Steps 5-6: fold s into the weights along the input channels and quantize
 * each output channel:  W' = fp32(W[n,k]*s_k);  w_scale_n = max_k|W'|/127;
 * Wq = clamp(round_half_even(W'/w_scale_n), -128, 127)  (IEEE fp32 division;
 * an all-zero channel gets scale 0 and codes 0).  Bit-exact. */
int sq_quantize_weight(const uint16_t *W, const float *s, int64_t N, int64_t K,
                       int8_t *Wq, float *w_scale, void *stream);

/* LoRA adapter table.  Adapters are packed side by side: adapter a of rank
 * r_a owns columns [off_a, off_a + round_up(r_a,16)) of the packed width
 * R = sum_a round_up(r_a,16) <= SQ_MAX_LORA_COLS, in
 *   A_pack [R, K] bf16 : rows off_a+j   = bf16(fp32(A_a[j,k] * s_k))
 *   B_pack [N, R] bf16 : cols off_a+j   = bf16(fp32(B_a[n,j] * lora_alpha/r))
 * with zeros in the padding rows/columns.  Folding s into A lets the LoRA
 * path read the dequantized activations Xq*x_scale (which approximate X/s)
 * and still compute X*A^T; folding lora_alpha/r into B applies the LoRA
 * scaling once, offline.  This call writes adapter (A [r,K], B [N,r], both
 * bf16, 1 <= r <= SQ_MAX_LORA_RANK) at column offset `off` (a multiple of 16)
 * of a pack of width R.  s == NULL packs A unchanged (the raw-input reading,
 * see sq_lora_shrink_raw). */
int sq_prepare_lora(const uint16_t *A, const uint16_t *B, const float *s, int64_t r,
                    int64_t K, int64_t N, float lora_alpha, int64_t R, int64_t off,
                    uint16_t *A_pack, uint16_t *B_pack, void *stream);

/* The whole adapter table in one call, from adapters held in separate
 * buffers (a list lora_A[], lora_B[] of per-request adapters, "[Feature]:
 * LoRA support for W8A8 SmoothQuant", Motivation: one adapter per request).
 * A[a] [ranks[a], K] and B[a] [N, ranks[a]] (bf16, device) are given as host
 * arrays of n_adapters device pointers, with lora_alpha[a] (host) and s
 * (device; NULL packs A unchanged, as sq_prepare_lora).  Adapter a goes to
 * columns [off_a, off_a + round_up(r_a, 16)), off_a the sum of the earlier
 * adapters' rounded ranks; R must be that total (sq_lora_pack_width).
 * Writes A_pack [R, K], B_pack [N, R] as sq_prepare_lora does for each
 * adapter, and lora_offset, lora_rank [n_adapters] (device int32) = off_a,
 * r_a: the table sq_linear_lora takes.  Errors: SQ_ERR_INVALID_ARG (null or
 * misaligned pointers, a rank outside [1, SQ_MAX_LORA_RANK], R not the
 * total), SQ_ERR_UNSUPPORTED_SHAPE (K % 16, K > SQ_MAX_K, total width above
 * SQ_MAX_LORA_COLS).  Enqueued on `stream`; the host arrays may be reused
 * when the call returns. */
int64_t sq_lora_pack_width(const int64_t *ranks, int n_adapters);
int sq_pack_lora(const uint16_t *const *A, const uint16_t *const *B, const int64_t *ranks,
                 const float *lora_alpha, int n_adapters, const float *s, int64_t K, int64_t N,
                 int64_t R, uint16_t *A_pack, uint16_t *B_pack, int32_t *lora_offset,
                 int32_t *lora_rank, void *stream);

/* ---------------------------------------------------------------------------
 * Hot path
 * ------------------------------------------------------------------------ */

/* Steps 2 and 6 (dynamic per-token scales): divide each channel by s_j, then
 * quantize each token:  xt = fp32(X[i,j]/s_j);  x_scale_i = max_j|xt|/127;
 * Xq = clamp(round_half_even(xt/x_scale_i), -128, 127), all divisions IEEE
 * fp32 (an all-zero token gets scale 0 and codes 0).  Bit-exact.
 * X [M,K] of x_dtype (SQ_DTYPE_BF16 or SQ_DTYPE_F32). */
int sq_quant_act(const void *X, int x_dtype, const float *s, int64_t M, int64_t K,
                 int8_t *Xq, float *x_scale, void *stream);

/* Per-tensor static level of Step 6 ("SmoothQuant" explainer, Step 6 and
 * "Calibration in practice": one activation scale for every token, fixed
 * offline from the calibration range; faster, and values outside the
 * calibrated range are clipped).
 * sq_static_act_scale: *scale = RN(max_j RN(act_absmax_j / s_j) / 127), IEEE
 * fp32 divisions.  act_absmax, s: [K] f32 device; scale: one f32, device. */
int sq_static_act_scale(const float *act_absmax, const float *s, int64_t K, float *scale,
                        void *stream);

/* xt = RN(X[i,j] / s_j);  Xq = clamp(round_half_even(RN(xt / scale)), -128, 127);
 * x_scale[i] = scale for every token (so sq_linear_lora takes it unchanged);
 * *clip_count += the number of codes the clamp changed (scale == 0: codes 0,
 * every nonzero xt counts).  scale: one f32 (device, e.g. from
 * sq_static_act_scale); clip_count: one u64 (device, 8-byte aligned; zero it
 * before a run to count that run).  Bit-exact. */
int sq_quant_act_static(const void *X, int x_dtype, const float *s, const float *scale,
                        int64_t M, int64_t K, int8_t *Xq, float *x_scale,
                        unsigned long long *clip_count, void *stream);

/* Step 5 with a normalization in front of the layer ("the inverse scale can
 * be folded into the normalization layer's weights"):
 * sq_fold_norm_weight: gamma_s[j] = RN(gamma[j] / s_j) (IEEE fp32 division;
 * offline).  gamma, s, gamma_s: [K] f32 device. */
int sq_fold_norm_weight(const float *gamma, const float *s, int64_t K, float *gamma_s,
                        void *stream);

/* RMS normalization with the folded weight fused with Step 6 (per token):
 *   r_i = RN32(1 / sqrt(ss_i / K + eps))  with ss_i the exact sum of the
 *         squares of the row, rounded once to fp64; the division by K, the
 *         + eps, the square root and the reciprocal are correctly rounded
 *         fp64 operations,
 *   xt = RN(RN(H[i,j] * r_i) * gamma_s[j]);  x_scale_i = RN(max_j |xt| / 127);
 *   Xq = clamp(round_half_even(RN(xt / x_scale_i)), -128, 127).
 * H [M,K] bf16 (the layer's pre-normalization input), device.  Bit-exact for
 * every finite row.  K % 16 == 0 and K <= 32768, else
 * SQ_ERR_UNSUPPORTED_SHAPE; eps >= 0. */
int sq_rmsnorm_quant_act(const uint16_t *H, const float *gamma_s, float eps, int64_t M, int64_t K,
                         int8_t *Xq, float *x_scale, void *stream);

/* Bytes of device workspace sq_linear_lora needs for M tokens and a LoRA
 * pack of width R (0 when R == 0). */
size_t sq_linear_lora_workspace_size(int64_t M, int64_t R);

/* Step 7 plus the LoRA delta, one launch sequence (M <= 64 tokens take a
 * form built for streaming the weights; larger M the tensor-core tile form):
 *   Y[i,n] = bf16( f32(acc[i,n]) * x_scale_i * w_scale_n + delta[i,n] ),
 *   acc = Xq Wq^T (exact int32), delta[i,:] = (x_scale_i Xq[i,:] A_pack_a^T)
 *   B_pack_a^T for the adapter a of token i (none: delta = 0).
 * Segments: seg_offsets [S+1] and seg_adapter [S] (device int32): token i
 * belongs to the first segment s with seg_offsets[s] <= i < seg_offsets[s+1]
 * and uses adapter seg_adapter[s]; -1 (or no segment) means no LoRA.  An
 * adapter index >= n_adapters is treated as -1 and recorded as
 * SQ_ERR_BAD_SEGMENTS.  lora_offset / lora_rank: [n_adapters] device int32
 * (column offset and rank of each adapter in the pack).  With R == 0,
 * n_adapters == 0 or S == 0 the layer is plain W8A8 and the LoRA arguments
 * may be NULL.  workspace: >= sq_linear_lora_workspace_size(M, R) bytes of
 * device memory, 256-byte aligned; its contents are scratch. */
int sq_linear_lora(const int8_t *Xq, const float *x_scale, const int8_t *Wq,
                   const float *w_scale, int64_t M, int64_t N, int64_t K,
                   const uint16_t *A_pack, const uint16_t *B_pack,
                   const int32_t *lora_offset, const int32_t *lora_rank, int n_adapters,
                   int64_t R, const int32_t *seg_offsets, const int32_t *seg_adapter,
                   int64_t S, uint16_t *Y, void *workspace, size_t workspace_bytes,
                   void *stream);

/* Scratch size of sq_linear_lora_noalloc (bytes). */
#define SQ_NOALLOC_SCRATCH_BYTES (16u << 20)

/* sq_linear_lora without a caller-provided workspace, for callers that cannot
 * allocate device memory: code that runs inside an engine which plans every
 * byte of device memory ahead and gives its plugins no allocator, or that
 * must not call cudaMalloc at that point (it blocks the device and may fail
 * under fragmentation).  The pages have no counterpart of this call.
 * The scratch is one static device array of SQ_NOALLOC_SCRATCH_BYTES (16 MiB)
 * that every GPU loading the library holds until the process exits; a call
 * whose sq_linear_lora_workspace_size(M, R) exceeds it returns
 * SQ_ERR_WORKSPACE (checked after the shapes, and only when an adapter is in
 * play, as sq_linear_lora checks a workspace).  The first call on each device
 * looks up the array's device address (cudaGetSymbolAddress), so make that
 * first call before any stream capture; on a device that is not compute
 * capability 10.0 every call returns SQ_ERR_UNSUPPORTED_DEVICE before its
 * arguments are looked at.  Each device has its own copy of the array and
 * every call on that device uses it, keeping what the last call left there:
 * calls that overlap on one GPU (for example on two streams) race, so
 * serialize them.  After cudaDeviceReset of a device the library must not be
 * used on it again.  Other arguments, results and errors as sq_linear_lora.
 * Allocates nothing. */
int sq_linear_lora_noalloc(const int8_t *Xq, const float *x_scale, const int8_t *Wq,
                           const float *w_scale, int64_t M, int64_t N, int64_t K,
                           const uint16_t *A_pack, const uint16_t *B_pack,
                           const int32_t *lora_offset, const int32_t *lora_rank, int n_adapters,
                           int64_t R, const int32_t *seg_offsets, const int32_t *seg_adapter,
                           int64_t S, uint16_t *Y, void *stream);

/* ---------------------------------------------------------------------------
 * Test entries: the same kernels with a different epilogue
 * ------------------------------------------------------------------------ */

/* acc [M,N] int32 = Xq Wq^T exactly (the INT32 accumulators of Step 7). */
int sq_gemm_i32(const int8_t *Xq, const int8_t *Wq, int64_t M, int64_t N, int64_t K,
                int32_t *acc, void *stream);

/* delta [M,N] f32: the LoRA delta alone, as sq_linear_lora adds it. */
int sq_lora_delta(const int8_t *Xq, const float *x_scale, int64_t M, int64_t N,
                  int64_t K, const uint16_t *A_pack, const uint16_t *B_pack,
                  const int32_t *lora_offset, const int32_t *lora_rank, int n_adapters,
                  int64_t R, const int32_t *seg_offsets, const int32_t *seg_adapter,
                  int64_t S, float *delta, void *workspace, size_t workspace_bytes,
                  void *stream);

/* ---------------------------------------------------------------------------
 * Offline diagnostic: layer-wise output error for one migration strength
 * ("SmoothQuant" explainer, "Reading the diagnostics": compare layer-wise
 * output error across alpha values; "Variants and related ideas": choose
 * alpha layer by layer by calibration error).  On the calibration tokens X
 * [M,K] (bf16 or f32, device) and the weights W [N,K] bf16 (device): the
 * calibration maxima of X and W, s(alpha), the quantized weights and
 * activations and the fused GEMM's Y (bf16, no adapters), then
 *   err[0] = sum (Y - X W^T)^2,  err[1] = sum (X W^T)^2
 * with X W^T from the unquantized operands (fp32 products and sums, fp64
 * totals).  err: two doubles, device, overwritten.  alpha in [0, 1].
 * workspace: >= sq_alpha_error_workspace_size(M, N, K) bytes, 256-byte
 * aligned device memory (scratch).  Errors: SQ_ERR_INVALID_ARG,
 * SQ_ERR_UNSUPPORTED_SHAPE (K % 16, N % 16), SQ_ERR_WORKSPACE. */
size_t sq_alpha_error_workspace_size(int64_t M, int64_t N, int64_t K);
int sq_alpha_output_error(const void *X, int x_dtype, const uint16_t *W, int64_t M, int64_t N,
                          int64_t K, float alpha, double *err, void *workspace,
                          size_t workspace_bytes, void *stream);

/* Largest number of alpha values of one sq_alpha_sweep. */
#define SQ_ALPHA_SWEEP_MAX 64

/* The per-layer choice of alpha by calibration error ("SmoothQuant"
 * explainer, "Variants and related ideas": pick alpha layer by layer by the
 * output error on calibration data; "Reading the diagnostics": a sharp
 * minimum suggests a good choice).  For each of the n values alphas[t] (host
 * array, 1 <= n <= SQ_ALPHA_SWEEP_MAX, each in [0, 1]) the two sums of
 * sq_alpha_output_error go to err[2t], err[2t+1]; then
 *   rel[t] = err[2t] / err[2t+1]   (IEEE fp64 division; 0 if err[2t+1] == 0)
 * and *best = the alpha with the smallest rel (the first one on ties).
 * err [2n] double, rel [n] double, best one float: device memory, written
 * on the stream (no host synchronization).  X, W, shapes and workspace as for
 * sq_alpha_output_error; errors as there, plus SQ_ERR_INVALID_ARG for n or
 * an alpha out of range. */
int sq_alpha_sweep(const void *X, int x_dtype, const uint16_t *W, int64_t M, int64_t N, int64_t K,
                   const float *alphas, int n, double *err, double *rel, float *best,
                   void *workspace, size_t workspace_bytes, void *stream);

/* ---------------------------------------------------------------------------
 * Raw-input reading of the LoRA path ("[Feature]: LoRA support for W8A8
 * SmoothQuant", Pitch: the low-rank path runs in BF16 after the INT8 GEMM
 * and is added to the dequantized output), taken on the layer's own bf16
 * activations instead of the dequantized codes:
 *   T[i,j] = sum_k X[i,k] * A_a[j,k]      (X bf16, A_a the adapter as given)
 *   Y[i,n] = bf16( f32(acc[i,n]) * x_scale_i * w_scale_n + sum_j T[i,j] * B_pack[n, off_a+j] )
 * The adapters are packed by sq_prepare_lora with s == NULL (A unchanged,
 * B scaled by lora_alpha/r as above).  T is kept in a caller-provided
 * workspace between the two calls.
 * ------------------------------------------------------------------------ */

/* Bytes of workspace for the T planes and mask words of M tokens and a pack
 * of width R (any M; 0 when R == 0 or M == 0). */
size_t sq_lora_t_workspace_size(int64_t M, int64_t R);

/* T for every token, written to `workspace` (>= sq_lora_t_workspace_size(M, R)
 * bytes, 256-byte aligned, device memory; contents replaced).  X [M,K] bf16
 * device; A_pack [R,K] bf16 packed with s == NULL; lora_offset, lora_rank,
 * seg_offsets, seg_adapter as for sq_linear_lora (tokens without an adapter
 * get T = 0).  Errors: SQ_ERR_INVALID_ARG (null or misaligned pointers),
 * SQ_ERR_UNSUPPORTED_SHAPE (K % 16, R % 16, limits), SQ_ERR_WORKSPACE. */
int sq_lora_shrink_raw(const uint16_t *X, int64_t M, int64_t K, const uint16_t *A_pack,
                       const int32_t *lora_offset, const int32_t *lora_rank, int n_adapters,
                       int64_t R, const int32_t *seg_offsets, const int32_t *seg_adapter,
                       int64_t S, void *workspace, size_t workspace_bytes, void *stream);

/* Y [M,N] bf16 = dequantized W8A8 output + T B_pack^T, with T from
 * sq_lora_shrink_raw on the same workspace, M and R (R == 0: plain W8A8).
 * Xq, x_scale, Wq, w_scale as for sq_linear_lora; the fused tensor-core GEMM
 * for every M.  Errors as sq_linear_lora. */
int sq_linear_lora_from_t(const int8_t *Xq, const float *x_scale, const int8_t *Wq,
                          const float *w_scale, int64_t M, int64_t N, int64_t K,
                          const uint16_t *B_pack, int64_t R, uint16_t *Y, const void *workspace,
                          size_t workspace_bytes, void *stream);

/* Test entry: delta [M,N] f32 = T B_pack^T alone, as sq_linear_lora_from_t
 * adds it (Xq and K only shape the call). */
int sq_lora_delta_from_t(const int8_t *Xq, int64_t M, int64_t N, int64_t K,
                         const uint16_t *B_pack, int64_t R, float *delta, const void *workspace,
                         size_t workspace_bytes, void *stream);

#ifdef __cplusplus
}
#endif
#endif /* SQ_W8A8_H */
