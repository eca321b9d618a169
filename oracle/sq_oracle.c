/*
 * CPU oracle for the SmoothQuant W8A8 linear layer with a per-request LoRA
 * delta.  TEST INFRASTRUCTURE ONLY: only the tests, the smoke check and the
 * CPU-baseline leg of the benchmark may load it.  It shares no code, header,
 * table or helper with the CUDA library and must never sit on the product
 * path.
 *
 * Plain, slow, obviously correct.  Floating point is done in fp64 and rounded
 * to fp32 only where the method stores an fp32 value; integer GEMMs are
 * accumulated in int64.  Rounding one fp64 result of a single +, -, *, / of
 * fp32 (or bf16) operands to fp32 gives exactly the IEEE fp32 result, because
 * 53 >= 2*24 + 2 (Figueroa, "When is double rounding innocuous?", 1995), so
 * every fp32 value produced here is the correctly rounded one.
 *
 * Sources (titles of the pages; sections named):
 *  [SQ]  "SmoothQuant" explainer (ozercemkelahmet.com/tools/smoothquant):
 *        How it works, Steps 2-7; "A short Python sketch"; "Calibration in
 *        practice"; "A worked example".
 *  [IS]  "[Feature]: LoRA support for W8A8 SmoothQuant" (TensorRT-LLM issue
 *        #12703), Pitch: the LoRA low-rank path runs in FP16/BF16 after the
 *        INT8 GEMM and its result is added to the dequantized output.
 *
 * Every function below is pinned by tests against values the pages print,
 * closed forms, invariants or brute force (tests/test_oracle_*.py).
 */
#include "sq_oracle.h"

#include <math.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

#define SQO_FLOOR ((double)1e-5f) /* clamp constant of the sketch ([SQ] sketch) */

/* ---- scalar helpers ---------------------------------------------------- */

static double bf16_value(uint16_t bits) {
  uint32_t u = (uint32_t)bits << 16;
  float f;
  memcpy(&f, &u, sizeof f);
  return (double)f;
}

static double x_value(const void *X, int dtype, int64_t idx) {
  if (dtype == SQO_F32) return (double)((const float *)X)[idx];
  return bf16_value(((const uint16_t *)X)[idx]);
}

/* Round an fp64 value to fp32, nearest-even (C conversion semantics). */
static float rn32(double v) { return (float)v; }

/* Round-half-to-even of a real value to an integer, written out. */
static double rne_int(double t) {
  double f = floor(t);
  double d = t - f; /* exact for |t| < 2^52 */
  if (d > 0.5) return f + 1.0;
  if (d < 0.5) return f;
  return (fmod(f, 2.0) == 0.0) ? f : f + 1.0;
}

/* clamp(round_half_even(t), -128, 127), the sketch's quantizer ([SQ] sketch). */
static int8_t quant_code(double t) {
  double r = rne_int(t);
  if (r < -128.0) r = -128.0;
  if (r > 127.0) r = 127.0;
  return (int8_t)r;
}

/* Round an fp32 value to bf16, nearest-even, by exact arithmetic on its
 * significand (8 significant bits for normal numbers, a fixed step of 2^-133
 * in the subnormal range). */
static uint16_t rn_bf16(float f) {
  double v = (double)f, r;
  if (v == 0.0 || isnan(v) || isinf(v)) {
    uint32_t u;
    memcpy(&u, &f, sizeof u);
    return (uint16_t)(u >> 16);
  }
  if (fabs(v) < ldexp(1.0, -126)) {
    r = ldexp(rne_int(ldexp(v, 133)), -133);
  } else {
    int e;
    double m = frexp(v, &e);              /* v = m * 2^e, 0.5 <= |m| < 1 */
    r = ldexp(rne_int(ldexp(m, 8)), e - 8); /* keep 8 significant bits */
  }
  float rf = (float)r; /* exact: r has at most 8 significant bits */
  uint32_t u;
  memcpy(&u, &rf, sizeof u);
  return (uint16_t)(u >> 16);
}

int sqo_num_threads(void) {
#ifdef _OPENMP
  return omp_get_max_threads();
#else
  return 1;
#endif
}

uint16_t sqo_round_bf16(float f) { return rn_bf16(f); }

/* ---- [SQ] Step 4 / "Calibration in practice": running per-channel max |X| */
void sqo_act_absmax_update(const void *X, int dtype, int64_t M, int64_t K,
                           float *act_absmax) {
  for (int64_t j = 0; j < K; ++j) {
    double m = act_absmax[j];
    for (int64_t i = 0; i < M; ++i) {
      double v = fabs(x_value(X, dtype, i * K + j));
      if (v > m) m = v;
    }
    act_absmax[j] = (float)m; /* exact: m is one of the inputs */
  }
}

/* ---- [SQ] sketch: w_max = |W|.max over output channels, per input channel */
void sqo_weight_absmax(const uint16_t *W, int64_t N, int64_t K, float *w_absmax) {
  for (int64_t j = 0; j < K; ++j) {
    double m = 0.0;
    for (int64_t n = 0; n < N; ++n) {
      double v = fabs(bf16_value(W[n * K + j]));
      if (v > m) m = v;
    }
    w_absmax[j] = (float)m;
  }
}

/* ---- [SQ] Step 3 and sketch:
 *   s_j = max( max(a_j,1e-5)^alpha / max(w_j,1e-5)^(1-alpha), 1e-5 )
 * in fp64 pow, rounded once to fp32. */
void sqo_compute_smoothing(const float *act_absmax, const float *w_absmax,
                           int64_t K, float alpha, float *s) {
  double al = (double)alpha;
  double be = 1.0 - al;
  for (int64_t j = 0; j < K; ++j) {
    double a = fmax((double)act_absmax[j], SQO_FLOOR);
    double w = fmax((double)w_absmax[j], SQO_FLOOR);
    double v = pow(a, al) / pow(w, be);
    s[j] = rn32(fmax(v, SQO_FLOOR));
  }
}

/* ---- [SQ] Steps 5-6 and sketch: fold diag(s) into W along the input
 * channels, then per-output-channel absmax INT8:
 *   W'[n,k] = fp32(W[n,k]*s_k); w_scale_n = fp32(max_k|W'[n,k]| / 127);
 *   Wq[n,k] = clamp(rne(fp32(W'[n,k] / w_scale_n)), -128, 127).
 * An all-zero output channel gets scale 0 and codes 0. */
void sqo_quantize_weight(const uint16_t *W, const float *s, int64_t N, int64_t K,
                         int8_t *Wq, float *w_scale) {
#pragma omp parallel for schedule(static)
  for (int64_t n = 0; n < N; ++n) {
    double amax = 0.0;
    for (int64_t k = 0; k < K; ++k) {
      double wp = (double)rn32(bf16_value(W[n * K + k]) * (double)s[k]);
      if (fabs(wp) > amax) amax = fabs(wp);
    }
    float sc = rn32(amax / 127.0);
    w_scale[n] = sc;
    for (int64_t k = 0; k < K; ++k) {
      double wp = (double)rn32(bf16_value(W[n * K + k]) * (double)s[k]);
      Wq[n * K + k] = (sc == 0.0f) ? 0 : quant_code((double)rn32(wp / (double)sc));
    }
  }
}

/* ---- [SQ] Steps 2, 5, 6 and sketch: divide each activation channel by s_j,
 * then per-token absmax INT8 (dynamic scales):
 *   xt[i,j] = fp32(X[i,j] / s_j); x_scale_i = fp32(max_j|xt[i,j]| / 127);
 *   Xq[i,j] = clamp(rne(fp32(xt[i,j] / x_scale_i)), -128, 127).
 * An all-zero token gets scale 0 and codes 0. */
void sqo_quant_act(const void *X, int dtype, const float *s, int64_t M, int64_t K,
                   int8_t *Xq, float *x_scale) {
#pragma omp parallel for schedule(static)
  for (int64_t i = 0; i < M; ++i) {
    double amax = 0.0;
    for (int64_t j = 0; j < K; ++j) {
      double xt = (double)rn32(x_value(X, dtype, i * K + j) / (double)s[j]);
      if (fabs(xt) > amax) amax = fabs(xt);
    }
    float sc = rn32(amax / 127.0);
    x_scale[i] = sc;
    for (int64_t j = 0; j < K; ++j) {
      double xt = (double)rn32(x_value(X, dtype, i * K + j) / (double)s[j]);
      Xq[i * K + j] = (sc == 0.0f) ? 0 : quant_code((double)rn32(xt / (double)sc));
    }
  }
}

/* ---- [SQ] Step 6, per-tensor static level ------------------------------
 * One activation scale for every token, fixed offline from the calibration
 * maxima of the smoothed activation ("Calibration in practice": static
 * scales are the faster, riskier choice):
 *   scale = RN32( max_j RN32(a_j / s_j) / 127 ).                           */
float sqo_static_act_scale(const float *act_absmax, const float *s, int64_t K) {
  double m = 0.0;
  for (int64_t j = 0; j < K; ++j) {
    double v = fabs((double)rn32((double)act_absmax[j] / (double)s[j]));
    if (v > m) m = v;
  }
  return rn32(m / 127.0);
}

/*   xt = RN32(x / s_j);  Xq = clamp(RNE(RN32(xt / scale)), -128, 127);
 *   x_scale_i = scale for every token.
 * Returns how many codes the clamp changed (values the calibrated range does
 * not cover).  scale == 0: every code is 0 and every nonzero xt counts. */
int64_t sqo_quant_act_static(const void *X, int dtype, const float *s, float scale, int64_t M,
                             int64_t K, int8_t *Xq, float *x_scale) {
  int64_t clipped = 0;
#pragma omp parallel for schedule(static) reduction(+ : clipped)
  for (int64_t i = 0; i < M; ++i) {
    x_scale[i] = scale;
    for (int64_t j = 0; j < K; ++j) {
      double xt = (double)rn32(x_value(X, dtype, i * K + j) / (double)s[j]);
      if (scale == 0.0f) {
        Xq[i * K + j] = 0;
        if (xt != 0.0) ++clipped;
        continue;
      }
      double r = rne_int((double)rn32(xt / (double)scale));
      if (r < -128.0 || r > 127.0) ++clipped;
      Xq[i * K + j] = quant_code(r);
    }
  }
  return clipped;
}

/* ---- [SQ] Step 5: the inverse scale folded into the normalization weight -
 * "The inverse scale can be folded into the normalization layer's weights":
 *   gamma_s[j] = RN32(gamma[j] / s_j)                                       */
void sqo_fold_norm_weight(const float *gamma, const float *s, int64_t K, float *gamma_s) {
  for (int64_t j = 0; j < K; ++j) gamma_s[j] = rn32((double)gamma[j] / (double)s[j]);
}

/* RMS normalization with the folded weight, then Step 6 per token:
 *   r_i  = RN32( 1 / sqrt( (sum_j h_ij^2) / K + eps ) )   (fp64 inside)
 *   xt   = RN32( RN32(h_ij * r_i) * gamma_s[j] )
 *   x_scale_i = RN32(max_j |xt| / 127),  Xq = clamp(RNE(RN32(xt / x_scale_i)))
 * H [M,K] bf16.  The sum of squares is defined as the exact sum of the
 * (exact) squares of the bf16 values, rounded once to fp64, so it does not
 * depend on any order of summation (a row's squares can span far more than
 * the 53 bits of an fp64 sum); the square root and the division are the
 * correctly rounded fp64 operations. */

/* Sum of the squares of K bf16 values, exact, rounded once to fp64 (nearest,
 * ties to even).  A finite bf16 value with exponent field E and fraction field
 * F is m * 2^(max(E,1) - 134) with the integer significand m = F (E == 0) or
 * 128 + F, so its square is the integer m^2 (< 2^16) times 2^(2*max(E,1) - 268):
 * the integer m^2 shifted left by 2*max(E,1) - 2 bits in a fixed-point number
 * whose unit is 2^-266.  That number is kept in 32-bit digits (the largest
 * square ends below bit 522, and up to 2^20 squares add at most 20 bits), then
 * its top 53 bits are rounded using the next bit and whether any bit below it
 * is set.  A row holding an infinity or a NaN gives the fp64 sum of its
 * squares (inf or NaN). */
#define SQO_SS_DIGITS 18
double sqo_sum_squares_bf16(const uint16_t *h, int64_t K) {
  uint32_t d[SQO_SS_DIGITS];
  memset(d, 0, sizeof d);
  for (int64_t j = 0; j < K; ++j) {
    unsigned E = (h[j] >> 7) & 0xFFu, F = h[j] & 0x7Fu;
    if (E == 0xFFu) { /* not finite */
      double s = 0.0;
      for (int64_t t = 0; t < K; ++t) s += bf16_value(h[t]) * bf16_value(h[t]);
      return s;
    }
    uint64_t m = (E == 0) ? F : (128u + F);
    if (m == 0) continue;
    unsigned pos = 2u * (E == 0 ? 1u : E) - 2u; /* bit position of m^2 */
    /* add (m^2 << pos) digit by digit with carry */
    uint64_t carry = (m * m) << (pos % 32u); /* < 2^48 */
    for (unsigned k = pos / 32u; carry != 0 && k < SQO_SS_DIGITS; ++k) {
      carry += d[k];
      d[k] = (uint32_t)carry;
      carry >>= 32;
    }
  }
  int top = -1; /* highest set bit */
  for (int k = SQO_SS_DIGITS - 1; k >= 0 && top < 0; --k)
    for (int b = 31; b >= 0; --b)
      if ((d[k] >> b) & 1u) { top = 32 * k + b; break; }
  if (top < 0) return 0.0;
#define SQO_BIT(p) ((p) >= 0 ? (int)((d[(p) / 32] >> ((p) % 32)) & 1u) : 0)
  /* the 53 bits from `top` down, as an integer */
  uint64_t sig = 0;
  for (int p = top; p > top - 53; --p) sig = (sig << 1) | (uint64_t)SQO_BIT(p);
  int lsb = top - 52; /* weight 2^(lsb - 266) of the last kept bit */
  if (lsb > 0) {
    int round = SQO_BIT(lsb - 1), sticky = 0;
    for (int p = lsb - 2; p >= 0; --p) sticky |= SQO_BIT(p);
    if (round && (sticky || (sig & 1u))) sig += 1; /* may reach 2^53: still exact */
  }
#undef SQO_BIT
  return ldexp((double)sig, lsb - 266);
}

void sqo_rmsnorm_quant_act(const uint16_t *H, const float *gamma_s, float eps, int64_t M,
                           int64_t K, int8_t *Xq, float *x_scale) {
#pragma omp parallel for schedule(static)
  for (int64_t i = 0; i < M; ++i) {
    /* the sum of squares is the exact one, rounded once to fp64 */
    double ss = sqo_sum_squares_bf16(H + i * K, K);
    float r = rn32(1.0 / sqrt(ss / (double)K + (double)eps));
    double amax = 0.0;
    for (int64_t j = 0; j < K; ++j) {
      double xt = (double)rn32((double)rn32(bf16_value(H[i * K + j]) * (double)r) * (double)gamma_s[j]);
      if (fabs(xt) > amax) amax = fabs(xt);
    }
    float sc = rn32(amax / 127.0);
    x_scale[i] = sc;
    for (int64_t j = 0; j < K; ++j) {
      double xt = (double)rn32((double)rn32(bf16_value(H[i * K + j]) * (double)r) * (double)gamma_s[j]);
      Xq[i * K + j] = (sc == 0.0f) ? 0 : quant_code((double)rn32(xt / (double)sc));
    }
  }
}

/* ---- LoRA operands with the smoothing and the scaling folded in ---------
 * The LoRA path consumes the dequantized activations Xq*x_scale, which
 * approximate X/s ([SQ] Step 2); un-smoothing them is folded into A, the same
 * "fold the scale into the next operand" move as [SQ] Step 5:
 *   A_s[j,k] = bf16(fp32(A[j,k]*s_k)),  B_s[n,j] = bf16(fp32(B[n,j]*scale)),
 *   scale = fp32(lora_alpha / r). */
void sqo_prepare_lora(const uint16_t *A, const uint16_t *B, const float *s,
                      int64_t r, int64_t K, int64_t N, float lora_alpha,
                      uint16_t *A_s, uint16_t *B_s) {
  float scale = rn32((double)lora_alpha / (double)r);
  /* s == NULL: the raw-input reading, A is kept as given (no smoothing fold) */
  for (int64_t j = 0; j < r; ++j)
    for (int64_t k = 0; k < K; ++k)
      A_s[j * K + k] = s ? rn_bf16(rn32(bf16_value(A[j * K + k]) * (double)s[k]))
                         : A[j * K + k];
  for (int64_t n = 0; n < N; ++n)
    for (int64_t j = 0; j < r; ++j)
      B_s[n * r + j] = rn_bf16(rn32(bf16_value(B[n * r + j]) * (double)scale));
}

/* ---- [SQ] Step 7: INT8 x INT8 products summed exactly (int64) ----------- */
void sqo_gemm_rows(const int8_t *Xq, const int8_t *Wq, int64_t M, int64_t N,
                   int64_t K, const int64_t *rows, int64_t nrows, int64_t *acc) {
  (void)M;
#pragma omp parallel for collapse(2) schedule(static)
  for (int64_t t = 0; t < nrows; ++t)
    for (int64_t n = 0; n < N; ++n) {
      const int8_t *x = Xq + rows[t] * K;
      const int8_t *w = Wq + n * K;
      int64_t sum = 0;
      for (int64_t k = 0; k < K; ++k) sum += (int64_t)x[k] * (int64_t)w[k];
      acc[t * N + n] = sum;
    }
}

void sqo_gemm_pairs(const int8_t *Xq, const int8_t *Wq, int64_t K,
                    const int64_t *rows, const int64_t *cols, int64_t npairs,
                    int64_t *acc) {
#pragma omp parallel for schedule(static)
  for (int64_t t = 0; t < npairs; ++t) {
    const int8_t *x = Xq + rows[t] * K;
    const int8_t *w = Wq + cols[t] * K;
    int64_t sum = 0;
    for (int64_t k = 0; k < K; ++k) sum += (int64_t)x[k] * (int64_t)w[k];
    acc[t] = sum;
  }
}

/* Adapter of token i: the adapter of the first segment s with
 * seg_offsets[s] <= i < seg_offsets[s+1]; -1 (none) when no segment holds
 * the token or its index is outside [0, n_adapters). */
int sqo_token_adapter(const int32_t *seg_offsets, const int32_t *seg_adapter,
                      int64_t S, int n_adapters, int64_t i) {
  for (int64_t s = 0; s < S; ++s) {
    if (seg_offsets[s] <= i && i < seg_offsets[s + 1]) {
      int a = seg_adapter[s];
      return (a >= 0 && a < n_adapters) ? a : -1;
    }
  }
  return -1;
}

/* ---- [SQ] Step 7 dequant + [IS] LoRA delta, for selected tokens ----------
 *   base[i,n]  = acc[i,n] * x_scale_i * w_scale_n
 *   xhat[i,k]  = Xq[i,k] * x_scale_i
 *   T[i,j]     = sum_k xhat[i,k] * A_s[a][j,k]
 *   delta[i,n] = sum_j T[i,j] * B_s[a][n,j]        (a = adapter of token i)
 *   Y[i,n]     = base[i,n] + delta[i,n]            (delta = 0 when a = -1)
 * all in fp64.  Any of Y / delta / acc may be NULL. */
void sqo_linear_lora_rows(const int8_t *Xq, const float *x_scale, const int8_t *Wq,
                          const float *w_scale, int64_t M, int64_t N, int64_t K,
                          int n_adapters, const uint16_t *const *A_s,
                          const uint16_t *const *B_s, const int64_t *ranks,
                          const int32_t *seg_offsets, const int32_t *seg_adapter,
                          int64_t S, const int64_t *rows, int64_t nrows, double *Y,
                          double *delta, int64_t *acc) {
  (void)M;
#pragma omp parallel for schedule(dynamic, 1)
  for (int64_t t = 0; t < nrows; ++t) {
    int64_t i = rows[t];
    int a = sqo_token_adapter(seg_offsets, seg_adapter, S, n_adapters, i);
    double xs = (double)x_scale[i];
    double *T = NULL;
    int64_t r = 0;
    if (a >= 0) {
      r = ranks[a];
      T = (double *)calloc((size_t)(r > 0 ? r : 1), sizeof(double));
      for (int64_t j = 0; j < r; ++j) {
        double sum = 0.0;
        for (int64_t k = 0; k < K; ++k)
          sum += ((double)Xq[i * K + k] * xs) * bf16_value(A_s[a][j * K + k]);
        T[j] = sum;
      }
    }
    for (int64_t n = 0; n < N; ++n) {
      int64_t sum = 0;
      for (int64_t k = 0; k < K; ++k) sum += (int64_t)Xq[i * K + k] * (int64_t)Wq[n * K + k];
      double base = (double)sum * xs * (double)w_scale[n];
      double d = 0.0;
      for (int64_t j = 0; j < r; ++j) d += T[j] * bf16_value(B_s[a][n * r + j]);
      if (acc) acc[t * N + n] = sum;
      if (delta) delta[t * N + n] = d;
      if (Y) Y[t * N + n] = base + d;
    }
    free(T);
  }
}

/* ---- [IS] Pitch, raw-input reading: the LoRA path in BF16 on the layer's
 * own (unquantized) activations, added to the dequantized INT8 output -----
 *   base[i,n]  = acc[i,n] * x_scale_i * w_scale_n           (as above)
 *   T[i,j]     = sum_k X[i,k] * A[a][j,k]                   (X bf16, A as given)
 *   delta[i,n] = sum_j T[i,j] * B_s[a][n,j]
 *   Y[i,n]     = base[i,n] + delta[i,n]
 * all in fp64.  X must be bf16 (dtype SQO_BF16).  Any of Y / delta may be NULL. */
void sqo_linear_lora_raw_rows(const uint16_t *X, const int8_t *Xq, const float *x_scale,
                              const int8_t *Wq, const float *w_scale, int64_t M, int64_t N,
                              int64_t K, int n_adapters, const uint16_t *const *A,
                              const uint16_t *const *B_s, const int64_t *ranks,
                              const int32_t *seg_offsets, const int32_t *seg_adapter,
                              int64_t S, const int64_t *rows, int64_t nrows, double *Y,
                              double *delta) {
  (void)M;
#pragma omp parallel for schedule(dynamic, 1)
  for (int64_t t = 0; t < nrows; ++t) {
    int64_t i = rows[t];
    int a = sqo_token_adapter(seg_offsets, seg_adapter, S, n_adapters, i);
    double xs = (double)x_scale[i];
    double *T = NULL;
    int64_t r = 0;
    if (a >= 0) {
      r = ranks[a];
      T = (double *)calloc((size_t)(r > 0 ? r : 1), sizeof(double));
      for (int64_t j = 0; j < r; ++j) {
        double sum = 0.0;
        for (int64_t k = 0; k < K; ++k)
          sum += bf16_value(X[i * K + k]) * bf16_value(A[a][j * K + k]);
        T[j] = sum;
      }
    }
    for (int64_t n = 0; n < N; ++n) {
      double d = 0.0;
      for (int64_t j = 0; j < r; ++j) d += T[j] * bf16_value(B_s[a][n * r + j]);
      if (delta) delta[t * N + n] = d;
      if (Y) {
        int64_t sum = 0;
        for (int64_t k = 0; k < K; ++k) sum += (int64_t)Xq[i * K + k] * (int64_t)Wq[n * K + k];
        Y[t * N + n] = (double)sum * xs * (double)w_scale[n] + d;
      }
    }
    free(T);
  }
}

/* ---- Unquantized reference: the layer the method approximates -----------
 *   Y[i,n] = sum_k X[i,k] W[n,k] + (lora_alpha/r) * sum_j (sum_k X[i,k] A[j,k]) B[n,j]
 * in fp64 from the original X, W, A, B (no smoothing, no rounding). */
void sqo_reference_rows(const void *X, int dtype, const uint16_t *W, int64_t M,
                        int64_t N, int64_t K, int n_adapters,
                        const uint16_t *const *A, const uint16_t *const *B,
                        const int64_t *ranks, const double *lora_alpha,
                        const int32_t *seg_offsets, const int32_t *seg_adapter,
                        int64_t S, const int64_t *rows, int64_t nrows, double *Y) {
  (void)M;
#pragma omp parallel for schedule(dynamic, 1)
  for (int64_t t = 0; t < nrows; ++t) {
    int64_t i = rows[t];
    int a = sqo_token_adapter(seg_offsets, seg_adapter, S, n_adapters, i);
    int64_t r = (a >= 0) ? ranks[a] : 0;
    double *T = (double *)calloc((size_t)(r > 0 ? r : 1), sizeof(double));
    for (int64_t j = 0; j < r; ++j) {
      double sum = 0.0;
      for (int64_t k = 0; k < K; ++k)
        sum += x_value(X, dtype, i * K + k) * bf16_value(A[a][j * K + k]);
      T[j] = sum;
    }
    for (int64_t n = 0; n < N; ++n) {
      double sum = 0.0;
      for (int64_t k = 0; k < K; ++k)
        sum += x_value(X, dtype, i * K + k) * bf16_value(W[n * K + k]);
      double d = 0.0;
      for (int64_t j = 0; j < r; ++j) d += T[j] * bf16_value(B[a][n * r + j]);
      Y[t * N + n] = sum + (r > 0 ? lora_alpha[a] / (double)r : 0.0) * d;
    }
    free(T);
  }
}

/* ---- [SQ] Step 2: the equivalent transform in exact-as-possible fp64 -----
 *   Y[i,n] = sum_k (X[i,k] / s_k) * (s_k * W[n,k])
 * used to check that smoothing alone leaves the layer unchanged. */
void sqo_smoothed_product_rows(const void *X, int dtype, const uint16_t *W,
                               const float *s, int64_t N, int64_t K,
                               const int64_t *rows, int64_t nrows, double *Y) {
#pragma omp parallel for collapse(2) schedule(static)
  for (int64_t t = 0; t < nrows; ++t)
    for (int64_t n = 0; n < N; ++n) {
      double sum = 0.0;
      for (int64_t k = 0; k < K; ++k) {
        double sk = (double)s[k];
        sum += (x_value(X, dtype, rows[t] * K + k) / sk) * (sk * bf16_value(W[n * K + k]));
      }
      Y[t * N + n] = sum;
    }
}
