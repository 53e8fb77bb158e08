/*
 * sq_oracle.c -- plain, slow CPU oracle for the SmoothQuant W8A8 smoothed
 * linear layer.
 *
 * TEST INFRASTRUCTURE ONLY.  Only the test suite, the smoke check and the
 * benchmark's CPU-baseline leg may load this file.  It shares no code,
 * header, table or helper with the CUDA library; neither side includes or
 * links the other.  Every step is a single-threaded loop written in the
 * order the method states it, with no blocking or fusion.
 *
 * Source of the method: "SmoothQuant (activation smoothing quantization)",
 * jisaku.com glossary page (2023):
 *   - section "Why activation quantization is hard": INT8 holds -128..127
 *     and a token is scaled so that its largest magnitude maps to 127;
 *   - section "The mathematics of the smoothing transformation":
 *     Y = X W = (X diag(s)^-1)(diag(s) W) = X~ W~;
 *   - section "Hyper-parameter alpha (migration strength)":
 *     s_j = max|X_j|^alpha / max|W_j|^(1-alpha), alpha = 0.5 default;
 *   - usage example: get_act_scales -> smooth_lm(alpha) -> quantize_model.
 *
 * Readings where the page is silent (all listed in the design notes):
 *   - arithmetic is IEEE fp32 with round-to-nearest-even everywhere; build
 *     with -ffp-contract=off so no multiply is fused into an add;
 *   - channel maxima are floored at 1e-5 before s is formed;
 *   - s^alpha is evaluated with sqrt for alpha in {0, .25, .5, .75, 1}
 *     and with double pow otherwise;
 *   - X~ = X * (1/s): the stored reciprocal is multiplied in;
 *   - activations are quantized per token (dynamic), weights per output
 *     channel: for a row v with absmax m, delta = m/127 and
 *     q = clamp(rne(v / delta), -127, 127) with an IEEE division; an
 *     all-zero row gives delta = 0 and q = 0;
 *   - the int32 product is dequantized as ((float)acc * dx_t) * dw_n and
 *     then rounded to the output type.
 */
#include <math.h>
#include <stdint.h>
#include <string.h>

#define OR_LAYOUT_KN 0 /* W[K][N]: Y = X W as the page writes it      */
#define OR_LAYOUT_NK 1 /* W[N][K]: output-major, as torch's nn.Linear */

/* Element W_jn (input channel j, output channel n) for either layout. */
static float w_at(const float *w, int layout, int64_t K, int64_t N,
                  int64_t j, int64_t n) {
  return layout == OR_LAYOUT_KN ? w[j * N + n] : w[n * K + j];
}

/* ---- quantizer for one value --------------------------------------------
 * v / delta with an IEEE division, rounded half to even (rintf under the
 * default rounding mode), then clamped to the symmetric range [-127, 127].
 * delta > 0 is the scale of the value's row (absmax / 127). */
int8_t or_quantize_value(float v, float delta) {
  float t = v / delta;
  float q = rintf(t);
  if (q > 127.0f) q = 127.0f;
  if (q < -127.0f) q = -127.0f;
  return (int8_t)q;
}

/* ---- step 1: calibration ------------------------------------------------
 * amax_j <- max(amax_j, max_t |x_tj|) over the tokens of one chunk; a
 * running maximum across calls (get_act_scales in the usage example). */
void or_calib_absmax(const float *x, int64_t T, int64_t K, float *amax) {
  for (int64_t t = 0; t < T; ++t)
    for (int64_t j = 0; j < K; ++j) {
      float v = fabsf(x[t * K + j]);
      if (v > amax[j]) amax[j] = v;
    }
}

/* ---- step 2: weight maximum per input channel ---------------------------
 * w_j = max_n |W_jn|: the max|W_j| of the alpha formula. */
void or_weight_absmax(const float *w, int layout, int64_t K, int64_t N,
                      float *wmax) {
  for (int64_t j = 0; j < K; ++j) {
    float m = 0.0f;
    for (int64_t n = 0; n < N; ++n) {
      float v = fabsf(w_at(w, layout, K, N, j, n));
      if (v > m) m = v;
    }
    wmax[j] = m;
  }
}

/* ---- step 3: smoothing factor -------------------------------------------
 * s_j = max|X_j|^alpha / max|W_j|^(1-alpha), inv_s_j = 1/s_j. */
void or_smooth_factor(const float *amax, const float *wmax, int64_t K,
                      float alpha, float *s, float *inv_s) {
  for (int64_t j = 0; j < K; ++j) {
    float a = amax[j] > 1e-5f ? amax[j] : 1e-5f;
    float w = wmax[j] > 1e-5f ? wmax[j] : 1e-5f;
    float sj;
    if (alpha == 1.0f) {
      sj = a; /* a^1 / w^0 */
    } else if (alpha == 0.0f) {
      sj = 1.0f / w; /* a^0 / w^1 */
    } else if (alpha == 0.5f) {
      sj = sqrtf(a) / sqrtf(w);
    } else if (alpha == 0.25f) {
      float a14 = sqrtf(sqrtf(a));
      float w34 = sqrtf(w) * sqrtf(sqrtf(w));
      sj = a14 / w34;
    } else if (alpha == 0.75f) {
      float a34 = sqrtf(a) * sqrtf(sqrtf(a));
      float w14 = sqrtf(sqrtf(w));
      sj = a34 / w14;
    } else {
      double num = pow((double)a, (double)alpha);
      double den = pow((double)w, 1.0 - (double)alpha);
      sj = (float)(num / den);
    }
    s[j] = sj;
    inv_s[j] = 1.0f / sj;
  }
}

/* ---- step 4: weight fold W~ = diag(s) W ---------------------------------
 * Output is W~ in W's own layout. */
void or_smooth_weight(const float *w, int layout, int64_t K, int64_t N,
                      const float *s, float *wt) {
  for (int64_t j = 0; j < K; ++j)
    for (int64_t n = 0; n < N; ++n) {
      float v = s[j] * w_at(w, layout, K, N, j, n);
      if (layout == OR_LAYOUT_KN)
        wt[j * N + n] = v;
      else
        wt[n * K + j] = v;
    }
}

/* ---- step 5: per-output-channel weight quantization ---------------------
 * For output channel n: m_n = max_j |W~_jn|, dw_n = m_n/127,
 * Wq[n][j] = clamp(rne(W~_jn / dw_n)).  Wq is stored [N][K]
 * (K contiguous) whatever W's layout. */
void or_smooth_quant_weight(const float *w, int layout, int64_t K, int64_t N,
                            const float *s, int8_t *wq, float *dw) {
  for (int64_t n = 0; n < N; ++n) {
    float m = 0.0f;
    for (int64_t j = 0; j < K; ++j) {
      float v = fabsf(s[j] * w_at(w, layout, K, N, j, n));
      if (v > m) m = v;
    }
    if (m == 0.0f) {
      dw[n] = 0.0f;
      for (int64_t j = 0; j < K; ++j) wq[n * K + j] = 0;
      continue;
    }
    dw[n] = m / 127.0f;
    for (int64_t j = 0; j < K; ++j)
      wq[n * K + j] = or_quantize_value(s[j] * w_at(w, layout, K, N, j, n), dw[n]);
  }
}

/* ---- step 6: activation smoothing X~ = X diag(s)^-1 ---------------------- */
void or_smooth_act(const float *x, int64_t M, int64_t K, const float *inv_s,
                   float *xt) {
  for (int64_t t = 0; t < M; ++t)
    for (int64_t j = 0; j < K; ++j) xt[t * K + j] = x[t * K + j] * inv_s[j];
}

/* ---- step 7: per-token dynamic activation quantization ------------------
 * For token t: m_t = max_j |X~_tj|, dx_t = m_t/127,
 * Xq[t][j] = clamp(rne(X~_tj / dx_t)). */
void or_quant_act(const float *x, int64_t M, int64_t K, const float *inv_s,
                  int8_t *xq, float *dx) {
  for (int64_t t = 0; t < M; ++t) {
    float m = 0.0f;
    for (int64_t j = 0; j < K; ++j) {
      float v = fabsf(x[t * K + j] * inv_s[j]);
      if (v > m) m = v;
    }
    if (m == 0.0f) {
      dx[t] = 0.0f;
      for (int64_t j = 0; j < K; ++j) xq[t * K + j] = 0;
      continue;
    }
    dx[t] = m / 127.0f;
    for (int64_t j = 0; j < K; ++j)
      xq[t * K + j] = or_quantize_value(x[t * K + j] * inv_s[j], dx[t]);
  }
}

/* ---- step 8: INT8 x INT8 -> int32 matrix product ------------------------
 * acc[t][n] = sum_j Xq[t][j] * Wq[n][j]: exact integer arithmetic. */
void or_gemm_i8(const int8_t *xq, const int8_t *wq, int64_t M, int64_t N,
                int64_t K, int32_t *acc) {
  for (int64_t t = 0; t < M; ++t)
    for (int64_t n = 0; n < N; ++n) {
      int32_t sum = 0;
      for (int64_t j = 0; j < K; ++j)
        sum += (int32_t)xq[t * K + j] * (int32_t)wq[n * K + j];
      acc[t * N + n] = sum;
    }
}

/* ---- step 9: dequantization ---------------------------------------------
 * y[t][n] = ((float)acc[t][n] * dx_t) * dw_n, fp32. */
void or_dequant(const int32_t *acc, const float *dx, const float *dw,
                int64_t M, int64_t N, float *y) {
  for (int64_t t = 0; t < M; ++t)
    for (int64_t n = 0; n < N; ++n) {
      float a = (float)acc[t * N + n];
      y[t * N + n] = (a * dx[t]) * dw[n];
    }
}

/* ---- output rounding ----------------------------------------------------
 * fp32 -> bfloat16, round to nearest even on the dropped 16 bits
 * (NaN kept quiet). */
void or_round_bf16(const float *y, int64_t count, uint16_t *out) {
  for (int64_t i = 0; i < count; ++i) {
    uint32_t u;
    memcpy(&u, &y[i], 4);
    if ((u & 0x7fffffffu) > 0x7f800000u) {
      out[i] = (uint16_t)((u >> 16) | 0x40u);
      continue;
    }
    uint32_t lsb = (u >> 16) & 1u;
    u += 0x7fffu + lsb;
    out[i] = (uint16_t)(u >> 16);
  }
}

/* fp32 -> IEEE binary16 with the compiler's round-to-nearest-even cast. */
void or_round_f16(const float *y, int64_t count, uint16_t *out) {
  for (int64_t i = 0; i < count; ++i) {
    _Float16 h = (_Float16)y[i];
    memcpy(&out[i], &h, 2);
  }
}

/* ---- upstream producer: RMSNorm, smoothing and per-token quantization ----
 * The usage example's smooth_lm(alpha) folds diag(s)^-1 into the layer that
 * produces X -- in transformer blocks an RMS normalisation -- offline, the
 * same way diag(s) is folded into W.  The norm's weight becomes
 *   gs_j = gamma_j * inv_s_j                     (fp32, once per layer)
 * and for token t the producer computes
 *   ss_t = sum_j x_tj^2            (double precision, sequential)
 *   r_t  = (float)(1 / sqrt(ss_t / K + eps))   (double, rounded once)
 *   v_tj = (x_tj * r_t) * gs_j                 (fp32, in that order)
 * then quantizes v per token as in or_quant_act. */
void or_fold_norm_weight(const float *gamma, const float *inv_s, int64_t K, float *gs) {
  for (int64_t j = 0; j < K; ++j) gs[j] = gamma[j] * inv_s[j];
}

void or_rmsnorm_quant_act(const float *x, int64_t M, int64_t K, const float *gs, float eps, int8_t *xq,
                          float *dx) {
  for (int64_t t = 0; t < M; ++t) {
    double ss = 0.0;
    for (int64_t j = 0; j < K; ++j) ss += (double)x[t * K + j] * (double)x[t * K + j];
    const float r = (float)(1.0 / sqrt(ss / (double)K + (double)eps));
    float m = 0.0f;
    for (int64_t j = 0; j < K; ++j) {
      float v = fabsf((x[t * K + j] * r) * gs[j]);
      if (v > m) m = v;
    }
    if (m == 0.0f) {
      dx[t] = 0.0f;
      for (int64_t j = 0; j < K; ++j) xq[t * K + j] = 0;
      continue;
    }
    dx[t] = m / 127.0f;
    for (int64_t j = 0; j < K; ++j) xq[t * K + j] = or_quantize_value((x[t * K + j] * r) * gs[j], dx[t]);
  }
}

/* Per-token normalisation factor r_t of or_rmsnorm_quant_act (exposed so
 * tests can see how close a product lies to a rounding boundary). */
void or_rmsnorm_factor(const float *x, int64_t M, int64_t K, float eps, float *r) {
  for (int64_t t = 0; t < M; ++t) {
    double ss = 0.0;
    for (int64_t j = 0; j < K; ++j) ss += (double)x[t * K + j] * (double)x[t * K + j];
    r[t] = (float)(1.0 / sqrt(ss / (double)K + (double)eps));
  }
}

/* ---- upstream producer: LayerNorm, smoothing and per-token quantization --
 * The same fold for a layer normalisation with weight gamma and bias beta
 * (the OPT models of the page's benchmarks use this form):
 *   gs_j = gamma_j * inv_s_j,  bs_j = beta_j * inv_s_j   (fp32, once per layer)
 * and for token t
 *   mu_t  = sum_j x_tj / K                     (double, sequential)
 *   var_t = sum_j (x_tj - mu_t)^2 / K          (double: each deviation and
 *                                               its square in double)
 *   r_t   = (float)(1 / sqrt(var_t + eps))     (double, rounded once)
 *   muf_t = (float)mu_t
 *   n_tj  = (x_tj - muf_t) * r_t                   (fp32, in that order)
 *   v_tj  = fma(n_tj, gs_j, bs_j)                  (the affine step of the
 *                                                   norm, rounded once)
 * then per-token quantization of v as in or_quant_act.  bs may be NULL (no
 * bias). */
static void or_layernorm_row_stats(const float *row, int64_t K, float eps, float *muf, float *r) {
  double sum = 0.0;
  for (int64_t j = 0; j < K; ++j) sum += (double)row[j];
  const double mu = sum / (double)K;
  double ss = 0.0;
  for (int64_t j = 0; j < K; ++j) {
    const double d = (double)row[j] - mu;
    ss += d * d;
  }
  *r = (float)(1.0 / sqrt(ss / (double)K + (double)eps));
  *muf = (float)mu;
}

void or_layernorm_stats(const float *x, int64_t M, int64_t K, float eps, float *mu, float *r) {
  for (int64_t t = 0; t < M; ++t) or_layernorm_row_stats(x + t * K, K, eps, &mu[t], &r[t]);
}

static float or_layernorm_value(float x, float muf, float r, float g, float b) {
  const float c = x - muf;
  const float n = c * r;
  return fmaf(n, g, b); /* the affine step n * g + b, rounded once */
}

/* The normalised, folded values v_tj of or_layernorm_quant_act before
 * quantization (exposed so tests can see how close v / delta lies to a
 * rounding boundary). */
void or_layernorm_values(const float *x, int64_t M, int64_t K, const float *gs, const float *bs, float eps,
                         float *v) {
  for (int64_t t = 0; t < M; ++t) {
    const float *row = x + t * K;
    float muf, r;
    or_layernorm_row_stats(row, K, eps, &muf, &r);
    for (int64_t j = 0; j < K; ++j) v[t * K + j] = or_layernorm_value(row[j], muf, r, gs[j], bs ? bs[j] : 0.0f);
  }
}

void or_layernorm_quant_act(const float *x, int64_t M, int64_t K, const float *gs, const float *bs, float eps,
                            int8_t *xq, float *dx) {
  for (int64_t t = 0; t < M; ++t) {
    const float *row = x + t * K;
    float muf, r;
    or_layernorm_row_stats(row, K, eps, &muf, &r);
    float m = 0.0f;
    for (int64_t j = 0; j < K; ++j) {
      float v = fabsf(or_layernorm_value(row[j], muf, r, gs[j], bs ? bs[j] : 0.0f));
      if (v > m) m = v;
    }
    if (m == 0.0f) {
      dx[t] = 0.0f;
      for (int64_t j = 0; j < K; ++j) xq[t * K + j] = 0;
      continue;
    }
    dx[t] = m / 127.0f;
    for (int64_t j = 0; j < K; ++j)
      xq[t * K + j] = or_quantize_value(or_layernorm_value(row[j], muf, r, gs[j], bs ? bs[j] : 0.0f), dx[t]);
  }
}

/* ---- static per-tensor activation scale --------------------------------
 * The page notes activations change per prompt, which is why the main path
 * quantizes per token at run time; the static alternative fixes one scale
 * from calibration.  After smoothing, channel j's calibrated maximum is
 * a_j * inv_s_j, so the tensor scale is delta = max_j(a_j * inv_s_j) / 127. */
float or_static_act_scale(const float *amax, const float *inv_s, int64_t K) {
  float m = 0.0f;
  for (int64_t j = 0; j < K; ++j) {
    float v = amax[j] * inv_s[j];
    if (v > m) m = v;
  }
  return m / 127.0f;
}

/* Static quantization with a fixed scale delta > 0: every smoothed value
 * is divided by delta and rounded; values beyond the calibrated range
 * saturate at +-127.  dx_t = delta for every token. */
void or_quant_act_static(const float *x, int64_t M, int64_t K, const float *inv_s, float delta,
                         int8_t *xq, float *dx) {
  for (int64_t t = 0; t < M; ++t) {
    dx[t] = delta;
    for (int64_t j = 0; j < K; ++j) xq[t * K + j] = or_quantize_value(x[t * K + j] * inv_s[j], delta);
  }
}

/* ---- FP8 (E4M3) variant --------------------------------------------------
 * The glossary page "Quantization Calibration GPTQ/AWQ/SmoothQuant 2026"
 * (jisaku.com glossary) lists FP8 SmoothQuant: the same smoothing with FP8
 * operands (its spec-comparison table: 8-bit weights, FP8 activations).
 * Readings: both operands in E4M3 -- the 8-bit float with 1 sign bit, 4
 * exponent bits of bias 7 and 3 mantissa bits, no infinities, the all-ones
 * exponent with mantissa 111 as NaN, largest finite value 448, subnormals
 * (m/8) * 2^-6 -- with the INT8 path's granularity: delta = m/448 per token
 * and per output channel, code = e4m3(v / delta) (IEEE division) rounded to
 * nearest, ties to the even code, saturating at +-448.  The product of two E4M3 values is
 * exact, and so is the sum over K in double: every product is a multiple of
 * 2^-18 below 448^2 < 2^18, so K <= 2^15 terms stay within 51 bits. */

/* Exact value of an E4M3 code. */
float or_e4m3_decode(uint8_t c) {
  const int e = (c >> 3) & 15, m = c & 7;
  if (e == 15 && m == 7) return NAN;
  const float mag = e == 0 ? ldexpf((float)m, -9) : ldexpf((float)(8 + m), e - 10);
  return (c & 0x80) ? -mag : mag;
}

/* The E4M3 code nearest to v (ties to the even code), +-448 beyond. */
uint8_t or_e4m3_encode(float v) {
  if (isnan(v)) return 0x7f;
  const uint8_t sign = signbit(v) ? 0x80 : 0x00;
  const float a = fabsf(v);
  if (a >= 448.0f) return sign | 0x7e;
  /* binade of a: a in [2^e, 2^(e+1)); below 2^-6 the spacing stays 2^-9 */
  int x;
  frexpf(a, &x);
  int e = a == 0.0f ? -6 : x - 1;
  if (e < -6) e = -6;
  const float quantum = ldexpf(1.0f, e - 3);
  const float q = rintf(a / quantum); /* a / 2^k is exact; rintf rounds half to even */
  const float r = q * quantum;         /* the rounded magnitude, <= 448 */
  if (r < ldexpf(1.0f, -6)) return sign | (uint8_t)(r / ldexpf(1.0f, -9)); /* subnormal or zero */
  frexpf(r, &x);
  const int er = x - 1;                                   /* r in [2^er, 2^(er+1)) */
  const int mant = (int)(r / ldexpf(1.0f, er - 3)) - 8;   /* 0..7 */
  return sign | (uint8_t)(((er + 7) << 3) | mant);
}

static uint8_t e4m3_quantize_value(float v, float delta) { return or_e4m3_encode(v / delta); }

/* Per-output-channel E4M3 weights: m_n = max_j |W~_jn|, dw_n = m_n/448,
 * Wq[n][j] = e4m3(W~_jn / dw_n), stored [N][K]. */
void or_smooth_quant_weight_e4m3(const float *w, int layout, int64_t K, int64_t N, const float *s, uint8_t *wq,
                                 float *dw) {
  for (int64_t n = 0; n < N; ++n) {
    float m = 0.0f;
    for (int64_t j = 0; j < K; ++j) {
      float v = fabsf(s[j] * w_at(w, layout, K, N, j, n));
      if (v > m) m = v;
    }
    if (m == 0.0f) {
      dw[n] = 0.0f;
      for (int64_t j = 0; j < K; ++j) wq[n * K + j] = 0;
      continue;
    }
    dw[n] = m / 448.0f;
    for (int64_t j = 0; j < K; ++j) wq[n * K + j] = e4m3_quantize_value(s[j] * w_at(w, layout, K, N, j, n), dw[n]);
  }
}

/* Per-token E4M3 activations: m_t = max_j |X~_tj|, dx_t = m_t/448,
 * Xq[t][j] = e4m3(X~_tj / dx_t). */
void or_quant_act_e4m3(const float *x, int64_t M, int64_t K, const float *inv_s, uint8_t *xq, float *dx) {
  for (int64_t t = 0; t < M; ++t) {
    float m = 0.0f;
    for (int64_t j = 0; j < K; ++j) {
      float v = fabsf(x[t * K + j] * inv_s[j]);
      if (v > m) m = v;
    }
    if (m == 0.0f) {
      dx[t] = 0.0f;
      for (int64_t j = 0; j < K; ++j) xq[t * K + j] = 0;
      continue;
    }
    dx[t] = m / 448.0f;
    for (int64_t j = 0; j < K; ++j) xq[t * K + j] = e4m3_quantize_value(x[t * K + j] * inv_s[j], dx[t]);
  }
}

/* acc[t][n] = sum_j e4m3(Xq[t][j]) * e4m3(Wq[n][j]), exact in double. */
void or_gemm_e4m3(const uint8_t *xq, const uint8_t *wq, int64_t M, int64_t N, int64_t K, double *acc) {
  for (int64_t t = 0; t < M; ++t)
    for (int64_t n = 0; n < N; ++n) {
      double sum = 0.0;
      for (int64_t j = 0; j < K; ++j)
        sum += (double)or_e4m3_decode(xq[t * K + j]) * (double)or_e4m3_decode(wq[n * K + j]);
      acc[t * N + n] = sum;
    }
}

/* y[t][n] = ((float)acc[t][n] * dx_t) * dw_n with an fp32 accumulator. */
void or_dequant_f32acc(const float *acc, const float *dx, const float *dw, int64_t M, int64_t N, float *y) {
  for (int64_t t = 0; t < M; ++t)
    for (int64_t n = 0; n < N; ++n) y[t * N + n] = (acc[t * N + n] * dx[t]) * dw[n];
}

/* ---- butterfly rotation (NEXT-4) -------------------------------------------
 * "ButterflyQuant" (lifetechia.com): a learnable orthogonal butterfly
 * transform of dimension n = 2^L built from Givens rotations, one per pair
 * per stage (angles theta[L][n/2]), applied to the activations before
 * quantization; the fixed Hadamard transform is the special case of every
 * angle pi/4.  Readings:
 *   - stage i (i = 0 .. L-1) pairs positions p and p + 2^i for every p
 *     whose bit i is clear -- the FFT butterfly the section describes.  The
 *     page's listing pairs neighbours (2j, 2j+1) at every stage without a
 *     permutation in between, which never mixes different pairs and so
 *     cannot give the O(n log n) transform containing Hadamard that its text
 *     names; the pairing above is the one that does.
 *   - the pair's index within stage i is j = ((p >> (i + 1)) << i) | (p mod 2^i)
 *     and its rotation, with c = cos(theta[i][j]), s = sin(theta[i][j]) as
 *     given fp32 tables, maps (a, b) = (v_p, v_{p+2^i}) to
 *       a' = c*a - s*b,   b' = s*a + c*b   (fp32, each product rounded)
 *   - a row of K channels is rotated block by block (K % n == 0), every
 *     n-block with the same angles;
 *   - with SmoothQuant, the rotation R acts on the smoothed activations and,
 *     as R is orthogonal, on the smoothed weights' K-vectors too:
 *     (R x~) . (R w~_n) = x~ . w~_n.  Both are then quantized as before. */
void or_butterfly_rotate(float *v, int64_t K, int64_t n, const float *c, const float *s) {
  int L = 0;
  while (((int64_t)1 << L) < n) ++L;
  for (int64_t b0 = 0; b0 < K; b0 += n) {
    float *blk = v + b0;
    for (int i = 0; i < L; ++i) {
      const int64_t h = (int64_t)1 << i;
      for (int64_t p = 0; p < n; ++p) {
        if (p & h) continue;
        const int64_t j = ((p >> (i + 1)) << i) | (p & (h - 1));
        const float ci = c[(int64_t)i * (n / 2) + j], si = s[(int64_t)i * (n / 2) + j];
        const float a = blk[p], b = blk[p + h];
        blk[p] = ci * a - si * b;
        blk[p + h] = si * a + ci * b;
      }
    }
  }
}

/* Per-token quantization of the rotated, smoothed activations:
 * x^_t = R(x_t * inv_s), then as or_quant_act. */
void or_quant_act_rotated(const float *x, int64_t M, int64_t K, const float *inv_s, int64_t n, const float *c,
                          const float *s, float *work, int8_t *xq, float *dx) {
  for (int64_t t = 0; t < M; ++t) {
    for (int64_t j = 0; j < K; ++j) work[j] = x[t * K + j] * inv_s[j];
    or_butterfly_rotate(work, K, n, c, s);
    float m = 0.0f;
    for (int64_t j = 0; j < K; ++j) {
      float a = fabsf(work[j]);
      if (a > m) m = a;
    }
    if (m == 0.0f) {
      dx[t] = 0.0f;
      for (int64_t j = 0; j < K; ++j) xq[t * K + j] = 0;
      continue;
    }
    dx[t] = m / 127.0f;
    for (int64_t j = 0; j < K; ++j) xq[t * K + j] = or_quantize_value(work[j], dx[t]);
  }
}

/* Per-output-channel quantization of the rotated, smoothed weights:
 * w^_n = R(s * w_n) over the K input channels, then as
 * or_smooth_quant_weight.  Wq [N][K]. */
void or_smooth_quant_weight_rotated(const float *w, int layout, int64_t K, int64_t N, const float *smooth,
                                    int64_t n, const float *c, const float *s, float *work, int8_t *wq,
                                    float *dw) {
  for (int64_t o = 0; o < N; ++o) {
    for (int64_t j = 0; j < K; ++j) work[j] = smooth[j] * w_at(w, layout, K, N, j, o);
    or_butterfly_rotate(work, K, n, c, s);
    float m = 0.0f;
    for (int64_t j = 0; j < K; ++j) {
      float a = fabsf(work[j]);
      if (a > m) m = a;
    }
    if (m == 0.0f) {
      dw[o] = 0.0f;
      for (int64_t j = 0; j < K; ++j) wq[o * K + j] = 0;
      continue;
    }
    dw[o] = m / 127.0f;
    for (int64_t j = 0; j < K; ++j) wq[o * K + j] = or_quantize_value(work[j], dw[o]);
  }
}
