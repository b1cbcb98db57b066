/*
 * slq_oracle.c -- plain, slow, scalar CPU oracle for the SLQ weight format.
 *
 * TEST INFRASTRUCTURE ONLY (see slq_oracle.h).  Each function states the
 * passage it follows.  Nothing here is blocked, fused or reordered: every
 * loop is the definition written out, one element at a time.
 *
 * Where the pages are silent the library fixes a reading, and this file
 * follows the same reading, stated where it is used:
 *   - scale is rounded to fp16 first and the encode uses that stored scale;
 *   - a group whose min equals its max is widened to include 0;
 *   - an all-zero group stores scale 1.0, zero 0, codes 0;
 *   - a nonzero fp32 scale that rounds to fp16 zero is stored as 2^-24;
 *     one that overflows fp16 is stored as 65504 and flagged;
 *   - codes are packed LSB-first into one bitstream per row, so a group of
 *     128 codes fills exactly 4*b uint32 words.
 *
 * Build: gcc -O2 -fno-fast-math -ffp-contract=off -shared -fPIC.
 */
#include "slq_oracle.h"

#include <math.h>
#include <stdlib.h>
#include <string.h>

#define GROUP 128

/* ---------------------------------------------------------------------- */
/* Number formats (IEEE 754 binary16 and bfloat16), written out by hand.   */
/* ---------------------------------------------------------------------- */

static uint32_t f32_bits(float f) {
  uint32_t u;
  memcpy(&u, &f, 4);
  return u;
}

static float bits_f32(uint32_t u) {
  float f;
  memcpy(&f, &u, 4);
  return f;
}

/* Round the integer x right by sh bits, to nearest, ties to even. */
static uint32_t shift_right_rne(uint32_t x, int sh) {
  if (sh <= 0) return x;
  if (sh >= 32) return 0; /* x < 2^24 here, so x / 2^sh < 1/2 */
  uint32_t q = x >> sh;
  uint32_t rem = x & ((1u << sh) - 1u);
  uint32_t half = 1u << (sh - 1);
  if (rem > half || (rem == half && (q & 1u))) q += 1u;
  return q;
}

uint16_t oracle_f32_to_f16_rn(float f) {
  uint32_t u = f32_bits(f);
  uint16_t sign = (uint16_t)((u >> 16) & 0x8000u);
  uint32_t e = (u >> 23) & 0xFFu;
  uint32_t m = u & 0x7FFFFFu;
  if (e == 0xFFu) return (uint16_t)(sign | (m ? 0x7E00u : 0x7C00u));
  if (e == 0u) return sign; /* |f| < 2^-126: far below half of 2^-24 */
  int E = (int)e - 127;     /* f = sig * 2^(E - 23) */
  uint32_t sig = (1u << 23) | m;
  if (E > 15) return (uint16_t)(sign | 0x7C00u);
  if (E >= -14) {
    /* Normal binary16: keep 11 significant bits. */
    uint32_t r = shift_right_rne(sig, 13);
    if (r == (1u << 11)) { /* rounding carried into the next binade */
      r = 1u << 10;
      E += 1;
    }
    if (E > 15) return (uint16_t)(sign | 0x7C00u);
    return (uint16_t)(sign | ((uint32_t)(E + 15) << 10) | (r - (1u << 10)));
  }
  /* Subnormal binary16: count units of 2^-24.  A result of 2^10 units is the
   * smallest normal, whose bit pattern is the same integer. */
  uint32_t r = shift_right_rne(sig, -E - 1);
  return (uint16_t)(sign | r);
}

double oracle_f16_to_f64(uint16_t h) {
  int sign = (h >> 15) & 1;
  int e = (h >> 10) & 0x1F;
  int m = h & 0x3FF;
  double v;
  if (e == 0)
    v = ldexp((double)m, -24);
  else if (e == 31)
    v = m ? NAN : INFINITY;
  else
    v = ldexp((double)(1024 + m), e - 25);
  return sign ? -v : v;
}

float oracle_bf16_to_f32(uint16_t h) { return bits_f32((uint32_t)h << 16); }

/* ---------------------------------------------------------------------- */
/* Quantize + pack.                                                        */
/* ---------------------------------------------------------------------- */

/* Write code q (bits wide) at stream bit position pos of one row's words,
 * least significant bit first: stream bit i is bit (i mod 32) of word i/32. */
static void put_code(uint32_t *row_words, int64_t pos, int bits, uint32_t q) {
  int64_t w = pos / 32;
  int sh = (int)(pos % 32);
  row_words[w] |= q << sh;
  if (sh + bits > 32) row_words[w + 1] |= q >> (32 - sh);
}

uint32_t oracle_code_at(const uint32_t *packed, int64_t K, int bits, int64_t n,
                        int64_t k) {
  const uint32_t *row = packed + n * (K * bits / 32);
  int64_t pos = k * bits;
  int64_t w = pos / 32;
  int sh = (int)(pos % 32);
  uint64_t window = row[w];
  if (sh + bits > 32) window |= (uint64_t)row[w + 1] << 32;
  return (uint32_t)((window >> sh) & ((1u << bits) - 1u));
}

/*
 * One group of 128 weights along K.  The pages fix: asymmetric integer grid,
 * group size 128, b in {2..8} (gist.science "The SLQ Pipeline"; GitHub README
 * "Pipeline"), round to nearest (RTN).  The library's format definition fixes
 * the arithmetic in binary32:
 *   scale = (max - min) / (2^b - 1), zero = clamp(rne(-min / scale)),
 *   q = clamp(rne(w / scale) + zero), codes in [0, 2^b - 1].
 */
static void group_params(const float *w, int bits, uint16_t *s16_out, float *z_out,
                         uint32_t *flags) {
  int nonfinite = 0;
  for (int k = 0; k < GROUP; ++k)
    if (!isfinite(w[k])) nonfinite = 1;
  if (nonfinite && flags) *flags |= ORACLE_FLAG_NONFINITE;

  /* Group statistics: min and max in binary32 (exact). */
  float mn = w[0], mx = w[0];
  for (int k = 1; k < GROUP; ++k) {
    if (w[k] < mn) mn = w[k];
    if (w[k] > mx) mx = w[k];
  }

  /* Reading: a constant group is widened to include 0, so that it
   * reconstructs to (about) itself instead of dividing by a zero range. */
  float lo = mn, hi = mx;
  if (hi == lo) {
    if (lo > 0.0f) lo = 0.0f;
    if (hi < 0.0f) hi = 0.0f;
  }

  const float maxq = (float)((1 << bits) - 1);
  float s32 = (hi - lo) / maxq; /* one binary32 subtraction, one IEEE division */

  /* Reading: the scale is stored in fp16 and the encode uses the stored
   * value, so the reconstruction bound holds for what the GEMM reads. */
  uint16_t s16;
  if (s32 == 0.0f) {
    s16 = 0x3C00u; /* all-zero group: scale 1.0 */
  } else {
    s16 = oracle_f32_to_f16_rn(s32);
    if ((s16 & 0x7FFFu) == 0u) {
      s16 = 0x0001u; /* nonzero scale below fp16 range: 2^-24 */
    } else if (s16 == 0x7C00u) {
      s16 = 0x7BFFu; /* beyond fp16 range: 65504, flagged */
      if (flags) *flags |= ORACLE_FLAG_SCALE_OVERFLOW;
    }
  }
  const float s = (float)oracle_f16_to_f64(s16);

  /* Zero point: rne(-min / scale), clamped to the code range. */
  float zf = rintf(-lo / s);
  if (zf != zf || zf < 0.0f) zf = 0.0f;
  if (zf > maxq) zf = maxq;
  *s16_out = s16;
  *z_out = zf;
}

/* Code of one weight: rne(w / scale) + zero, clamped to the code range.  The
 * sum is taken in binary32: it is exact whenever the result is inside the
 * range. */
static uint32_t encode_one(float w, float s, float zf, int bits) {
  const float maxq = (float)((1 << bits) - 1);
  float v = rintf(w / s) + zf;
  if (v != v || v < 0.0f) v = 0.0f;
  if (v > maxq) v = maxq;
  return (uint32_t)v;
}

static void quantize_group(const uint16_t *src, int bits, uint16_t *s16_out,
                           uint8_t *z_out, uint32_t *codes, uint32_t *flags) {
  float w[GROUP];
  for (int k = 0; k < GROUP; ++k) w[k] = oracle_bf16_to_f32(src[k]);
  float zf;
  group_params(w, bits, s16_out, &zf, flags);
  const float s = (float)oracle_f16_to_f64(*s16_out);
  for (int k = 0; k < GROUP; ++k) codes[k] = encode_one(w[k], s, zf, bits);
  *z_out = (uint8_t)zf;
}

int oracle_quantize(const uint16_t *w_bf16, int64_t N, int64_t K, int bits,
                    uint32_t *packed, uint16_t *scales_f16, uint8_t *zeros,
                    uint32_t *flags) {
  if (bits < 2 || bits > 8 || N < 0 || K < 0 || K % GROUP != 0) return -1;
  const int64_t G = K / GROUP;
  const int64_t words_per_row = K * bits / 32;
  memset(packed, 0, (size_t)(N * words_per_row) * sizeof(uint32_t));
  uint32_t codes[GROUP];
  for (int64_t n = 0; n < N; ++n) {
    uint32_t *row_words = packed + n * words_per_row;
    for (int64_t g = 0; g < G; ++g) {
      quantize_group(w_bf16 + n * K + g * GROUP, bits, &scales_f16[n * G + g],
                     &zeros[n * G + g], codes, flags);
      for (int j = 0; j < GROUP; ++j)
        put_code(row_words, (g * GROUP + j) * bits, bits, codes[j]);
    }
  }
  return 0;
}

/* ---------------------------------------------------------------------- */
/* GPTQ with this format's quantizer.                                      */
/* ---------------------------------------------------------------------- */

/* In-place lower Cholesky factor of the n x n row-major matrix a (a = L L^T);
 * the upper triangle is zeroed.  Returns -1 if a is not positive definite. */
static int cholesky_lower(double *a, int64_t n) {
  for (int64_t j = 0; j < n; ++j) {
    double d = a[j * n + j];
    for (int64_t k = 0; k < j; ++k) d -= a[j * n + k] * a[j * n + k];
    if (!(d > 0.0)) return -1;
    d = sqrt(d);
    a[j * n + j] = d;
    for (int64_t i = j + 1; i < n; ++i) {
      double v = a[i * n + j];
      for (int64_t k = 0; k < j; ++k) v -= a[i * n + k] * a[j * n + k];
      a[i * n + j] = v / d;
    }
    for (int64_t k = j + 1; k < n; ++k) a[j * n + k] = 0.0;
  }
  return 0;
}

/*
 * GPTQ (Frantar et al., "GPTQ: Accurate Post-Training Quantization for
 * Generative Pre-trained Transformers"): the encoder the pages run for every
 * layer at every b (GitHub README, "Pipeline" and "1. Quantize": layer-wise
 * GPTQ, asymmetric INT, group size 128).  Each row of W is encoded column by
 * column; after a column is fixed, the error it leaves is spread over the
 * row's later columns so as to minimize the change of X W^T on the
 * calibration rows X.  Readings where the pages are silent:
 *   - H = X^T X in binary64 (the usual factor 2/T does not change the
 *     result); a column with H_kk = 0 (an input that is always zero) gets
 *     H_kk = 1 and its weights set to 0;
 *   - damping H += damp * mean(diag H) * I;
 *   - columns in their natural order (no activation ordering);
 *   - a group's scale and zero come from the group's current, already
 *     updated weights when its first column is reached, by the RTN rules
 *     above;
 *   - the weights are carried in binary64 and rounded to binary32 for the
 *     encode decision;
 *   - with U the upper Cholesky factor of H^-1 (H^-1 = U^T U), fixing column
 *     k with dequantized value d moves every later column j of the row by
 *     -(w_k - d) / U_kk * U_kj.
 * x_bf16: [T, K] calibration rows.  Returns 0; -1 on an invalid argument;
 * -2 if the damped H is not positive definite or memory runs out.
 */
int oracle_gptq(const uint16_t *w_bf16, int64_t N, int64_t K, int bits,
                const uint16_t *x_bf16, int64_t T, double damp, uint32_t *packed,
                uint16_t *scales_f16, uint8_t *zeros, uint32_t *flags) {
  if (bits < 2 || bits > 8 || N < 0 || K < GROUP || K % GROUP != 0 || T < 1 ||
      !(damp >= 0.0) || isinf(damp))
    return -1;
  const int64_t G = K / GROUP;
  const int64_t words_per_row = K * bits / 32;
  double *h = (double *)calloc((size_t)(K * K), sizeof(double));
  double *inv = (double *)calloc((size_t)(K * K), sizeof(double));
  double *x = (double *)malloc((size_t)K * sizeof(double));
  double *w = (double *)malloc((size_t)K * sizeof(double));
  unsigned char *dead = (unsigned char *)calloc((size_t)K, 1);
  int rc = -2;
  if (!h || !inv || !x || !w || !dead) goto done;

  /* H = X^T X. */
  for (int64_t t = 0; t < T; ++t) {
    for (int64_t k = 0; k < K; ++k) x[k] = (double)oracle_bf16_to_f32(x_bf16[t * K + k]);
    for (int64_t i = 0; i < K; ++i)
      for (int64_t j = 0; j <= i; ++j) h[i * K + j] += x[i] * x[j];
  }
  for (int64_t i = 0; i < K; ++i)
    for (int64_t j = 0; j < i; ++j) h[j * K + i] = h[i * K + j];
  double mean = 0.0;
  for (int64_t k = 0; k < K; ++k) {
    if (h[k * K + k] == 0.0) {
      h[k * K + k] = 1.0;
      dead[k] = 1;
    }
    mean += h[k * K + k];
  }
  mean /= (double)K;
  for (int64_t k = 0; k < K; ++k) h[k * K + k] += damp * mean;

  /* H^-1 = L^-T L^-1 from H = L L^T, then U^T = the lower factor of H^-1. */
  if (cholesky_lower(h, K) != 0) goto done;
  for (int64_t c = 0; c < K; ++c) { /* column c of L^-1 by forward substitution */
    for (int64_t i = 0; i < K; ++i) {
      double v = (i == c) ? 1.0 : 0.0;
      for (int64_t k = c; k < i; ++k) v -= h[i * K + k] * inv[k * K + c];
      inv[i * K + c] = (i < c) ? 0.0 : v / h[i * K + i];
    }
  }
  for (int64_t i = 0; i < K; ++i) /* h := (L^-1)^T L^-1, i.e. H^-1 */
    for (int64_t j = 0; j < K; ++j) {
      double v = 0.0;
      for (int64_t k = (i > j ? i : j); k < K; ++k) v += inv[k * K + i] * inv[k * K + j];
      h[i * K + j] = v;
    }
  if (cholesky_lower(h, K) != 0) goto done; /* h = U^T: U_kj = h[j][k] */

  memset(packed, 0, (size_t)(N * words_per_row) * sizeof(uint32_t));
  for (int64_t n = 0; n < N; ++n) {
    uint32_t *row_words = packed + n * words_per_row;
    for (int64_t k = 0; k < K; ++k)
      w[k] = dead[k] ? 0.0 : (double)oracle_bf16_to_f32(w_bf16[n * K + k]);
    uint16_t s16 = 0;
    float s = 0.0f, zf = 0.0f;
    for (int64_t k = 0; k < K; ++k) {
      if (k % GROUP == 0) {
        float wg[GROUP];
        for (int j = 0; j < GROUP; ++j) wg[j] = (float)w[k + j];
        group_params(wg, bits, &s16, &zf, flags);
        s = (float)oracle_f16_to_f64(s16);
        scales_f16[n * G + k / GROUP] = s16;
        zeros[n * G + k / GROUP] = (uint8_t)zf;
      }
      const uint32_t q = encode_one((float)w[k], s, zf, bits);
      put_code(row_words, k * bits, bits, q);
      const double d = oracle_f16_to_f64(s16) * ((double)q - (double)zf);
      const double u_kk = h[k * K + k];
      const double e = (w[k] - d) / u_kk;
      for (int64_t j = k + 1; j < K; ++j) w[j] -= e * h[j * K + k];
    }
  }
  rc = 0;
done:
  free(h);
  free(inv);
  free(x);
  free(w);
  free(dead);
  return rc;
}

/* ---------------------------------------------------------------------- */
/* Dequantize and GEMM (weight-only, bf16 activations).                    */
/* ---------------------------------------------------------------------- */

/* w' = s * (q - z): the fake-quantized weight the pages store (GitHub README,
 * "1. Quantize" and "4. Build and serve a checkpoint").  Exact in binary64. */
static void dequantize_row(const uint32_t *packed, const uint16_t *scales_f16,
                           const uint8_t *zeros, int64_t K, int bits, int64_t n,
                           double *out) {
  const int64_t G = K / GROUP;
  for (int64_t k = 0; k < K; ++k) {
    int64_t g = k / GROUP;
    double s = oracle_f16_to_f64(scales_f16[n * G + g]);
    double q = (double)oracle_code_at(packed, K, bits, n, k);
    double z = (double)zeros[n * G + g];
    out[k] = s * (q - z);
  }
}

int oracle_dequantize(const uint32_t *packed, const uint16_t *scales_f16,
                      const uint8_t *zeros, int64_t N, int64_t K, int bits,
                      double *w_out) {
  if (bits < 2 || bits > 8 || K % GROUP != 0) return -1;
  for (int64_t n = 0; n < N; ++n)
    dequantize_row(packed, scales_f16, zeros, K, bits, n, w_out + n * K);
  return 0;
}

/* Y = X W^T with w' as above: y[m, n] = sum_k x[m, k] * w'[n, k], binary64,
 * k ascending.  This is the weight-only linear layer that the serving
 * kernels compute (gist.science "Inference Speedup"; GitHub README intro). */
int oracle_gemm(const uint16_t *x_bf16, const int64_t *rows, int64_t n_rows,
                int64_t N, int64_t K, int bits, const uint32_t *packed,
                const uint16_t *scales_f16, const uint8_t *zeros, double *y) {
  if (bits < 2 || bits > 8 || K % GROUP != 0) return -1;
  /* Widen the sampled rows of X once (bf16 -> double is exact). */
  double *xd = (double *)malloc((size_t)(n_rows * K) * sizeof(double));
  double *wrow = (double *)malloc((size_t)K * sizeof(double));
  if (!xd || !wrow) {
    free(xd);
    free(wrow);
    return -2;
  }
  for (int64_t i = 0; i < n_rows; ++i) {
    int64_t m = rows ? rows[i] : i;
    for (int64_t k = 0; k < K; ++k)
      xd[i * K + k] = (double)oracle_bf16_to_f32(x_bf16[m * K + k]);
  }
  for (int64_t n = 0; n < N; ++n) {
    dequantize_row(packed, scales_f16, zeros, K, bits, n, wrow);
    for (int64_t i = 0; i < n_rows; ++i) {
      double acc = 0.0;
      for (int64_t k = 0; k < K; ++k) acc += xd[i * K + k] * wrow[k];
      y[i * N + n] = acc;
    }
  }
  free(xd);
  free(wrow);
  return 0;
}

/* ---------------------------------------------------------------------- */
/* EAR and KL between two softmaxed logit rows.                            */
/* ---------------------------------------------------------------------- */

/* log sum_v exp(u_v), shifted by the maximum so no term overflows. */
static double logsumexp(const double *u, int64_t V) {
  double mx = u[0];
  for (int64_t v = 1; v < V; ++v)
    if (u[v] > mx) mx = u[v];
  if (isinf(mx)) return mx;
  double sum = 0.0;
  for (int64_t v = 0; v < V; ++v) sum += exp(u[v] - mx);
  return mx + log(sum);
}

/*
 * For one token: p = softmax(a / tau) (reference model), q = softmax(b / tau)
 * (quantized model).  EAR = sum_v min(p_v, q_v), the probability that the two
 * models agree under the optimal coupling (gist.science "Fidelity Metrics";
 * reddit abstract).  The pages' evaluation restricts it to the top-K tokens;
 * this is the full-vocabulary case, K = V.  KL(p || q) = sum_v p_v (log p_v -
 * log q_v) in nats (gist.science "Fidelity Metrics", Task-Lossless search
 * signal).  log p_v is taken as the log-softmax a_v / tau - logsumexp, so a
 * p_v that underflows to 0 contributes 0 * finite = 0.
 */
int oracle_ear_kl(const uint16_t *a_bf16, const uint16_t *b_bf16,
                  const int64_t *rows, int64_t n_rows, int64_t V, double tau,
                  double *ear, double *kl) {
  if (V < 1 || !(tau > 0.0) || isinf(tau)) return -1;
  double *x = (double *)malloc((size_t)V * sizeof(double));
  double *y = (double *)malloc((size_t)V * sizeof(double));
  if (!x || !y) {
    free(x);
    free(y);
    return -2;
  }
  for (int64_t i = 0; i < n_rows; ++i) {
    int64_t t = rows ? rows[i] : i;
    for (int64_t v = 0; v < V; ++v) {
      x[v] = (double)oracle_bf16_to_f32(a_bf16[t * V + v]) / tau;
      y[v] = (double)oracle_bf16_to_f32(b_bf16[t * V + v]) / tau;
    }
    double la = logsumexp(x, V);
    double lb = logsumexp(y, V);
    double e = 0.0, d = 0.0;
    for (int64_t v = 0; v < V; ++v) {
      double log_p = x[v] - la;
      double log_q = y[v] - lb;
      double p = exp(log_p);
      double q = exp(log_q);
      e += (p < q) ? p : q;
      d += p * (log_p - log_q);
    }
    ear[i] = e;
    kl[i] = d;
  }
  free(x);
  free(y);
  return 0;
}

/*
 * Top-K form of the same metrics, the one the pages' search and evaluation
 * use: EAR = (1/N) sum_i sum_{k=1..K} min(p_i(k), q_i(k)) restricted to the
 * top-K tokens (gist.science summary, Methodology section 2 "Fidelity
 * Metrics", Definition; GitHub README "2. Build the sensitivity database":
 * top-K = 10; eval/run_ear.py and eval/run_kl.py, "EAR and top-K KL").
 *
 * Readings (the pages leave them open):
 *   - the top-K set T is the K tokens with the largest reference logits a
 *     (the original model's distribution p), ties to the lower index;
 *   - EAR sums min(p_v, q_v) over T with p and q the full-vocabulary
 *     softmaxes (not renormalized), so it is at most the full EAR and equals
 *     it when K = V;
 *   - KL is KL(p_T || q_T) between p and q renormalized over T, a proper
 *     divergence that equals the full KL when K = V.
 * Selection is K passes of "largest remaining logit" over the row.
 */
int oracle_ear_kl_topk(const uint16_t *a_bf16, const uint16_t *b_bf16,
                       const int64_t *rows, int64_t n_rows, int64_t V, int64_t K,
                       double tau, double *ear, double *kl, int64_t *top) {
  if (V < 1 || K < 1 || K > V || !(tau > 0.0) || isinf(tau)) return -1;
  double *x = (double *)malloc((size_t)V * sizeof(double));
  double *y = (double *)malloc((size_t)V * sizeof(double));
  unsigned char *taken = (unsigned char *)calloc((size_t)V, 1);
  int64_t *sel = (int64_t *)malloc((size_t)K * sizeof(int64_t));
  if (!x || !y || !taken || !sel) {
    free(x);
    free(y);
    free(taken);
    free(sel);
    return -2;
  }
  for (int64_t i = 0; i < n_rows; ++i) {
    int64_t t = rows ? rows[i] : i;
    for (int64_t v = 0; v < V; ++v) {
      x[v] = (double)oracle_bf16_to_f32(a_bf16[t * V + v]) / tau;
      y[v] = (double)oracle_bf16_to_f32(b_bf16[t * V + v]) / tau;
      taken[v] = 0;
    }
    /* T: K passes, each taking the largest remaining a (lowest index on ties). */
    for (int64_t k = 0; k < K; ++k) {
      int64_t best = -1;
      for (int64_t v = 0; v < V; ++v) {
        if (taken[v]) continue;
        if (best < 0 || x[v] > x[best]) best = v;
      }
      taken[best] = 1;
      sel[k] = best;
      if (top) top[i * K + k] = best;
    }
    double la = logsumexp(x, V);
    double lb = logsumexp(y, V);
    double e = 0.0, pt = 0.0, qt = 0.0;
    for (int64_t k = 0; k < K; ++k) {
      double p = exp(x[sel[k]] - la);
      double q = exp(y[sel[k]] - lb);
      e += (p < q) ? p : q;
      pt += p;
      qt += q;
    }
    /* KL(p_T || q_T) with p_T = p / pt, q_T = q / qt, from the log-softmax. */
    double d = 0.0;
    for (int64_t k = 0; k < K; ++k) {
      double log_pt = (x[sel[k]] - la) - log(pt);
      double log_qt = (y[sel[k]] - lb) - log(qt);
      d += exp(log_pt) * (log_pt - log_qt);
    }
    ear[i] = e;
    kl[i] = d;
  }
  free(x);
  free(y);
  free(taken);
  free(sel);
  return 0;
}


/* ------------------------------------------------------------------------
 * Grid noise of the symmetric-vs-asymmetric ablation.  The pages' gamma^2
 * law says a symmetric grid over [-M, M] has gamma^2 = (2M / R)^2 times the
 * noise variance of an asymmetric grid over [lo, hi], because its step is
 * gamma times larger and rounding noise scales with the step squared.  Per
 * group this computes gamma and the squared reconstruction error of each
 * grid, nearest point by rounding the binary64 position (w - start) / step
 * (ties go to the even index; either neighbour gives the same error).
 * ------------------------------------------------------------------------ */
static double grid_sse(const double *w, int n, double start, double step, int levels) {
  double sse = 0.0;
  for (int k = 0; k < n; ++k) {
    double r;
    if (step == 0.0) {
      r = start;
    } else {
      double i = nearbyint((w[k] - start) / step);
      if (i < 0.0) i = 0.0;
      if (i > (double)levels) i = (double)levels;
      r = start + i * step;
    }
    double e = w[k] - r;
    sse += e * e;
  }
  return sse;
}

int oracle_grid_noise(const uint16_t *w_bf16, int64_t N, int64_t K, int bits,
                      double *gamma, double *sse_asym, double *sse_sym) {
  if (N < 0 || K < GROUP || K % GROUP || bits < 2 || bits > 8) return -1;
  const int levels = (1 << bits) - 1;
  const int64_t G = K / GROUP;
  double w[GROUP];
  for (int64_t n = 0; n < N; ++n) {
    for (int64_t g = 0; g < G; ++g) {
      double lo = 0.0, hi = 0.0, m = 0.0;
      for (int k = 0; k < GROUP; ++k) {
        w[k] = (double)oracle_bf16_to_f32(w_bf16[n * K + g * GROUP + k]);
        if (k == 0 || w[k] < lo) lo = w[k];
        if (k == 0 || w[k] > hi) hi = w[k];
        if (fabs(w[k]) > m) m = fabs(w[k]);
      }
      const double range = hi - lo;
      const int64_t o = n * G + g;
      gamma[o] = range > 0.0 ? 2.0 * m / range : 1.0;
      sse_asym[o] = grid_sse(w, GROUP, lo, range / levels, levels);
      sse_sym[o] = grid_sse(w, GROUP, -m, 2.0 * m / levels, levels);
    }
  }
  return 0;
}
