/*
 * slq_oracle.h -- plain, slow CPU oracle for the SLQ weight format.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing on the product path may include, link,
 * load or call this code: only the tests, the package's smoke check and the
 * benchmark's CPU-baseline leg use it.  It shares no code with the CUDA
 * library (weight_only_mixed_b200/csrc) and includes none of its headers.
 *
 * What it computes (sources are the web pages on "Statistically-Lossless
 * Quantization of Large Language Models", Helcig, Kurtic, Alistarh):
 *   - asymmetric INT-b group quantization, group size 128 along K, b in 2..8
 *     (gist.science summary, "Methodology" section 3 "The SLQ Pipeline";
 *     GitHub README "Pipeline" paragraph and "Evaluation" Uniform-4 note),
 *     round-to-nearest encode (reddit excerpt of the paper's introduction,
 *     which names RTN as the plain lossy baseline);
 *   - the packed per-layer-bitwidth storage that the serving kernels read
 *     (GitHub README, "4. Build and serve a checkpoint": weights are packed to
 *     their per-layer bitwidths on load);
 *   - dequantization w = s * (q - z) and the weight-only GEMM Y = X W^T;
 *   - the Expected Acceptance Rate EAR = sum_v min(p_v, q_v) and KL(p || q)
 *     between two softmaxed logit rows (gist.science summary, "Methodology"
 *     section 2 "Fidelity Metrics"; reddit abstract: EAR is the maximum
 *     token-agreement probability under optimal coupling);
 *   - GPTQ with this format's quantizer, the encoder the pages run for every
 *     layer at every b (GitHub README, "Pipeline" and "1. Quantize");
 *   - the per-group noise of a symmetric against an asymmetric grid, the
 *     ablation behind the gamma^2 variance law (wispaper.ai blog, section on
 *     the gamma^2 law; gist.science summary, "Methodology" section 1).
 *
 * Precision: encode decisions in IEEE binary32 (the library's format
 * definition fixes fp32 for scale, zero and code); dequantize, GEMM and
 * EAR/KL in binary64.  Build with -O2 -fno-fast-math -ffp-contract=off.
 */
#ifndef SLQ_ORACLE_H
#define SLQ_ORACLE_H

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Flags OR-ed into *flags by oracle_quantize (same meaning as the library). */
#define ORACLE_FLAG_NONFINITE 1u
#define ORACLE_FLAG_SCALE_OVERFLOW 2u

/* binary32 -> binary16 bits, round to nearest even, subnormals kept,
 * overflow to +/-inf, NaN to a quiet NaN.  Written out from IEEE 754. */
uint16_t oracle_f32_to_f16_rn(float f);
/* binary16 bits -> double (exact). */
double oracle_f16_to_f64(uint16_t h);
/* bfloat16 bits -> float (exact). */
float oracle_bf16_to_f32(uint16_t h);

/* Quantize W (bf16 bits, [N, K] row-major, K % 128 == 0) to b bits.
 * packed: uint32 [N, K*b/32]; scales: fp16 bits [N, K/128]; zeros: [N, K/128].
 * flags may be NULL.  Returns 0, or -1 on an invalid argument. */
int oracle_quantize(const uint16_t *w_bf16, int64_t N, int64_t K, int bits,
                    uint32_t *packed, uint16_t *scales_f16, uint8_t *zeros,
                    uint32_t *flags);

/* GPTQ encode of W (bf16 bits, [N, K]) to b bits in the same format as
 * oracle_quantize, with calibration rows x (bf16 bits, [T, K]) and relative
 * damping damp (readings in slq_oracle.c).  flags may be NULL.  Returns 0,
 * -1 on an invalid argument, -2 if the damped X^T X is singular or memory
 * runs out. */
int oracle_gptq(const uint16_t *w_bf16, int64_t N, int64_t K, int bits,
                const uint16_t *x_bf16, int64_t T, double damp, uint32_t *packed,
                uint16_t *scales_f16, uint8_t *zeros, uint32_t *flags);

/* Read code k of row n back out of the packed stream. */
uint32_t oracle_code_at(const uint32_t *packed, int64_t K, int bits,
                        int64_t n, int64_t k);

/* w'[n, k] = s16[n, g] * (q[n, k] - z[n, g]) in binary64 (exact). */
int oracle_dequantize(const uint32_t *packed, const uint16_t *scales_f16,
                      const uint8_t *zeros, int64_t N, int64_t K, int bits,
                      double *w_out);

/* y[i, n] = sum_k x[rows[i], k] * w'[n, k] in binary64, k ascending.
 * x: bf16 bits [M_total, K]; rows: n_rows indices into x's rows (NULL means
 * rows 0..n_rows-1); y: [n_rows, N] doubles. */
int oracle_gemm(const uint16_t *x_bf16, const int64_t *rows, int64_t n_rows,
                int64_t N, int64_t K, int bits, const uint32_t *packed,
                const uint16_t *scales_f16, const uint8_t *zeros, double *y);

/* Per-token EAR and KL(p || q) with p = softmax(a / tau), q = softmax(b / tau),
 * natural log.  a, b: bf16 bits [T, V]; rows: n_rows token indices (NULL means
 * 0..n_rows-1); ear, kl: [n_rows] doubles. */
int oracle_ear_kl(const uint16_t *a_bf16, const uint16_t *b_bf16,
                  const int64_t *rows, int64_t n_rows, int64_t V, double tau,
                  double *ear, double *kl);

/* Top-K EAR and KL (readings in slq_oracle.c): T = the K largest a (ties to
 * the lower index); ear = sum over T of min(p, q) with full softmaxes; kl =
 * KL between p and q renormalized over T.  top (nullable): [n_rows, K] the
 * selected token indices, largest first. */
int oracle_ear_kl_topk(const uint16_t *a_bf16, const uint16_t *b_bf16,
                       const int64_t *rows, int64_t n_rows, int64_t V, int64_t K,
                       double tau, double *ear, double *kl, int64_t *top);

/* Per-group grid noise for the symmetric-vs-asymmetric ablation (the gamma^2
 * variance law: wispaper.ai blog, section on the gamma^2 law; gist.science
 * summary, Methodology section 1).  For each 128-group g of row n of W (bf16
 * bits, [N, K], K % 128 == 0), with lo = min w, hi = max w, M = max |w|,
 * R = hi - lo, and L = 2^b - 1 intervals:
 *   gamma[n, g]    = 2M / R (1 when R == 0);
 *   sse_asym[n, g] = sum over the group of (w - nearest point of the grid
 *                    lo + i R / L)^2, i = 0..L;
 *   sse_sym[n, g]  = the same for the grid -M + i 2M / L.
 * Both grids in binary64 without scale rounding: this measures the grids
 * the law compares, not the stored format.  Non-finite weights give
 * non-finite results.  Returns 0, or -1 on an invalid argument. */
int oracle_grid_noise(const uint16_t *w_bf16, int64_t N, int64_t K, int bits,
                      double *gamma, double *sse_asym, double *sse_sym);

#ifdef __cplusplus
}
#endif
#endif
