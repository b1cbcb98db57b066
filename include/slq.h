/*
 * slq.h -- C ABI of the SLQ weight-format library (libslq.so, sm_100a).
 *
 * The library implements the hot path of "Statistically-Lossless
 * Quantization of Large Language Models" (Helcig, Kurtic, Alistarh): the
 * layer-wise asymmetric INT-b weight format with group size 128 along K and
 * a bitwidth b in {2, ..., 8} per layer, and the three operations that run on
 * it: quantize+pack, the fused dequantize-GEMM, and the EAR/KL fidelity
 * reduction.
 *
 * Conventions for every entry point:
 *   - Pointers named *_host are host memory; all others are DEVICE memory
 *     (cudaMalloc or any allocator) owned by the caller.  The library never
 *     allocates, frees or synchronizes; it only launches kernels on `stream`
 *     (a cudaStream_t passed as void*, NULL = legacy default stream).
 *   - Arrays are dense and row-major.  bf16 arrays and packed codes start on
 *     a 16-byte boundary; the others on their element size (both checked).
 *     Inputs and outputs must not overlap (checked).
 *   - bf16 / fp16 data is raw 16-bit IEEE bfloat16 / binary16 bits.
 *   - Argument errors are reported synchronously, before anything is
 *     launched.  A failed launch returns SLQ_ERR_CUDA.  Conditions that depend
 *     on the data are reported asynchronously: kernels OR bits into the
 *     optional device word *flags (caller zeroes it, reads it after a sync).
 *   - The only supported device is compute capability 10.0 (B200, sm_100a);
 *     any other device, or no device, gives SLQ_ERR_UNSUPPORTED_DEVICE.  There
 *     is no CPU or other-architecture fallback.
 *   - Calls keep no state between them and may be issued from several host
 *     threads on different streams.
 */
#ifndef SLQ_H
#define SLQ_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  SLQ_OK = 0,
  SLQ_ERR_INVALID_ARGUMENT = 1,
  SLQ_ERR_UNSUPPORTED_DEVICE = 2,
  SLQ_ERR_CUDA = 3,
  SLQ_ERR_TIMEOUT = 4
} slq_status;

typedef enum { SLQ_DTYPE_BF16 = 0, SLQ_DTYPE_F32 = 1 } slq_dtype;

/* Bits OR-ed into *flags by the kernels. */
enum {
  SLQ_FLAG_NONFINITE = 1u,      /* a weight was inf or NaN: that group's output is unspecified */
  SLQ_FLAG_SCALE_OVERFLOW = 2u, /* a group's range exceeded fp16: scale stored as 65504 */
  SLQ_FLAG_TIMEOUT = 4u,        /* a bounded on-chip wait gave up; outputs are unspecified */
  SLQ_FLAG_NOT_POSITIVE_DEFINITE = 8u /* slq_gptq: a Cholesky pivot was not positive; outputs unspecified */
};

/* GEMM kernel choice for slq_gemm_ex.  Every kernel forms exact bf16 values
 * from the codes, multiplies on the tensor cores with fp32 accumulation, one
 * product per 128-wide group, and applies the fp16 group scale to that fp32
 * product; they differ in how the work is split. */
typedef enum {
  SLQ_GEMM_AUTO = 0,   /* GEMV for M <= 16, TILED above */
  SLQ_GEMM_DECODE = 1, /* M <= 16: packed weights streamed by TMA, dequantized in registers
                          into mma.sync fragments, the row tiles x groups split evenly over
                          two CTAs per SM (stream-K; needs a workspace) */
  SLQ_GEMM_TILED = 2,  /* any M >= 1: 128 x {64, 128, 256} output tiles, exact bf16 (q - z)
                          written into TMEM, tcgen05.mma with A from TMEM into per-group
                          TMEM product buffers folded by the group scale in fp32 registers,
                          K split over a thread-block cluster for narrow tiles */
  SLQ_GEMM_GEMV = 3    /* M <= 16: one CTA per 16- or 32-row tile whose warps split K, packed
                          weights streamed with cp.async into per-warp shared-memory rings,
                          dequantized in registers into mma.sync fragments; partial tiles
                          added in shared memory (no workspace) */
} slq_gemm_path;

/* Group size along K, fixed by the format ("asymmetric INT, group size 128",
 * gist.science summary, Methodology section 3 "The SLQ Pipeline"). */
#define SLQ_GROUP 128

/* Largest sizes accepted: every row count and K below 2^31, and
 * N*K, M*K, M*N, T*V below 2^40 elements. */

/* Library version, as 10000*major + 100*minor + patch. */
int slq_version(void);

/* Human-readable name of a status code (static string). */
const char *slq_status_string(slq_status status);

/* Number of uint32 words of the packed codes of an [N, K] layer at `bits`
 * bits: N*K*bits/32 (each 128-code group fills exactly 4*bits words).
 * Returns 0 for invalid arguments. */
size_t slq_packed_words(int64_t N, int64_t K, int bits);

/* Which kernel slq_gemm would run for these sizes (SLQ_GEMM_GEMV or
 * SLQ_GEMM_TILED).  Host-only; launches nothing. */
slq_gemm_path slq_gemm_select(int64_t M, int64_t N, int64_t K, int bits);

/* Bytes of device workspace the SLQ_GEMM_DECODE kernel needs for
 * Y[M, N] = X[M, K] W[N, K]^T on the CURRENT device (it splits the layer over
 * that device's SMs); 0 when it needs none (every row tile falls in one CTA)
 * and for M > 16.  Only slq_gemm_ex with SLQ_GEMM_DECODE takes a workspace.
 * Returns 0 for invalid arguments.
 *
 * Workspace rules: device memory owned by the caller, 256-byte aligned, not
 * overlapping any other argument.  Its first 64 KiB hold per-row-tile
 * counters that must be ALL ZERO before its first use; every call that
 * completes without SLQ_FLAG_TIMEOUT leaves them zero again (the rest is
 * scratch), so one buffer serves any number of calls -- of any layer sizes --
 * issued one after another on a stream.  Calls that may run at the same time
 * need separate buffers.  After a call that raised SLQ_FLAG_TIMEOUT the caller
 * must zero the first 64 KiB again.  The decode kernel takes N up to
 * 16384 * 128 = 2097152 (SLQ_ERR_INVALID_ARGUMENT above). */
size_t slq_gemm_workspace_bytes(int64_t M, int64_t N, int64_t K, int bits);

/*
 * slq_quantize -- round-to-nearest asymmetric INT-`bits` encode of W, group
 * size 128 along K, packed to the layer's bitwidth.
 *
 * Source: the pages fix an asymmetric integer grid, group size 128 and
 * b in 2..8 per layer (gist.science summary, Methodology section 3 "The SLQ
 * Pipeline"; GitHub README, "Pipeline" paragraph), round-to-nearest as the
 * plain encoder (reddit excerpt of the paper's introduction: RTN), and
 * weights packed to per-layer bitwidths when the model is loaded (GitHub
 * README, "4. Build and serve a checkpoint").  Per group of 128 weights, in
 * IEEE binary32: lo = min, hi = max (a constant group is widened to include
 * 0); s = fp16_rn((hi - lo) / (2^b - 1)) (an all-zero group gets 1.0, a
 * nonzero step below fp16 range 2^-24, one above it 65504 + flag);
 * z = clamp(rne(-lo / s), 0, 2^b - 1); q = clamp(rne(w / s) + z, 0, 2^b - 1).
 *
 * W_bf16      [N, K] bf16, device, read-only.
 * N, K        N >= 0 (0 launches nothing), K >= 128 and K % 128 == 0.
 * bits        2..8.
 * packed      [N, K*bits/32] uint32, device, written.  Row n is one bit
 *             stream, least significant bit first (stream bit i is bit i%32
 *             of word i/32); code k of the row occupies stream bits
 *             [k*bits, k*bits + bits).
 * scales_f16  [N, K/128] fp16, device, written.
 * zeros       [N, K/128] uint8, device, written.
 * flags       device uint32 or NULL; SLQ_FLAG_NONFINITE / _SCALE_OVERFLOW.
 * stream      cudaStream_t.
 */
slq_status slq_quantize(const void *W_bf16, int64_t N, int64_t K, int bits,
                        uint32_t *packed, void *scales_f16, uint8_t *zeros,
                        uint32_t *flags, void *stream);

/*
 * slq_gemm -- fused dequantize-GEMM Y = X W^T with w[n, k] = s[n, g] *
 * (q[n, k] - z[n, g]), g = k / 128; bf16 X, fp32 accumulation, bf16 or fp32 Y.
 *
 * Source: the weight-only quantized linear layer served with mixed per-layer
 * bitwidths, to which the pages credit their 1.7-3.7x serving speedup
 * (gist.science summary, Key Results "Inference Speedup"; GitHub README
 * intro and "4. Build and serve a checkpoint").
 *
 * X_bf16      [M, K] bf16, device.
 * M, N, K     M >= 0, N >= 0 (either 0 launches nothing), K >= 128, K % 128 == 0.
 * bits, packed, scales_f16, zeros   as written by slq_quantize.
 * Y           [M, N] of y_dtype, device, written.  With SLQ_DTYPE_BF16 each
 *             element is the round-to-nearest-even bf16 of the fp32 value the
 *             same kernel writes with SLQ_DTYPE_F32: the order of every sum is
 *             fixed by the sizes and the device, never by timing, so repeated
 *             calls give identical bits.
 * flags       device uint32 or NULL; SLQ_FLAG_TIMEOUT.
 *
 * The kernels this call selects (SLQ_GEMM_GEMV for M <= 16, SLQ_GEMM_TILED
 * above) use no memory beyond their arguments: there is no workspace.
 */
slq_status slq_gemm(const void *X_bf16, int64_t M, int64_t N, int64_t K,
                    int bits, const uint32_t *packed, const void *scales_f16,
                    const uint8_t *zeros, void *Y, slq_dtype y_dtype,
                    uint32_t *flags, void *stream);

/* slq_gemm with an explicit kernel choice (SLQ_GEMM_DECODE and SLQ_GEMM_GEMV
 * need M <= 16).  Only SLQ_GEMM_DECODE needs a workspace, of
 * slq_gemm_workspace_bytes bytes under the workspace rules above, and takes
 * N <= 2097152; `workspace` may be NULL / 0 for every other path and when
 * that size is 0 (SLQ_ERR_INVALID_ARGUMENT if too small).  Same arguments and
 * results otherwise. */
slq_status slq_gemm_ex(const void *X_bf16, int64_t M, int64_t N, int64_t K,
                       int bits, const uint32_t *packed,
                       const void *scales_f16, const uint8_t *zeros, void *Y,
                       slq_dtype y_dtype, slq_gemm_path path, void *workspace,
                       size_t workspace_bytes, uint32_t *flags, void *stream);

/* One layer of slq_gemm_group: Y = X W^T with the arguments of slq_gemm. */
typedef struct {
  const void *X_bf16;        /* [M, K] bf16, device */
  int64_t N, K;              /* N >= 0 (0: the layer is skipped), K >= 128, K % 128 == 0 */
  int bits;                  /* 2..8 */
  const uint32_t *packed;    /* as written by slq_quantize */
  const void *scales_f16;
  const uint8_t *zeros;
  void *Y;                   /* [M, N] of the call's y_dtype, device, written */
} slq_gemm_layer;

/*
 * slq_gemm_group -- several decode-step layers in ONE launch of the
 * SLQ_GEMM_GEMV kernel: for each layer i, Y_i = X_i W_i^T.
 *
 * Source: the pages serve every linear layer of a block at its own bitwidth
 * (GitHub README, "4. Build and serve a checkpoint"; gist.science summary,
 * Key Results "Inference Speedup").  The projections that read the same
 * input in a decoder block (q, k, v; gate, up) can run as one launch even
 * when their b differ, which removes the per-launch start and tail costs
 * that dominate decode-sized layers.
 *
 * layers      host array of `count` slq_gemm_layer; any mix of b, N and K.
 * count       1 .. slq_gemm_group_max().
 * M           0..16 (0 launches nothing), shared by the layers.
 * y_dtype, flags, stream   as for slq_gemm.
 *
 * Each Y_i meets slq_gemm's tolerance, and repeated calls with the same
 * layers give identical bits; the order of the K-split sum follows the
 * group's size, so Y_i may differ in the last bits from a single-layer call.
 * No output may overlap any layer's inputs or another output
 * (SLQ_ERR_INVALID_ARGUMENT); every layer is validated as in slq_gemm.
 */
slq_status slq_gemm_group(const slq_gemm_layer *layers, int count, int64_t M,
                          slq_dtype y_dtype, uint32_t *flags, void *stream);

/* Most layers slq_gemm_group takes in one call (8). */
int slq_gemm_group_max(void);

/*
 * slq_gemm_decode_static -- slq_gemm for decode batches (M <= 16) that
 * allocates nothing and takes no workspace.
 *
 * The pages have no counterpart to this call; it exists for callers that
 * cannot obtain device memory for the workspace slq_gemm needs: a plugin run
 * inside a host engine that owns every device allocation and hands it only
 * the layer's tensors, or a decode loop that must not call cudaMalloc
 * (which may synchronize the device) once it is running.
 *
 * The decode kernel's split-K partial sums and tile counters live in a fixed
 * array of SLQ_DECODE_STATIC_SCRATCH_BYTES bytes inside the library, one per
 * device that loads it, held until the process exits.  Each call clears the
 * counters (an asynchronous memset on `stream`) and then runs the same kernel
 * as slq_gemm_ex(..., SLQ_GEMM_DECODE, ...), with the same results.
 *
 * Arguments, layouts and results are those of slq_gemm, without workspace.
 *   M            0..16; larger M gives SLQ_ERR_INVALID_ARGUMENT.
 *   It runs the SLQ_GEMM_DECODE kernel; layers whose workspace for it
 *   (slq_gemm_workspace_bytes) exceeds SLQ_DECODE_STATIC_SCRATCH_BYTES give
 *   SLQ_ERR_INVALID_ARGUMENT.
 *
 * Every call shares the one array of its device: calls that may run at the
 * same time on the GPU (different streams, or several host threads) race on
 * it and give wrong results; issue them one after another on one stream.
 * The first call on a device looks up the array's device address (with that
 * device current), and so does the first call after the device was reset
 * (cudaDeviceReset gives it a new copy of the array); make such a call before
 * any stream capture.
 */
#define SLQ_DECODE_STATIC_SCRATCH_BYTES ((size_t)8 << 20)

slq_status slq_gemm_decode_static(const void *X_bf16, int64_t M, int64_t N,
                                  int64_t K, int bits, const uint32_t *packed,
                                  const void *scales_f16, const uint8_t *zeros,
                                  void *Y, slq_dtype y_dtype, uint32_t *flags,
                                  void *stream);

/*
 * slq_ear_kl -- per-token Expected Acceptance Rate and KL divergence between
 * the next-token distributions of a reference and a quantized model.
 *
 * Source: gist.science summary, Methodology section 2 "Fidelity Metrics"
 * (EAR = sum over tokens of min(p, q), averaged over positions; KL as the
 * task-lossless search signal) and the reddit abstract (EAR is the maximum
 * token-agreement probability under optimal coupling).  The pages restrict
 * the sum to the top-K tokens in their evaluation; this call sums over the
 * whole vocabulary (K = V).  With x = a / temperature, y = b / temperature,
 * p = softmax(x), q = softmax(y):
 *   ear_tok[t] = sum_v min(p_v, q_v)
 *   kl_tok[t]  = sum_v p_v (log p_v - log q_v)        (nats)
 *
 * logits_p_bf16  [T, V] bf16, device: reference-model logits (p).
 * logits_q_bf16  [T, V] bf16, device: quantized-model logits (q).
 * T, V           T >= 0 (0 launches nothing), V >= 1.
 * temperature    finite, > 0.
 * ear_tok, kl_tok  [T] fp32, device, written.
 * ear_mean, kl_mean  device double or NULL: the mean over the T tokens.
 * flags          device uint32 or NULL; SLQ_FLAG_TIMEOUT.
 */
slq_status slq_ear_kl(const void *logits_p_bf16, const void *logits_q_bf16,
                      int64_t T, int64_t V, float temperature, float *ear_tok,
                      float *kl_tok, double *ear_mean, double *kl_mean,
                      uint32_t *flags, void *stream);

/*
 * slq_ear_kl_topk -- the top-K form of slq_ear_kl, the one the pages' search
 * and evaluation use: EAR = (1/N) sum_i sum_{k=1..K} min(p_i(k), q_i(k))
 * restricted to the top-K tokens (gist.science summary, Methodology section 2
 * "Fidelity Metrics", Definition; GitHub README "2. Build the sensitivity
 * database": top-K = 10).  Readings where the pages are open: the top-K set
 * T_t is the K largest reference logits of token t (ties to the lower
 * index); EAR sums min(p, q) over T_t with p, q the full-vocabulary
 * softmaxes; KL is KL(p_T || q_T) with p and q renormalized over T_t.  With
 * K = V both equal slq_ear_kl.
 *
 * top_k        1 .. min(V, slq_ear_kl_topk_max()) (16); other arguments,
 *              layouts and errors as for slq_ear_kl.
 */
slq_status slq_ear_kl_topk(const void *logits_p_bf16, const void *logits_q_bf16,
                           int64_t T, int64_t V, int top_k, float temperature,
                           float *ear_tok, float *kl_tok, double *ear_mean,
                           double *kl_mean, uint32_t *flags, void *stream);

/* Largest top_k slq_ear_kl_topk takes (16). */
int slq_ear_kl_topk_max(void);

/*
 * slq_grid_noise -- per-group rounding noise of the asymmetric b-bit grid
 * (the format's) and of the symmetric one it replaces.
 *
 * Source: wispaper.ai blog, the section on the gamma^2 variance law, and the
 * gist.science summary, Methodology section 1 "Theoretical Foundation": for a
 * group with range R = max w - min w and largest magnitude M = max |w|,
 * gamma = 2 M / R; a symmetric grid over [-M, M] has gamma times the step of
 * an asymmetric grid over [min w, max w], so gamma^2 times its rounding-noise
 * variance.  For every 128-weight group g (row n, groups along K) this call
 * writes, with L = 2^bits - 1:
 *   gamma[g]    = 2 M / R, or 1 when R = 0
 *   sse_asym[g] = sum over the group of (w - nearest point of
 *                 {min w + i R / L : i = 0..L})^2
 *   sse_sym[g]  = the same for {-M + i 2 M / L : i = 0..L}
 * The grids are continuous (no fp16 scale or integer zero point): this is the
 * quantity the pages' variance argument speaks of, not the stored format's
 * error.  Group statistics are exact; per-weight errors are binary32.
 *
 * W_bf16     [N, K] row-major bf16, device, 16-byte aligned.
 * N, K       N >= 0 (0 launches nothing), K a positive multiple of 128.
 * bits       2..8.
 * gamma, sse_asym, sse_sym  [N, K / 128] fp32, device, written; disjoint
 *            from W.
 * flags      device uint32 or NULL: SLQ_FLAG_NONFINITE when a group holds a
 *            NaN or an infinity (that group's outputs are then meaningless).
 * Errors: SLQ_ERR_INVALID_ARGUMENT for sizes, bits, alignment or overlap
 * before any launch; SLQ_ERR_CUDA for a failed launch.
 */
slq_status slq_grid_noise(const void *W_bf16, int64_t N, int64_t K, int bits,
                          float *gamma, float *sse_asym, float *sse_sym,
                          uint32_t *flags, void *stream);

/*
 * slq_gptq -- GPTQ encode of W with calibration rows X into the same format
 * as slq_quantize (asymmetric INT-`bits`, groups of 128 along K, fp16 scales,
 * uint8 zeros, LSB-first packed codes).
 *
 * Source: the pages' encoder is layer-wise GPTQ at every b with asymmetric
 * INT, group size 128 (GitHub README, "Pipeline" and "1. Quantize"); GPTQ as
 * published by Frantar et al.  Readings where the pages are silent:
 * H = X^T X in binary64; an input column that is always zero gets H_kk = 1
 * and its weights set to 0; damping H += damp * mean(diag H) * I; columns in
 * natural order; a group's scale and zero come from its current, already
 * updated weights at its first column, by slq_quantize's rules; weights are
 * carried in binary64 and rounded to binary32 for each encode; with U the
 * upper Cholesky factor of H^-1 (H^-1 = U^T U), fixing column k with
 * dequantized value d moves every later column j by -(w_k - d) / U_kk * U_kj.
 * Every value is formed by the same sequence of correctly rounded binary64
 * (binary32 for the encode) operations as that definition, so the outputs do
 * not depend on the launch shape.
 *
 * W_bf16     [N, K] row-major bf16, device.  N >= 0 (0 writes nothing).
 * K          a positive multiple of 128, at most 16384.
 * bits       2..8.
 * X_bf16     [T, K] row-major bf16, device: calibration rows, T >= 1.
 * damp       finite, >= 0 (the pages' runs use 0.01).
 * packed, scales_f16, zeros   outputs as for slq_quantize.
 * workspace  device, 16-byte aligned, slq_gptq_workspace_bytes(N, K) bytes
 *            or more, owned by the caller, not read across calls.
 * flags      device uint32 or NULL: SLQ_FLAG_NONFINITE, _SCALE_OVERFLOW as
 *            for slq_quantize; SLQ_FLAG_NOT_POSITIVE_DEFINITE when the damped
 *            H (or its inverse) has a non-positive Cholesky pivot.
 * Runs 6 K/32 + 2 K/128 + 3 launches on `stream`.  Errors:
 * SLQ_ERR_INVALID_ARGUMENT for sizes, alignment, a short workspace or
 * overlapping buffers, before any launch; SLQ_ERR_CUDA for a failed launch.
 */
slq_status slq_gptq(const void *W_bf16, int64_t N, int64_t K, int bits,
                    const void *X_bf16, int64_t T, double damp, uint32_t *packed,
                    void *scales_f16, uint8_t *zeros, void *workspace,
                    size_t workspace_bytes, uint32_t *flags, void *stream);

/* Workspace bytes slq_gptq needs for an [N, K] layer (0 for invalid sizes):
 * three K x K binary64 matrices, the layer in binary64, and 128 binary64
 * errors per row. */
size_t slq_gptq_workspace_bytes(int64_t N, int64_t K);

#ifdef __cplusplus
}
#endif
#endif /* SLQ_H */
