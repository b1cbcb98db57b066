// gptq.cu -- GPTQ encoder emitting the library's format (asymmetric INT-b,
// groups of 128 along K, fp16 scale, uint8 zero, LSB-first codes).
//
// The pages' encoder is layer-wise GPTQ at every b with this quantizer
// (GitHub README, "Pipeline" and "1. Quantize"; RTN is the baseline).  GPTQ
// (Frantar et al.) encodes each row of W column by column and spreads the
// error of every fixed column over the row's later columns through the upper
// Cholesky factor U of the inverse Hessian H^-1 = (X^T X + damping)^-1, which
// minimizes the change of X W^T on the calibration rows X.
//
// Readings (shared with the oracle, which fixes them): H = X^T X in binary64;
// a column with H_kk = 0 (an input that is always zero) gets H_kk = 1 and its
// weights set to 0; damping H += damp * mean(diag H) * I; natural column order;
// a group's scale and zero come from its current, already updated weights at
// its first column, by the RTN rules; weights carried in binary64 and rounded
// to binary32 for each encode; fixing column k with dequantized value d moves
// every later column j by -(w_k - d) / U_kk * U_kj.
//
// Arithmetic.  Every step is binary64 (binary32 for the encode decisions,
// as the format defines), and every element's value is formed by the same
// sequence of correctly rounded operations as in the definition: each sum
// runs in ascending index order, products and sums are rounded separately
// (explicit __dmul_rn / __dadd_rn / __dsub_rn, no fused multiply-add), and
// the blocked column updates apply a block's 128 terms to every later column
// in column order, exactly as the column-by-column definition does.  The
// codes, scales and zeros are therefore the definition's own, bit for bit,
// whatever the launch shape.  The factorizations run right-looking in blocks
// of 32: a block is finished by one CTA, and the updates it owes every later
// element are applied by a parallel trailing kernel, each element walking the
// block's columns (or rows) in order -- the same subtractions, in the same
// order, as the left-looking definition.  Parallelism comes from independent
// elements: (i, j) pairs of H and H^-1, the trailing elements of each block,
// rows of W, and (row, column) pairs of each group's trailing update.
//
// Storage (binary64 workspace): Hm holds H, then its lower Cholesky factor
// column-major (element (i, k) at Hm[k K + i]), then H^-1, then the factor of
// H^-1, i.e. U^T (U_kj at Hm[k K + j]); Dg holds Z = L^-1 row-major; Lr holds
// Z transposed.
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include "internal.h"

namespace slq {
namespace {

constexpr unsigned kFull = 0xffffffffu;

__device__ __forceinline__ double bf16_to_f64(uint16_t v) {
  return static_cast<double>(__uint_as_float(static_cast<uint32_t>(v) << 16));
}

// ---------------------------------------------------------------------------
// H = X^T X: 32 x 32 tiles of the lower triangle; each element sums over the
// rows t of X in ascending order.
// ---------------------------------------------------------------------------
constexpr int kT = 32;  // tile edge

__global__ void __launch_bounds__(256) hessian_kernel(const uint16_t* __restrict__ X, int64_t T, int K,
                                                      double* __restrict__ H) {
  const int bi = blockIdx.y, bj = blockIdx.x;
  if (bj > bi) return;
  __shared__ double xi[kT][kT + 1], xj[kT][kT + 1];  // [t][i], [t][j]
  const int tx = threadIdx.x & 31, ty = threadIdx.x >> 5;  // 8 rows of threads
  double acc[4] = {0.0, 0.0, 0.0, 0.0};                    // elements (4 ty + e, tx)
  for (int64_t t0 = 0; t0 < T; t0 += kT) {
    for (int r = ty; r < kT; r += 8) {
      const int64_t t = t0 + r;
      xi[r][tx] = t < T ? bf16_to_f64(X[t * K + bi * kT + tx]) : 0.0;
      xj[r][tx] = t < T ? bf16_to_f64(X[t * K + bj * kT + tx]) : 0.0;
    }
    __syncthreads();
    const int tn = T - t0 < kT ? static_cast<int>(T - t0) : kT;
    for (int r = 0; r < tn; ++r) {
      const double b = xj[r][tx];
#pragma unroll
      for (int e = 0; e < 4; ++e) acc[e] = __dadd_rn(acc[e], __dmul_rn(xi[r][4 * ty + e], b));
    }
    __syncthreads();
  }
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    const int i = bi * kT + 4 * ty + e, j = bj * kT + tx;
    if (j <= i) {
      H[static_cast<int64_t>(i) * K + j] = acc[e];
      H[static_cast<int64_t>(j) * K + i] = acc[e];
    }
  }
}

// Dead inputs, then the damping from the mean of the diagonal (summed in
// ascending order by one thread, as the definition does).
__global__ void prep_kernel(double* __restrict__ H, int K, uint8_t* __restrict__ dead,
                            double* __restrict__ mean_out) {
  double mean = 0.0;
  for (int k = 0; k < K; ++k) {
    double& h = H[static_cast<int64_t>(k) * K + k];
    dead[k] = h == 0.0;
    if (h == 0.0) h = 1.0;
    mean = __dadd_rn(mean, h);
  }
  *mean_out = __ddiv_rn(mean, static_cast<double>(K));
}

__global__ void damp_kernel(double* __restrict__ H, int K, double damp, const double* __restrict__ mean) {
  const int k = blockIdx.x * blockDim.x + threadIdx.x;
  if (k < K) {
    double& h = H[static_cast<int64_t>(k) * K + k];
    h = __dadd_rn(h, __dmul_rn(damp, *mean));
  }
}

// ---------------------------------------------------------------------------
// Lower Cholesky factor, A symmetric and column-major (element (i, j) at
// A[j K + i]), overwritten by L.  The definition, per element:
//   d_j = a_jj - sum_{k<j} L_jk L_jk;  L_jj = sqrt(d_j);
//   L_ij = (a_ij - sum_{k<j} L_ik L_jk) / L_jj          (i > j, k ascending).
// Right-looking blocked form with the same per-element sequence: once column
// k is final, every later element (i, j) has L_ik L_jk subtracted, in k order
// -- inside a 32-column panel by one CTA, below and to the right of it by the
// trailing kernel, each element walking the panel's columns in order.
// ---------------------------------------------------------------------------
constexpr int kP = 32;  // panel width (rows of a triangular-inverse block)

__global__ void __launch_bounds__(1024) chol_panel_kernel(double* __restrict__ A, int K, int p0,
                                                          uint32_t* __restrict__ flags) {
  __shared__ double dsh;
  const int pend = p0 + kP;
  for (int j = p0; j < pend; ++j) {
    double* colj = A + static_cast<int64_t>(j) * K;
    if (threadIdx.x == 0) {
      double d = colj[j];
      if (!(d > 0.0)) {
        if (flags) atomicOr(flags, kFlagNotPositiveDefinite);
        d = 1.0;  // keep going; the outputs are flagged as unspecified
      }
      d = __dsqrt_rn(d);
      colj[j] = d;
      dsh = d;
    }
    __syncthreads();
    const double d = dsh;
    for (int i = j + 1 + threadIdx.x; i < K; i += blockDim.x) colj[i] = __ddiv_rn(colj[i], d);
    __syncthreads();
    // The panel's later columns j' (and rows i >= j'): a_ij' -= L_ij L_j'j.
    const int ncol = pend - j - 1;
    if (ncol > 0) {
      const int64_t rows = K - (j + 1);
      for (int64_t idx = threadIdx.x; idx < rows * ncol; idx += blockDim.x) {
        const int jp = j + 1 + static_cast<int>(idx % ncol);
        const int i = j + 1 + static_cast<int>(idx / ncol);
        if (i >= jp) {
          double& a = A[static_cast<int64_t>(jp) * K + i];
          a = __dsub_rn(a, __dmul_rn(colj[i], colj[jp]));
        }
      }
    }
    __syncthreads();
  }
}

// Elements (i, j) with j >= p0 + 32, i >= j: a_ij -= L_ik L_jk for the
// panel's k in order.  64 x 64 tiles of the lower triangle.
constexpr int kC = 64;
__global__ void __launch_bounds__(256) chol_trailing_kernel(double* __restrict__ A, int K, int p0) {
  const int q0 = p0 + kP;
  const int bi = blockIdx.y, bj = blockIdx.x;
  if (bj > bi) return;
  const int i0 = q0 + bi * kC, j0 = q0 + bj * kC;
  __shared__ double li[kP][kC + 1], lj[kP][kC + 1];  // [k][row]
  for (int idx = threadIdx.x; idx < kP * kC; idx += blockDim.x) {
    const int k = idx / kC, r = idx % kC;
    const double* col = A + static_cast<int64_t>(p0 + k) * K;
    li[k][r] = i0 + r < K ? col[i0 + r] : 0.0;
    lj[k][r] = j0 + r < K ? col[j0 + r] : 0.0;
  }
  __syncthreads();
  const int r = threadIdx.x % kC, c0 = threadIdx.x / kC;  // row r, columns c0 + 4 e
  const int i = i0 + r;
  if (i >= K) return;
#pragma unroll 4
  for (int e = 0; e < kC / 4; ++e) {
    const int c = c0 + 4 * e, j = j0 + c;
    if (j >= K || j > i) continue;
    double& a = A[static_cast<int64_t>(j) * K + i];
    double v = a;
    for (int k = 0; k < kP; ++k) v = __dsub_rn(v, __dmul_rn(li[k][r], lj[k][c]));
    a = v;
  }
}

// ---------------------------------------------------------------------------
// Z = L^-1, row-major V (V[i][c] = Z_ic once row i is final).  The
// definition, per element: Z_ic = (delta_ic - sum_{k=c}^{i-1} L_ik Z_kc) /
// L_ii, k ascending.  Right-looking by rows with the same sequence: V starts
// as the identity; once row k is final, every later row i has L_ik Z_kc
// subtracted from V[i][c] for c <= k -- inside a block of 32 rows by one
// CTA, below it by the trailing kernel, each element walking the block's
// rows in order.  L is read from the column-major factor.
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(256) identity_kernel(double* __restrict__ V, int K) {
  const int64_t idx = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (idx < static_cast<int64_t>(K) * K) V[idx] = (idx / K == idx % K) ? 1.0 : 0.0;
}

__global__ void __launch_bounds__(1024) inv_block_kernel(const double* __restrict__ L, int K, int r0,
                                                         double* __restrict__ V) {
  const int rend = r0 + kP;
  for (int i = r0; i < rend; ++i) {
    double* vi = V + static_cast<int64_t>(i) * K;
    const double lii = L[static_cast<int64_t>(i) * K + i];
    for (int c = threadIdx.x; c <= i; c += blockDim.x) vi[c] = __ddiv_rn(vi[c], lii);
    __syncthreads();
    // The block's later rows i' (columns c <= i): v_i'c -= L_i'i Z_ic.
    const int nrow = rend - i - 1;
    if (nrow > 0) {
      const int64_t cols = i + 1;
      for (int64_t idx = threadIdx.x; idx < cols * nrow; idx += blockDim.x) {
        const int ip = i + 1 + static_cast<int>(idx / cols);
        const int c = static_cast<int>(idx % cols);
        double& v = V[static_cast<int64_t>(ip) * K + c];
        v = __dsub_rn(v, __dmul_rn(L[static_cast<int64_t>(i) * K + ip], vi[c]));
      }
    }
    __syncthreads();
  }
}

// Rows i' >= r0 + 32, columns c < r0 + 32: v_i'c -= L_i'k Z_kc for the
// block's rows k >= c, in order.  64 x 64 tiles.
__global__ void __launch_bounds__(256) inv_trailing_kernel(const double* __restrict__ L, int K, int r0,
                                                           double* __restrict__ V) {
  const int i0 = r0 + kP + blockIdx.y * kC, c0 = blockIdx.x * kC;
  __shared__ double lk[kP][kC + 1], zk[kP][kC + 1];  // [k][row i'], [k][column c]
  for (int idx = threadIdx.x; idx < kP * kC; idx += blockDim.x) {
    const int k = idx / kC, r = idx % kC;
    lk[k][r] = i0 + r < K ? L[static_cast<int64_t>(r0 + k) * K + i0 + r] : 0.0;  // L_{i0+r, r0+k}
    zk[k][r] = c0 + r < r0 + kP ? V[static_cast<int64_t>(r0 + k) * K + c0 + r] : 0.0;
  }
  __syncthreads();
  const int c = threadIdx.x % kC, rr = threadIdx.x / kC;  // column c, rows rr + 4 e
  const int cg = c0 + c;
  if (cg >= r0 + kP) return;
  const int kstart = cg > r0 ? cg - r0 : 0;  // the block's rows k >= c
#pragma unroll 4
  for (int e = 0; e < kC / 4; ++e) {
    const int ip = i0 + rr + 4 * e;
    if (ip >= K) continue;
    double& a = V[static_cast<int64_t>(ip) * K + cg];
    double v = a;
    for (int k = kstart; k < kP; ++k) v = __dsub_rn(v, __dmul_rn(lk[k][rr + 4 * e], zk[k][c]));
    a = v;
  }
}

// ZT[i][k] = Z_ki from the row-major V (a tiled transpose; zero above).
__global__ void __launch_bounds__(256) transpose_kernel(const double* __restrict__ V, int K,
                                                        double* __restrict__ ZT) {
  __shared__ double tile[kT][kT + 1];
  const int tx = threadIdx.x & 31, ty = threadIdx.x >> 5;
  const int c0 = blockIdx.x * kT, k0 = blockIdx.y * kT;
  for (int r = ty; r < kT; r += 8) tile[r][tx] = V[static_cast<int64_t>(k0 + r) * K + c0 + tx];  // Z_{k0+r, c0+tx}
  __syncthreads();
  for (int r = ty; r < kT; r += 8) {
    const int i = c0 + r, k = k0 + tx;
    ZT[static_cast<int64_t>(i) * K + k] = k >= i ? tile[tx][r] : 0.0;
  }
}

// H^-1 = Z^T Z: (H^-1)_ij = sum_{k >= max(i, j)} Z_ki Z_kj, ascending k.  The
// terms below max(i, j) are exact zeros, so a sum that starts at the tile's
// first nonzero chunk is the same value.  Lower triangle, written column-major.
__global__ void __launch_bounds__(256) inverse_product_kernel(const double* __restrict__ ZT, int K,
                                                              double* __restrict__ A) {
  const int bi = blockIdx.y, bj = blockIdx.x;
  if (bj > bi) return;
  __shared__ double zi[kT][kT + 1], zj[kT][kT + 1];  // [i][k], [j][k]
  const int tx = threadIdx.x & 31, ty = threadIdx.x >> 5;
  double acc[4] = {0.0, 0.0, 0.0, 0.0};  // elements (4 ty + e, tx)
  for (int k0 = bi * kT; k0 < K; k0 += kT) {
    for (int r = ty; r < kT; r += 8) {
      zi[r][tx] = ZT[static_cast<int64_t>(bi * kT + r) * K + k0 + tx];
      zj[r][tx] = ZT[static_cast<int64_t>(bj * kT + r) * K + k0 + tx];
    }
    __syncthreads();
    for (int k = 0; k < kT; ++k) {
      const double b = zj[tx][k];
#pragma unroll
      for (int e = 0; e < 4; ++e) acc[e] = __dadd_rn(acc[e], __dmul_rn(zi[4 * ty + e][k], b));
    }
    __syncthreads();
  }
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    const int i = bi * kT + 4 * ty + e, j = bj * kT + tx;
    if (j <= i) A[static_cast<int64_t>(j) * K + i] = acc[e];  // column-major (i, j)
  }
}

// ---------------------------------------------------------------------------
// The encode.
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(256) init_rows_kernel(const uint16_t* __restrict__ W, int64_t total, int K,
                                                        const uint8_t* __restrict__ dead,
                                                        double* __restrict__ W64) {
  const int64_t idx = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (idx < total) W64[idx] = dead[idx % K] ? 0.0 : bf16_to_f64(W[idx]);
}

constexpr int kRowsPerCta = 8;  // one warp per row

// One group (128 columns k0 .. k0 + 127) of every row: the group's scale and
// zero from the current weights, then the 128 columns in order, each code
// decided in binary32 and its error spread over the group's later columns.
// The errors e are kept for the trailing update.  Lane l holds columns
// k0 + l + 32 r, r = 0..3.
__global__ void __launch_bounds__(kRowsPerCta * 32) gptq_group_kernel(
    double* __restrict__ W64, int N, int K, int bits, const double* __restrict__ U, int k0,
    double* __restrict__ E, uint32_t* __restrict__ packed, uint16_t* __restrict__ scales,
    uint8_t* __restrict__ zeros, uint32_t* __restrict__ flags) {
  extern __shared__ double ub[];  // [128][128]: ub[kk][jj] = U_{k0+kk, k0+jj}
  __shared__ uint8_t codes[kRowsPerCta][kGroup];
  for (int idx = threadIdx.x; idx < kGroup * kGroup; idx += blockDim.x) {
    const int kk = idx / kGroup, jj = idx % kGroup;
    ub[idx] = U[static_cast<int64_t>(k0 + kk) * K + k0 + jj];
  }
  __syncthreads();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int n = blockIdx.x * kRowsPerCta + warp;
  if (n >= N) return;
  double* row = W64 + static_cast<int64_t>(n) * K + k0;
  double w[4];
#pragma unroll
  for (int r = 0; r < 4; ++r) w[r] = row[lane + 32 * r];

  // Scale and zero by the RTN rules on the binary32 values.
  float fmn = __double2float_rn(w[0]), fmx = fmn;
  bool nonfinite = false;
#pragma unroll
  for (int r = 0; r < 4; ++r) {
    const float f = __double2float_rn(w[r]);
    nonfinite |= !isfinite(f);
    fmn = fminf(fmn, f);
    fmx = fmaxf(fmx, f);
  }
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) {
    fmn = fminf(fmn, __shfl_xor_sync(kFull, fmn, off));
    fmx = fmaxf(fmx, __shfl_xor_sync(kFull, fmx, off));
  }
  nonfinite = __any_sync(kFull, nonfinite);
  const float maxq = static_cast<float>((1 << bits) - 1);
  float lo = fmn, hi = fmx;
  if (hi == lo) {
    if (lo > 0.0f) lo = 0.0f;
    if (hi < 0.0f) hi = 0.0f;
  }
  const float s32 = __fdiv_rn(__fsub_rn(hi, lo), maxq);
  uint16_t s16;
  bool overflow = false;
  if (s32 == 0.0f) {
    s16 = 0x3C00u;
  } else {
    s16 = __half_as_ushort(__float2half_rn(s32));
    if ((s16 & 0x7FFFu) == 0u) {
      s16 = 0x0001u;
    } else if (s16 == 0x7C00u) {
      s16 = 0x7BFFu;
      overflow = true;
    }
  }
  const float s = __half2float(__ushort_as_half(s16));
  float zf = rintf(__fdiv_rn(-lo, s));
  if (zf != zf || zf < 0.0f) zf = 0.0f;
  if (zf > maxq) zf = maxq;
  const double s64 = static_cast<double>(s), z64 = static_cast<double>(zf);

  // The columns in order.
  double* erow = E + static_cast<int64_t>(n) * kGroup;
#pragma unroll
  for (int r = 0; r < 4; ++r) {
#pragma unroll 1
    for (int l = 0; l < 32; ++l) {
      const int kk = 32 * r + l;
      const double wk = __shfl_sync(kFull, w[r], l);
      float v = __fadd_rn(rintf(__fdiv_rn(__double2float_rn(wk), s)), zf);
      if (v != v || v < 0.0f) v = 0.0f;
      if (v > maxq) v = maxq;
      const double d = __dmul_rn(s64, __dsub_rn(static_cast<double>(v), z64));
      const double e = __ddiv_rn(__dsub_rn(wk, d), ub[kk * kGroup + kk]);
      if (lane == l) {
        codes[warp][kk] = static_cast<uint8_t>(v);
        erow[kk] = e;
      }
#pragma unroll
      for (int r2 = 0; r2 < 4; ++r2) {
        const int jj = lane + 32 * r2;
        if (jj > kk) w[r2] = __dsub_rn(w[r2], __dmul_rn(e, ub[kk * kGroup + jj]));
      }
    }
  }
  __syncwarp();
  // Pack the group's 128 codes: word i holds the bits [32 i, 32 i + 32) of
  // the LSB-first stream (4 b words per group).
  const int G = K / kGroup;
  uint32_t* dst = packed + (static_cast<int64_t>(n) * G + k0 / kGroup) * 4 * bits;
  if (lane < 4 * bits) {
    uint32_t word = 0;
    const int bit0 = 32 * lane;
    for (int kk = bit0 / bits; kk < kGroup && kk * bits < bit0 + 32; ++kk) {
      const int pos = kk * bits - bit0;  // may be negative for a code straddling in
      const uint32_t q = codes[warp][kk];
      word |= pos >= 0 ? (q << pos) : (q >> -pos);
    }
    dst[lane] = word;
  }
  if (lane == 0) {
    scales[static_cast<int64_t>(n) * G + k0 / kGroup] = s16;
    zeros[static_cast<int64_t>(n) * G + k0 / kGroup] = static_cast<uint8_t>(zf);
    if (flags && nonfinite) atomicOr(flags, kFlagNonfinite);
    if (flags && overflow) atomicOr(flags, kFlagScaleOverflow);
  }
}

// Trailing update after group k0: w_nj -= e_nk U_kj for k = k0 .. k0 + 127 in
// order, for every row n and column j >= k0 + 128.  Tile: 32 rows x 64
// columns, eight elements per thread.
constexpr int kTrRows = 32, kTrCols = 64;
__global__ void __launch_bounds__(256) trailing_kernel(double* __restrict__ W64, int N, int K,
                                                       const double* __restrict__ U, int k0,
                                                       const double* __restrict__ E) {
  extern __shared__ double sm[];
  double* es = sm;                         // [kTrRows][128]
  double* us = sm + kTrRows * kGroup;      // [128][kTrCols + 1]
  const int n0 = blockIdx.y * kTrRows;
  const int j0 = k0 + kGroup + blockIdx.x * kTrCols;
  for (int idx = threadIdx.x; idx < kTrRows * kGroup; idx += blockDim.x) {
    const int r = idx / kGroup, kk = idx % kGroup;
    es[idx] = n0 + r < N ? E[static_cast<int64_t>(n0 + r) * kGroup + kk] : 0.0;
  }
  for (int idx = threadIdx.x; idx < kGroup * kTrCols; idx += blockDim.x) {
    const int kk = idx / kTrCols, c = idx % kTrCols;
    us[kk * (kTrCols + 1) + c] = j0 + c < K ? U[static_cast<int64_t>(k0 + kk) * K + j0 + c] : 0.0;
  }
  __syncthreads();
  const int c = threadIdx.x % kTrCols, r0 = threadIdx.x / kTrCols;  // 4 row phases
  const int j = j0 + c;
  if (j >= K) return;
  double w[kTrRows / 4];
#pragma unroll
  for (int e = 0; e < kTrRows / 4; ++e) {
    const int n = n0 + r0 + 4 * e;
    w[e] = n < N ? W64[static_cast<int64_t>(n) * K + j] : 0.0;
  }
  for (int kk = 0; kk < kGroup; ++kk) {
    const double u = us[kk * (kTrCols + 1) + c];
#pragma unroll
    for (int e = 0; e < kTrRows / 4; ++e)
      w[e] = __dsub_rn(w[e], __dmul_rn(es[(r0 + 4 * e) * kGroup + kk], u));
  }
#pragma unroll
  for (int e = 0; e < kTrRows / 4; ++e) {
    const int n = n0 + r0 + 4 * e;
    if (n < N) W64[static_cast<int64_t>(n) * K + j] = w[e];
  }
}

struct Ws {
  double *hm, *lr, *dg, *w64, *e, *mean;
  uint8_t* dead;
};

Ws carve(void* base, int64_t N, int64_t K) {
  Ws w;
  double* p = static_cast<double*>(base);
  w.hm = p;
  p += K * K;
  w.lr = p;
  p += K * K;
  w.dg = p;
  p += K * K;
  w.w64 = p;
  p += N * K;
  w.e = p;
  p += N * kGroup;
  w.mean = p;
  p += 2;
  w.dead = reinterpret_cast<uint8_t*>(p);
  return w;
}

cudaError_t cholesky(double* A, int K, uint32_t* flags, cudaStream_t stream) {
  for (int p0 = 0; p0 < K; p0 += kP) {
    chol_panel_kernel<<<1, 1024, 0, stream>>>(A, K, p0, flags);
    const int rest = K - p0 - kP;
    if (rest > 0) {
      const int t = (rest + kC - 1) / kC;
      chol_trailing_kernel<<<dim3(t, t), 256, 0, stream>>>(A, K, p0);
    }
  }
  return cudaGetLastError();
}

// Z = L^-1 into V (row-major), L column-major.
cudaError_t tri_inverse(const double* L, int K, double* V, cudaStream_t stream) {
  identity_kernel<<<static_cast<unsigned>((static_cast<int64_t>(K) * K + 255) / 256), 256, 0, stream>>>(V, K);
  for (int r0 = 0; r0 < K; r0 += kP) {
    inv_block_kernel<<<1, 1024, 0, stream>>>(L, K, r0, V);
    const int rest = K - r0 - kP;
    if (rest > 0)
      inv_trailing_kernel<<<dim3((r0 + kP + kC - 1) / kC, (rest + kC - 1) / kC), 256, 0, stream>>>(L, K, r0, V);
  }
  return cudaGetLastError();
}

}  // namespace

size_t gptq_workspace_bytes(int64_t N, int64_t K) {
  return static_cast<size_t>(3 * K * K + N * K + N * kGroup + 2) * sizeof(double) +
         static_cast<size_t>((K + 15) / 16 * 16);
}

cudaError_t launch_gptq(const uint16_t* W, int64_t N, int64_t K, int bits, const uint16_t* X, int64_t T,
                        double damp, uint32_t* packed, uint16_t* scales, uint8_t* zeros, void* workspace,
                        uint32_t* flags, cudaStream_t stream) {
  const int k = static_cast<int>(K);
  const Ws ws = carve(workspace, N, K);
  const dim3 tiles(k / kT, k / kT);
  hessian_kernel<<<tiles, 256, 0, stream>>>(X, T, k, ws.hm);
  prep_kernel<<<1, 1, 0, stream>>>(ws.hm, k, ws.dead, ws.mean);
  damp_kernel<<<(k + 255) / 256, 256, 0, stream>>>(ws.hm, k, damp, ws.mean);
  cudaError_t e = cholesky(ws.hm, k, flags, stream);
  if (e != cudaSuccess) return e;
  e = tri_inverse(ws.hm, k, ws.dg, stream);
  if (e != cudaSuccess) return e;
  transpose_kernel<<<tiles, 256, 0, stream>>>(ws.dg, k, ws.lr);
  inverse_product_kernel<<<tiles, 256, 0, stream>>>(ws.lr, k, ws.hm);
  e = cholesky(ws.hm, k, flags, stream);  // U^T, column-major: U_kj at hm[k K + j]
  if (e != cudaSuccess) return e;
  if (N == 0) return cudaGetLastError();
  init_rows_kernel<<<static_cast<unsigned>((N * K + 255) / 256), 256, 0, stream>>>(W, N * K, k, ws.dead,
                                                                                  ws.w64);
  static SmemAttr group_attr, trail_attr;
  constexpr int kGroupSmem = kGroup * kGroup * sizeof(double);
  constexpr int kTrailSmem = (kTrRows * kGroup + kGroup * (kTrCols + 1)) * sizeof(double);
  e = group_attr.ensure(gptq_group_kernel, kGroupSmem);
  if (e == cudaSuccess) e = trail_attr.ensure(trailing_kernel, kTrailSmem);
  if (e != cudaSuccess) return e;
  const int n = static_cast<int>(N);
  for (int k0 = 0; k0 < k; k0 += kGroup) {
    gptq_group_kernel<<<(n + kRowsPerCta - 1) / kRowsPerCta, kRowsPerCta * 32, kGroupSmem, stream>>>(
        ws.w64, n, k, bits, ws.hm, k0, ws.e, packed, scales, zeros, flags);
    const int rest = k - k0 - kGroup;
    if (rest > 0) {
      const dim3 grid((rest + kTrCols - 1) / kTrCols, (n + kTrRows - 1) / kTrRows);
      trailing_kernel<<<grid, 256, kTrailSmem, stream>>>(ws.w64, n, k, ws.hm, k0, ws.e);
    }
  }
  return cudaGetLastError();
}

}  // namespace slq
