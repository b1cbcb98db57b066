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
// whatever the launch shape.  Parallelism comes from independent elements:
// (i, j) pairs of H and H^-1, rows of a Cholesky column, columns of the
// triangular inverse, rows of W, and (row, column) pairs of each trailing
// update.
//
// Storage (binary64 workspace): Hm holds H, then its lower Cholesky factor
// column-major (element (i, k) at Hm[k K + i]), then H^-1, then the factor of
// H^-1, i.e. U^T (U_kj at Hm[k K + j]); Lr holds L row-major, then the
// inverse's columns transposed; Dg holds the inverse along diagonals
// (Dg[s K + c] = (L^-1)[c + s][c]), the access order of its column sweeps.
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
// Lower Cholesky factor, left-looking, one launch per column j (A symmetric,
// read column-major; column j of L overwrites column j):
//   d = a_jj - sum_{k<j} L_jk^2;  L_jj = sqrt(d);
//   L_ij = (a_ij - sum_{k<j} L_ik L_jk) / L_jj   (i > j).
// Every thread forms d itself (the same operations, so the same value).
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(256) chol_col_kernel(double* __restrict__ A, int K, int j,
                                                       uint32_t* __restrict__ flags) {
  const int i = j + blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= K) return;
  const double* colj = A;  // element (r, k) at A[k K + r]
  double d = A[static_cast<int64_t>(j) * K + j];
  double v = A[static_cast<int64_t>(j) * K + i];
  // Unrolled so that the loads of several steps are in flight: the chains
  // themselves (d and v, in k order) are unchanged.
#pragma unroll 8
  for (int k = 0; k < j; ++k) {
    const double ljk = colj[static_cast<int64_t>(k) * K + j];
    d = __dsub_rn(d, __dmul_rn(ljk, ljk));
    v = __dsub_rn(v, __dmul_rn(colj[static_cast<int64_t>(k) * K + i], ljk));
  }
  if (!(d > 0.0)) {
    if (i == j && flags) atomicOr(flags, kFlagNotPositiveDefinite);
    d = 1.0;  // keep going; the outputs are flagged as unspecified
  }
  d = __dsqrt_rn(d);
  A[static_cast<int64_t>(j) * K + i] = i == j ? d : __ddiv_rn(v, d);
}

// Lr[i][k] = L_ik (row-major, zero above the diagonal) from the column-major factor.
__global__ void __launch_bounds__(256) lower_to_rows_kernel(const double* __restrict__ A, int K,
                                                            double* __restrict__ Lr) {
  __shared__ double tile[kT][kT + 1];
  const int tx = threadIdx.x & 31, ty = threadIdx.x >> 5;
  const int k0 = blockIdx.x * kT, i0 = blockIdx.y * kT;
  for (int r = ty; r < kT; r += 8) tile[r][tx] = A[static_cast<int64_t>(k0 + r) * K + i0 + tx];  // (i0+tx, k0+r)
  __syncthreads();
  for (int r = ty; r < kT; r += 8) {
    const int i = i0 + r, k = k0 + tx;
    Lr[static_cast<int64_t>(i) * K + k] = k <= i ? tile[tx][r] : 0.0;
  }
}

// ---------------------------------------------------------------------------
// Z = L^-1 by forward substitution, one thread per column c:
//   Z_ic = (delta_ic - sum_{k=c}^{i-1} L_ik Z_kc) / L_ii   (i >= c).
// Stored along diagonals, Dg[s K + c] = Z_{c+s, c}, so that the threads of a
// warp read consecutive addresses.
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(128) tri_inverse_kernel(const double* __restrict__ Lr, int K,
                                                          double* __restrict__ Dg) {
  const int c = blockIdx.x * blockDim.x + threadIdx.x;
  const int c0 = blockIdx.x * blockDim.x;  // the warp walks rows together from its first column
  if (c >= K) return;
  for (int i = c0; i < K; ++i) {
    if (i < c) continue;
    const double* li = Lr + static_cast<int64_t>(i) * K + c;  // L_{i, c + s}
    double v = i == c ? 1.0 : 0.0;
    const int n = i - c;
#pragma unroll 8
    for (int s = 0; s < n; ++s) v = __dsub_rn(v, __dmul_rn(li[s], Dg[static_cast<int64_t>(s) * K + c]));
    Dg[static_cast<int64_t>(n) * K + c] = __ddiv_rn(v, Lr[static_cast<int64_t>(i) * K + i]);
  }
}

// ZT[i][k] = Z_ki (zero for k < i) from the diagonal storage.
__global__ void __launch_bounds__(256) diag_to_rows_kernel(const double* __restrict__ Dg, int K,
                                                           double* __restrict__ ZT) {
  const int64_t idx = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (idx >= static_cast<int64_t>(K) * K) return;
  const int i = static_cast<int>(idx / K), k = static_cast<int>(idx % K);
  ZT[idx] = k >= i ? Dg[static_cast<int64_t>(k - i) * K + i] : 0.0;
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
  for (int j = 0; j < K; ++j) {
    chol_col_kernel<<<(K - j + 255) / 256, 256, 0, stream>>>(A, K, j, flags);
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
  lower_to_rows_kernel<<<tiles, 256, 0, stream>>>(ws.hm, k, ws.lr);
  tri_inverse_kernel<<<(k + 127) / 128, 128, 0, stream>>>(ws.lr, k, ws.dg);
  diag_to_rows_kernel<<<static_cast<unsigned>((K * K + 255) / 256), 256, 0, stream>>>(ws.dg, k, ws.lr);
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
