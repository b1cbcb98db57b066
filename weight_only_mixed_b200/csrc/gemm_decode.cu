// gemm_decode.cu -- decode-shaped dequantize-GEMM, Y = X W^T for M <= 16.
//
// The layer the pages credit with the serving speedup (gist.science summary,
// Key Results "Inference Speedup": weight-only mixed-bitwidth kernels in vLLM;
// GitHub README intro).  At decode sizes the layer is bound by HBM bandwidth
// on the packed weights, so the kernel streams each packed word exactly once,
// dequantizes in registers and never stages weights through shared memory.
//
// Work split.  A warp owns RT tiles of 16 weight rows (n) and a set of 128-wide
// groups along K; lane (r = lane/4, t = lane%4) reads, for rows r and r+8 of
// each tile, the b words [t*b, t*b + b) of every group -- the 32 codes
// [32t, 32t+32) of that row's group.  The 4 warps of a CTA take interleaved
// groups of the CTA's K slice; the C CTAs of a cluster (1 x C) take contiguous
// K slices, and the partial sums meet through distributed shared memory in a
// fixed order (deterministic, no atomics, no global workspace).
//
// Arithmetic.  The contraction runs on the tensor cores through
// mma.m16n8k16 (bf16 x bf16 -> fp32) with the weights as the 16-row A operand
// and X^T as the 8-column B operand (M <= 8: one n8 tile; M <= 16: two).
// Because the k order inside a group is free, each lane's codes are fed in the
// order its bit-unpacking produces them and its X values are permuted the same
// way.  Codes become exact bf16 values of (q - z) with the integer-in-mantissa
// trick: OR the code into the mantissa of bf16 128.0 (0x4300) and subtract
// bf16 (128 + z); both steps are exact for codes below 128 (b <= 7); b = 8 goes
// through binary32 (2^23 + q) - (2^23 + z) instead.  The fp16 scale of the
// group multiplies the group's fp32 partial sum, so the only rounding is the
// fp32 accumulation itself.
#include <cooperative_groups.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include "internal.h"
#include "ptx.cuh"

namespace cg = cooperative_groups;

namespace slq {
namespace {

constexpr int kWarps = 4;
constexpr int kThreads = kWarps * 32;
constexpr int kMaxCluster = 8;

// ---------------------------------------------------------------------------
// Packed-word loads: b words of one lane, aligned as the layout allows.
// ---------------------------------------------------------------------------
template <int B>
__device__ __forceinline__ void load_lane_words(const uint32_t* p, uint32_t (&w)[B]) {
  if constexpr (B == 2) {
    const uint2 v = ld_stream_v2(p);
    w[0] = v.x; w[1] = v.y;
  } else if constexpr (B == 4) {
    const uint4 v = ld_stream_v4(p);
    w[0] = v.x; w[1] = v.y; w[2] = v.z; w[3] = v.w;
  } else if constexpr (B == 8) {
    const uint4 v0 = ld_stream_v4(p);
    const uint4 v1 = ld_stream_v4(p + 4);
    w[0] = v0.x; w[1] = v0.y; w[2] = v0.z; w[3] = v0.w;
    w[4] = v1.x; w[5] = v1.y; w[6] = v1.z; w[7] = v1.w;
  } else if constexpr (B == 6) {
#pragma unroll
    for (int i = 0; i < 3; ++i) {
      const uint2 v = ld_ro_v2(p + 2 * i);
      w[2 * i] = v.x; w[2 * i + 1] = v.y;
    }
  } else {
#pragma unroll
    for (int i = 0; i < B; ++i) w[i] = ld_ro_u32(p + i);
  }
}

// ---------------------------------------------------------------------------
// Pair order: the 32 codes of a lane become 16 bf16x2 registers; pair p holds
// codes (lo(p), hi(p)) of the lane's 32.  X is permuted identically.
// ---------------------------------------------------------------------------
template <int B>
__host__ __device__ constexpr int pair_lo(int p) {
  if constexpr (B == 2) return 16 * (p / 8) + (p % 8);
  else if constexpr (B == 4) return 8 * (p / 4) + (p % 4);
  else return 2 * p;
}
template <int B>
__host__ __device__ constexpr int pair_hi(int p) {
  if constexpr (B == 2) return 16 * (p / 8) + (p % 8) + 8;
  else if constexpr (B == 4) return 8 * (p / 4) + (p % 4) + 4;
  else return 2 * p + 1;
}

__device__ __forceinline__ uint32_t bf16x2_sub(uint32_t a, uint32_t b) {
  __nv_bfloat162 r = __hsub2(*reinterpret_cast<__nv_bfloat162*>(&a),
                             *reinterpret_cast<__nv_bfloat162*>(&b));
  return *reinterpret_cast<uint32_t*>(&r);
}

// Code i (0..31) of the lane's B-word stream.
template <int B>
__device__ __forceinline__ uint32_t code_at(const uint32_t (&w)[B], int i) {
  const int o = B * i;
  const int wi = o >> 5;
  const int sh = o & 31;
  constexpr uint32_t mask = (1u << B) - 1u;
  if (sh + B <= 32) return (w[wi] >> sh) & mask;
  return __funnelshift_r(w[wi], w[wi + 1], sh) & mask;
}

// 16 bf16x2 registers of (q - z), exact, in pair order.
template <int B>
__device__ __forceinline__ void dequant_pairs(const uint32_t (&w)[B], uint32_t z,
                                              uint32_t (&a)[16]) {
  if constexpr (B == 8) {
    const float zf = __uint_as_float(0x4B000000u | z);  // 2^23 + z
#pragma unroll
    for (int i = 0; i < 8; ++i) {
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const float lo = __uint_as_float(__byte_perm(w[i], 0x4B000000u, 0x7540 | (2 * h)));
        const float hi = __uint_as_float(__byte_perm(w[i], 0x4B000000u, 0x7540 | (2 * h + 1)));
        __nv_bfloat162 v = __floats2bfloat162_rn(__fsub_rn(lo, zf), __fsub_rn(hi, zf));
        a[2 * i + h] = *reinterpret_cast<uint32_t*>(&v);
      }
    }
  } else {
    const uint32_t z2 = (0x4300u | z) * 0x00010001u;  // bf16x2 (128 + z, 128 + z)
    if constexpr (B == 2) {
#pragma unroll
      for (int i = 0; i < 2; ++i)
#pragma unroll
        for (int j = 0; j < 8; ++j)
          a[8 * i + j] = bf16x2_sub(((w[i] >> (2 * j)) & 0x00030003u) | 0x43004300u, z2);
    } else if constexpr (B == 4) {
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j)
          a[4 * i + j] = bf16x2_sub(((w[i] >> (4 * j)) & 0x000F000Fu) | 0x43004300u, z2);
    } else {
#pragma unroll
      for (int p = 0; p < 16; ++p) {
        const uint32_t lo = code_at<B>(w, 2 * p);
        const uint32_t hi = code_at<B>(w, 2 * p + 1);
        a[p] = bf16x2_sub(lo | (hi << 16) | 0x43004300u, z2);
      }
    }
  }
}

// X values of one lane (32 bf16 in 16 words) permuted into pair order.
template <int B>
__device__ __forceinline__ void permute_x(const uint32_t (&x)[16], uint32_t (&b)[16]) {
#pragma unroll
  for (int p = 0; p < 16; ++p) {
    const int lo = pair_lo<B>(p), hi = pair_hi<B>(p);
    if (hi == lo + 1 && (lo % 2) == 0) {
      b[p] = x[lo / 2];
    } else {
      const uint32_t sel = ((lo & 1) ? 0x32u : 0x10u) | (((hi & 1) ? 0x76u : 0x54u) << 8);
      b[p] = __byte_perm(x[lo / 2], x[hi / 2], sel);
    }
  }
}

__device__ __forceinline__ void mma_bf16_16816(float (&d)[4], uint32_t a0, uint32_t a1,
                                               uint32_t a2, uint32_t a3, uint32_t b0,
                                               uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 "
      "{%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, {%0, %1, %2, %3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// ---------------------------------------------------------------------------
// The kernel.  Grid (ceil(N / 16RT), C), cluster (1, C, 1).
// ---------------------------------------------------------------------------
template <int B, int NT, int RT>
__global__ void __launch_bounds__(kThreads)
    gemm_decode_kernel(const uint16_t* __restrict__ X, int M, int N, int K,
                       const uint32_t* __restrict__ packed, const uint16_t* __restrict__ scales,
                       const uint8_t* __restrict__ zeros, void* __restrict__ Y, int y_f32,
                       int groups_per_slice) {
  constexpr int kRows = 16 * RT;
  constexpr int kCols = 8 * NT;
  __shared__ float red[kWarps][kRows * kCols];
  __shared__ float part[kRows * kCols];

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int r = lane >> 2;
  const int t = lane & 3;
  const int G = K / kGroup;
  const int64_t words_per_row = static_cast<int64_t>(G) * 4 * B;
  const int row0 = blockIdx.x * kRows;
  const int slice = blockIdx.y;
  const int nslices = gridDim.y;
  const int g_begin = slice * groups_per_slice;
  const int g_end = min(G, g_begin + groups_per_slice);

  float acc[RT][NT][4];
#pragma unroll
  for (int i = 0; i < RT; ++i)
#pragma unroll
    for (int j = 0; j < NT; ++j)
#pragma unroll
      for (int e = 0; e < 4; ++e) acc[i][j][e] = 0.0f;

  // Rows of this lane: row0 + 16i + r + 8h.
  int rows[RT][2];
#pragma unroll
  for (int i = 0; i < RT; ++i)
#pragma unroll
    for (int h = 0; h < 2; ++h) rows[i][h] = row0 + 16 * i + r + 8 * h;

  uint32_t wcur[RT][2][B];
  auto load_group = [&](int g, uint32_t (&dst)[RT][2][B]) {
#pragma unroll
    for (int i = 0; i < RT; ++i)
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        if (rows[i][h] < N) {
          load_lane_words<B>(packed + rows[i][h] * words_per_row + static_cast<int64_t>(g) * 4 * B + t * B,
                             dst[i][h]);
        } else {
#pragma unroll
          for (int q = 0; q < B; ++q) dst[i][h][q] = 0u;
        }
      }
  };

  int g = g_begin + warp;
  if (g < g_end) load_group(g, wcur);
  for (; g < g_end; g += kWarps) {
    // Prefetch the next group of this warp while this one is consumed.
    uint32_t wnext[RT][2][B];
    const int gn = g + kWarps;
    if (gn < g_end) load_group(gn, wnext);

    // X fragments: columns m = r + 8j, k in [128g + 32t, 128g + 32t + 32).
    uint32_t xb[NT][16];
#pragma unroll
    for (int j = 0; j < NT; ++j) {
      const int m = r + 8 * j;
      uint32_t raw[16];
      if (m < M) {
        const uint16_t* xp = X + static_cast<int64_t>(m) * K + static_cast<int64_t>(g) * kGroup + 32 * t;
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const uint4 v = ld_ro_v4(xp + 8 * q);
          raw[4 * q] = v.x; raw[4 * q + 1] = v.y; raw[4 * q + 2] = v.z; raw[4 * q + 3] = v.w;
        }
      } else {
#pragma unroll
        for (int q = 0; q < 16; ++q) raw[q] = 0u;
      }
      permute_x<B>(raw, xb[j]);
    }

#pragma unroll
    for (int i = 0; i < RT; ++i) {
      float sc[2];
      uint32_t zz[2];
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const int R = rows[i][h];
        if (R < N) {
          const int64_t gi = static_cast<int64_t>(R) * G + g;
          sc[h] = __half2float(__ushort_as_half(scales[gi]));
          zz[h] = zeros[gi];
        } else {
          sc[h] = 0.0f;
          zz[h] = 0u;
        }
      }
      uint32_t a0[16], a1[16];
      dequant_pairs<B>(wcur[i][0], zz[0], a0);
      dequant_pairs<B>(wcur[i][1], zz[1], a1);
#pragma unroll
      for (int j = 0; j < NT; ++j) {
        float d[4] = {0.0f, 0.0f, 0.0f, 0.0f};
#pragma unroll
        for (int c = 0; c < 8; ++c)
          mma_bf16_16816(d, a0[2 * c], a1[2 * c], a0[2 * c + 1], a1[2 * c + 1], xb[j][2 * c],
                         xb[j][2 * c + 1]);
        acc[i][j][0] += sc[0] * d[0];
        acc[i][j][1] += sc[0] * d[1];
        acc[i][j][2] += sc[1] * d[2];
        acc[i][j][3] += sc[1] * d[3];
      }
    }

    if (gn < g_end) {
#pragma unroll
      for (int i = 0; i < RT; ++i)
#pragma unroll
        for (int h = 0; h < 2; ++h)
#pragma unroll
          for (int q = 0; q < B; ++q) wcur[i][h][q] = wnext[i][h][q];
    }
  }

  // Warp partials -> shared memory; C fragment: rows (r, r+8), cols (2t, 2t+1).
#pragma unroll
  for (int i = 0; i < RT; ++i)
#pragma unroll
    for (int j = 0; j < NT; ++j) {
      const int c0 = 8 * j + 2 * t;
      red[warp][(16 * i + r) * kCols + c0] = acc[i][j][0];
      red[warp][(16 * i + r) * kCols + c0 + 1] = acc[i][j][1];
      red[warp][(16 * i + r + 8) * kCols + c0] = acc[i][j][2];
      red[warp][(16 * i + r + 8) * kCols + c0 + 1] = acc[i][j][3];
    }
  __syncthreads();
  // Entry e = m * kRows + row: consecutive threads take consecutive rows n,
  // so the final stores of Y[m, n] are contiguous in n.
  for (int e = threadIdx.x; e < kRows * kCols; e += kThreads) {
    const int row = e % kRows, m = e / kRows;
    const int idx = row * kCols + m;
    float v = red[0][idx];
#pragma unroll
    for (int w = 1; w < kWarps; ++w) v += red[w][idx];
    part[e] = v;
  }

  auto store = [&](int e, float v) {
    const int n = row0 + e % kRows;
    const int m = e / kRows;
    if (n < N && m < M) {
      const int64_t o = static_cast<int64_t>(m) * N + n;
      if (y_f32)
        static_cast<float*>(Y)[o] = v;
      else
        static_cast<__nv_bfloat16*>(Y)[o] = __float2bfloat16_rn(v);
    }
  };

  if (nslices == 1) {
    __syncthreads();
    for (int e = threadIdx.x; e < kRows * kCols; e += kThreads) store(e, part[e]);
    return;
  }
  cg::cluster_group cluster = cg::this_cluster();
  cluster.sync();  // every CTA's `part` is complete and visible cluster-wide
  if (cluster.block_rank() == 0) {
    for (int e = threadIdx.x; e < kRows * kCols; e += kThreads) {
      float v = part[e];
      for (int c = 1; c < nslices; ++c) v += cluster.map_shared_rank(part, c)[e];
      store(e, v);
    }
  }
  cluster.sync();  // keep every CTA's shared memory alive until rank 0 has read it
}

template <int B, int NT, int RT>
cudaError_t launch_cfg(const uint16_t* X, int M, int N, int K, const uint32_t* packed,
                       const uint16_t* scales, const uint8_t* zeros, void* Y, bool y_f32,
                       cudaStream_t stream) {
  int sms = 148, dev = 0;
  if (cudaGetDevice(&dev) == cudaSuccess)
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const int G = K / kGroup;
  const int row_blocks = (N + 16 * RT - 1) / (16 * RT);
  // Enough CTAs to cover every SM about twice; split K across a cluster when
  // the layer has too few rows for that.
  int C = (2 * sms + row_blocks - 1) / row_blocks;
  if (C > kMaxCluster) C = kMaxCluster;
  if (C > G) C = G;
  if (C < 1) C = 1;
  const int per_slice = (G + C - 1) / C;
  C = (G + per_slice - 1) / per_slice;  // no empty slices

  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(row_blocks), static_cast<unsigned>(C), 1);
  cfg.blockDim = dim3(kThreads, 1, 1);
  cfg.dynamicSmemBytes = 0;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 1;
  attr[0].val.clusterDim.y = static_cast<unsigned>(C);
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, gemm_decode_kernel<B, NT, RT>, X, M, N, K, packed, scales,
                            zeros, Y, y_f32 ? 1 : 0, per_slice);
}

template <int B>
cudaError_t launch_b(const uint16_t* X, int M, int N, int K, const uint32_t* packed,
                     const uint16_t* scales, const uint8_t* zeros, void* Y, bool y_f32,
                     cudaStream_t stream) {
  if (M <= 8) return launch_cfg<B, 1, 2>(X, M, N, K, packed, scales, zeros, Y, y_f32, stream);
  return launch_cfg<B, 2, 2>(X, M, N, K, packed, scales, zeros, Y, y_f32, stream);
}

}  // namespace

cudaError_t launch_gemm_decode(const uint16_t* X, int64_t M, int64_t N, int64_t K, int bits,
                               const uint32_t* packed, const uint16_t* scales,
                               const uint8_t* zeros, void* Y, bool y_f32, cudaStream_t stream) {
  const int m = static_cast<int>(M), n = static_cast<int>(N), k = static_cast<int>(K);
  switch (bits) {
    case 2: return launch_b<2>(X, m, n, k, packed, scales, zeros, Y, y_f32, stream);
    case 3: return launch_b<3>(X, m, n, k, packed, scales, zeros, Y, y_f32, stream);
    case 4: return launch_b<4>(X, m, n, k, packed, scales, zeros, Y, y_f32, stream);
    case 5: return launch_b<5>(X, m, n, k, packed, scales, zeros, Y, y_f32, stream);
    case 6: return launch_b<6>(X, m, n, k, packed, scales, zeros, Y, y_f32, stream);
    case 7: return launch_b<7>(X, m, n, k, packed, scales, zeros, Y, y_f32, stream);
    case 8: return launch_b<8>(X, m, n, k, packed, scales, zeros, Y, y_f32, stream);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace slq
