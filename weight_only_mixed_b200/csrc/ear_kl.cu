// ear_kl.cu -- Expected Acceptance Rate and KL(p || q) over softmaxed logits.
//
// Source: pages on "Statistically-Lossless Quantization of Large Language
// Models", gist.science summary, Methodology section 2 "Fidelity Metrics"
// (EAR = sum of min(p, q), averaged over token positions; KL as the
// task-lossless search signal) and the reddit abstract (EAR is the maximum
// token-agreement probability under optimal coupling).  Full-vocabulary form.
//
// Per token, with c = log2(e) / temperature, the kernels work in base 2:
//   S_a = sum_v 2^((a_v - max a) c),   S_b likewise,
//   W   = sum_v 2^((a_v - max a) c) (a_v - b_v),
//   EAR = sum_v 2^(min((a_v - max a) c - log2 S_a, (b_v - max b) c - log2 S_b)),
//   KL  = (W / S_a) / T - ((max a - max b) / T + ln S_a - ln S_b)     [nats]
// which is sum_v p_v (log p_v - log q_v) with p, q the two softmaxes: the
// log-domain form needs no per-element logarithm and has no 0 * log 0 case.
// Differences of two bf16 logits are exact in fp32, so every exponent argument
// is one rounding away from exact.
#include <cooperative_groups.h>
#include <cuda_bf16.h>

#include "internal.h"
#include "ptx.cuh"

namespace cg = cooperative_groups;

namespace slq {
namespace {

constexpr unsigned kFull = 0xffffffffu;

__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

__device__ __forceinline__ float lg2(float x) {
  float y;
  asm("lg2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

__device__ __forceinline__ float bf16_lo(uint32_t v) { return __uint_as_float(v << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t v) { return __uint_as_float(v & 0xffff0000u); }

// Running softmax statistics of one logit stream (base 2, max-shifted).
struct Stat {
  float m;  // running max of the raw logit
  float s;  // sum of 2^((x - m) c)
};

// Online softmax statistics for a and b plus W = sum 2^((a - m_a) c)(a - b).
struct RowStat {
  Stat a, b;
  float w;
};

__device__ __forceinline__ void push(RowStat& st, float a, float b, float c) {
  if (a > st.a.m) {
    const float f = ex2((st.a.m - a) * c);
    st.a.s *= f;
    st.w *= f;
    st.a.m = a;
  }
  const float ea = ex2((a - st.a.m) * c);
  st.a.s += ea;
  st.w += ea * (a - b);
  if (b > st.b.m) {
    st.b.s *= ex2((st.b.m - b) * c);
    st.b.m = b;
  }
  st.b.s += ex2((b - st.b.m) * c);
}

__device__ __forceinline__ void merge_stat(Stat& x, float& wx, const Stat& y, float wy, float c,
                                           bool with_w) {
  if (y.m == -INFINITY) return;
  if (x.m == -INFINITY) {
    x = y;
    if (with_w) wx = wy;
    return;
  }
  const float m = fmaxf(x.m, y.m);
  const float fx = ex2((x.m - m) * c), fy = ex2((y.m - m) * c);
  x.s = x.s * fx + y.s * fy;
  if (with_w) wx = wx * fx + wy * fy;
  x.m = m;
}

__device__ __forceinline__ void merge(RowStat& x, const RowStat& y, float c) {
  float dummy = 0.0f;
  merge_stat(x.a, x.w, y.a, y.w, c, true);
  merge_stat(x.b, dummy, y.b, 0.0f, c, false);
}

__device__ __forceinline__ RowStat shfl_xor(const RowStat& v, int off) {
  RowStat r;
  r.a.m = __shfl_xor_sync(kFull, v.a.m, off);
  r.a.s = __shfl_xor_sync(kFull, v.a.s, off);
  r.b.m = __shfl_xor_sync(kFull, v.b.m, off);
  r.b.s = __shfl_xor_sync(kFull, v.b.s, off);
  r.w = __shfl_xor_sync(kFull, v.w, off);
  return r;
}

// Block-wide reduction of RowStat (fixed order); result valid in every thread.
template <int kThreads>
__device__ RowStat block_reduce(RowStat v, float c) {
  __shared__ RowStat sh[kThreads / 32];
  __shared__ RowStat total;
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) merge(v, shfl_xor(v, off), c);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (lane == 0) sh[warp] = v;
  __syncthreads();
  if (warp == 0) {
    RowStat u = (lane < kThreads / 32) ? sh[lane] : RowStat{{-INFINITY, 0.0f}, {-INFINITY, 0.0f}, 0.0f};
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) merge(u, shfl_xor(u, off), c);
    if (lane == 0) total = u;
  }
  __syncthreads();
  const RowStat r = total;
  __syncthreads();
  return r;
}

template <int kThreads>
__device__ float block_sum(float v) {
  __shared__ float sh[kThreads / 32];
  __shared__ float total;
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) v += __shfl_xor_sync(kFull, v, off);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (lane == 0) sh[warp] = v;
  __syncthreads();
  if (warp == 0) {
    float u = (lane < kThreads / 32) ? sh[lane] : 0.0f;
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) u += __shfl_xor_sync(kFull, u, off);
    if (lane == 0) total = u;
  }
  __syncthreads();
  const float r = total;
  __syncthreads();
  return r;
}

// ---------------------------------------------------------------------------
// Row-per-CTA kernel, any V: pass 1 = online statistics, pass 2 = EAR terms
// (the second read of the row mostly hits L2).  16-byte loads when V % 8 == 0.
// ---------------------------------------------------------------------------
template <int kThreads, bool kVec>
__global__ void __launch_bounds__(kThreads)
    ear_kl_rows_kernel(const uint16_t* __restrict__ A, const uint16_t* __restrict__ Bq, int64_t T,
                       int64_t V, float c, float inv_temp, float* __restrict__ ear_tok,
                       float* __restrict__ kl_tok) {
  for (int64_t t = blockIdx.x; t < T; t += gridDim.x) {
    const uint16_t* a_row = A + t * V;
    const uint16_t* b_row = Bq + t * V;
    RowStat st{{-INFINITY, 0.0f}, {-INFINITY, 0.0f}, 0.0f};
    if constexpr (kVec) {
      const int64_t nv = V / 8;
      for (int64_t i = threadIdx.x; i < nv; i += kThreads) {
        const uint4 va = ld_stream_v4(a_row + 8 * i);
        const uint4 vb = ld_stream_v4(b_row + 8 * i);
        const uint32_t wa[4] = {va.x, va.y, va.z, va.w};
        const uint32_t wb[4] = {vb.x, vb.y, vb.z, vb.w};
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          push(st, bf16_lo(wa[q]), bf16_lo(wb[q]), c);
          push(st, bf16_hi(wa[q]), bf16_hi(wb[q]), c);
        }
      }
    } else {
      for (int64_t v = threadIdx.x; v < V; v += kThreads)
        push(st, __uint_as_float(static_cast<uint32_t>(a_row[v]) << 16),
             __uint_as_float(static_cast<uint32_t>(b_row[v]) << 16), c);
    }
    const RowStat tot = block_reduce<kThreads>(st, c);
    const float la = lg2(tot.a.s), lb = lg2(tot.b.s);
    const float ma = tot.a.m, mb = tot.b.m;

    // Pass 2: sum_v 2^min(u_v, w_v), four accumulators per thread.
    float acc[4] = {0.0f, 0.0f, 0.0f, 0.0f};
    if constexpr (kVec) {
      const int64_t nv = V / 8;
      for (int64_t i = threadIdx.x; i < nv; i += kThreads) {
        const uint4 va = ld_ro_v4(a_row + 8 * i);
        const uint4 vb = ld_ro_v4(b_row + 8 * i);
        const uint32_t wa[4] = {va.x, va.y, va.z, va.w};
        const uint32_t wb[4] = {vb.x, vb.y, vb.z, vb.w};
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          acc[q] += ex2(fminf((bf16_lo(wa[q]) - ma) * c - la, (bf16_lo(wb[q]) - mb) * c - lb));
          acc[q] += ex2(fminf((bf16_hi(wa[q]) - ma) * c - la, (bf16_hi(wb[q]) - mb) * c - lb));
        }
      }
    } else {
      int q = 0;
      for (int64_t v = threadIdx.x; v < V; v += kThreads) {
        const float a = __uint_as_float(static_cast<uint32_t>(a_row[v]) << 16);
        const float b = __uint_as_float(static_cast<uint32_t>(b_row[v]) << 16);
        acc[q] += ex2(fminf((a - ma) * c - la, (b - mb) * c - lb));
        q = (q + 1) & 3;
      }
    }
    const float ear = block_sum<kThreads>((acc[0] + acc[1]) + (acc[2] + acc[3]));
    if (threadIdx.x == 0) {
      constexpr float kLn2 = 0.693147180559945309f;
      ear_tok[t] = ear;
      kl_tok[t] = (tot.w / tot.a.s) * inv_temp - ((ma - mb) * inv_temp + (la - lb) * kLn2);
    }
  }
}

// ---------------------------------------------------------------------------
// Cluster kernel (V % 8 == 0): one HBM pass.  A cluster of CS CTAs (8, or 16
// where the GPU allows it) owns one token row at a time; CTA r keeps slice r
// of both logit rows in shared memory (double-buffered 1-D bulk copies: the
// next row lands while this one is processed).  Per row: one pass of online
// softmax statistics (running max with rescaling) -> one block reduction ->
// the statistics are exchanged through distributed shared memory and merged
// in rank order -> the EAR sum over the resident slice.  Rank 0 adds the EAR
// partials of row i after the exchange of row i+1, so each row costs a single
// cluster barrier.
// ---------------------------------------------------------------------------
constexpr int kClusterThreads = 512;

struct SliceStat {
  float ma, sa, w, mb, sb;
};

template <int CS>
__global__ void __launch_bounds__(kClusterThreads)
    ear_kl_cluster_kernel(const uint16_t* __restrict__ A, const uint16_t* __restrict__ Bq,
                          int64_t T, int64_t V, int units_per_cta, float c, float inv_temp,
                          float* __restrict__ ear_tok, float* __restrict__ kl_tok,
                          uint32_t* __restrict__ flags) {
  extern __shared__ __align__(128) uint8_t smem[];
  cg::cluster_group cluster = cg::this_cluster();
  const int rank = static_cast<int>(cluster.block_rank());
  const int64_t cluster_id = blockIdx.x / CS;
  const int64_t nclusters = gridDim.x / CS;

  const int64_t v8 = V / 8;
  const int64_t r0 = static_cast<int64_t>(rank) * units_per_cta;
  const int64_t u0 = r0 < v8 ? r0 : v8;
  const int64_t u1 = (u0 + units_per_cta) < v8 ? (u0 + units_per_cta) : v8;
  const int nu = static_cast<int>(u1 - u0);  // 16-byte units of this CTA's slice
  const size_t slice_bytes = static_cast<size_t>(units_per_cta) * 16;

  // [buf][tensor][slice] | barriers | stats[2] | ear[2] | merged
  uint8_t* data = smem;
  uint64_t* full = reinterpret_cast<uint64_t*>(data + 4 * slice_bytes);
  SliceStat* stats = reinterpret_cast<SliceStat*>(full + 2);
  float* ear_part = reinterpret_cast<float*>(stats + 2);
  SliceStat* merged = reinterpret_cast<SliceStat*>(ear_part + 2);
  __shared__ int aborted;

  const int64_t nrows = (T > cluster_id) ? (T - cluster_id + nclusters - 1) / nclusters : 0;

  if (threadIdx.x == 0) {
    mbar_init(&full[0], 1);
    mbar_init(&full[1], 1);
    aborted = 0;
    fence_mbarrier_init();
  }
  __syncthreads();
  cluster.sync();  // every CTA of the cluster is running before any remote access

  auto issue = [&](int64_t i) {
    const int buf = static_cast<int>(i & 1);
    const int64_t t = cluster_id + i * nclusters;
    const uint32_t bytes = static_cast<uint32_t>(nu) * 16;
    mbar_arrive_expect_tx(&full[buf], 2 * bytes);
    if (bytes) {
      bulk_load(data + (2 * buf) * slice_bytes, A + t * V + u0 * 8, bytes, &full[buf]);
      bulk_load(data + (2 * buf + 1) * slice_bytes, Bq + t * V + u0 * 8, bytes, &full[buf]);
    }
  };
  int64_t issued = 0;
  if (threadIdx.x == 0)
    for (; issued < 2 && issued < nrows; ++issued) issue(issued);

  for (int64_t i = 0; i < nrows; ++i) {
    const int buf = static_cast<int>(i & 1);
    const int64_t t = cluster_id + i * nclusters;
    if (!aborted) {
      if (!mbar_wait_bounded(&full[buf], static_cast<uint32_t>((i >> 1) & 1))) {
        aborted = 1;
        if (flags) atomicOr(flags, kFlagTimeout);
      }
    }
    __syncthreads();
    const bool live = !aborted;
    const uint4* sa4 = reinterpret_cast<const uint4*>(data + (2 * buf) * slice_bytes);
    const uint4* sb4 = reinterpret_cast<const uint4*>(data + (2 * buf + 1) * slice_bytes);

    // One pass of online softmax statistics over the resident slice.
    RowStat st{{-INFINITY, 0.0f}, {-INFINITY, 0.0f}, 0.0f};
    if (live) {
      for (int k = threadIdx.x; k < nu; k += kClusterThreads) {
        const uint4 va = sa4[k], vb = sb4[k];
        const uint32_t wa[4] = {va.x, va.y, va.z, va.w};
        const uint32_t wb[4] = {vb.x, vb.y, vb.z, vb.w};
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          push(st, bf16_lo(wa[q]), bf16_lo(wb[q]), c);
          push(st, bf16_hi(wa[q]), bf16_hi(wb[q]), c);
        }
      }
    }
    const RowStat tot = block_reduce<kClusterThreads>(st, c);
    if (threadIdx.x == 0) stats[buf] = SliceStat{tot.a.m, tot.a.s, tot.w, tot.b.m, tot.b.s};

    cluster.sync();  // statistics of row i (and EAR partials of row i-1) are visible

    if (threadIdx.x < 32) {
      // Merge the CS slices in rank order (lane 0 does the fixed-order sums).
      SliceStat r = {-INFINITY, 0.0f, 0.0f, -INFINITY, 0.0f};
      if (threadIdx.x < CS) r = cluster.map_shared_rank(stats, static_cast<int>(threadIdx.x))[buf];
      float prev_ear = 0.0f;
      if (rank == 0 && i > 0 && threadIdx.x < CS)
        prev_ear = cluster.map_shared_rank(ear_part, static_cast<int>(threadIdx.x))[buf ^ 1];
      float Ma = -INFINITY, Mb = -INFINITY;
#pragma unroll
      for (int j = 0; j < CS; ++j) {
        Ma = fmaxf(Ma, __shfl_sync(kFull, r.ma, j));
        Mb = fmaxf(Mb, __shfl_sync(kFull, r.mb, j));
      }
      float Sa = 0.0f, Sb = 0.0f, W = 0.0f, E = 0.0f;
#pragma unroll
      for (int j = 0; j < CS; ++j) {
        const float ma = __shfl_sync(kFull, r.ma, j), mb = __shfl_sync(kFull, r.mb, j);
        const float sa = __shfl_sync(kFull, r.sa, j), sb = __shfl_sync(kFull, r.sb, j);
        const float w = __shfl_sync(kFull, r.w, j);
        E += __shfl_sync(kFull, prev_ear, j);
        if (ma != -INFINITY) {
          const float f = ex2((ma - Ma) * c);
          Sa = fmaf(sa, f, Sa);
          W = fmaf(w, f, W);
        }
        if (mb != -INFINITY) Sb = fmaf(sb, ex2((mb - Mb) * c), Sb);
      }
      if (threadIdx.x == 0) {
        *merged = SliceStat{Ma, Sa, W, Mb, Sb};
        if (rank == 0) {
          constexpr float kLn2 = 0.693147180559945309f;
          if (live)
            kl_tok[t] = (W / Sa) * inv_temp - ((Ma - Mb) * inv_temp + (lg2(Sa) - lg2(Sb)) * kLn2);
          if (i > 0) ear_tok[t - nclusters] = E;
        }
      }
    }
    __syncthreads();
    const SliceStat g = *merged;
    const float la = lg2(g.sa), lb = lg2(g.sb);

    // EAR terms of the resident slice: sum 2^min(log2 p, log2 q).
    float e_acc[2] = {0.0f, 0.0f};
    if (live) {
      for (int k = threadIdx.x; k < nu; k += kClusterThreads) {
        const uint4 va = sa4[k], vb = sb4[k];
        const uint32_t wa[4] = {va.x, va.y, va.z, va.w};
        const uint32_t wb[4] = {vb.x, vb.y, vb.z, vb.w};
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          e_acc[q & 1] += ex2(fminf((bf16_lo(wa[q]) - g.ma) * c - la, (bf16_lo(wb[q]) - g.mb) * c - lb));
          e_acc[q & 1] += ex2(fminf((bf16_hi(wa[q]) - g.ma) * c - la, (bf16_hi(wb[q]) - g.mb) * c - lb));
        }
      }
    }
    const float es = block_sum<kClusterThreads>(e_acc[0] + e_acc[1]);
    if (threadIdx.x == 0) ear_part[buf] = es;
    // block_sum ended with __syncthreads: every read of this buffer is done.
    if (threadIdx.x == 0 && !aborted && issued < nrows && issued == i + 2) {
      fence_proxy_async_smem();
      issue(issued);
      ++issued;
    }
  }
  cluster.sync();  // EAR partials of the last row are visible
  if (rank == 0 && threadIdx.x == 0 && nrows > 0) {
    const int buf = static_cast<int>((nrows - 1) & 1);
    float e = 0.0f;
    for (int j = 0; j < CS; ++j) e += cluster.map_shared_rank(ear_part, j)[buf];
    ear_tok[cluster_id + (nrows - 1) * nclusters] = e;
  }
  // Copies issued but never consumed (only after a timeout) must land first.
  if (threadIdx.x == 0 && aborted) {
    for (int64_t i = (issued > 2 ? issued - 2 : 0); i < issued; ++i)
      mbar_wait_bounded(&full[i & 1], static_cast<uint32_t>((i >> 1) & 1));
  }
  cluster.sync();  // keep shared memory alive until rank 0 has read it
}

// Means over tokens in binary64, one block, fixed summation order.
__global__ void __launch_bounds__(1024)
    token_mean_kernel(const float* __restrict__ ear_tok, const float* __restrict__ kl_tok,
                      int64_t T, double* __restrict__ ear_mean, double* __restrict__ kl_mean) {
  __shared__ double se[1024], sk[1024];
  double e = 0.0, k = 0.0;
  for (int64_t t = threadIdx.x; t < T; t += 1024) {
    e += static_cast<double>(ear_tok[t]);
    k += static_cast<double>(kl_tok[t]);
  }
  se[threadIdx.x] = e;
  sk[threadIdx.x] = k;
  __syncthreads();
  for (int s = 512; s > 0; s >>= 1) {
    if (static_cast<int>(threadIdx.x) < s) {
      se[threadIdx.x] += se[threadIdx.x + s];
      sk[threadIdx.x] += sk[threadIdx.x + s];
    }
    __syncthreads();
  }
  if (threadIdx.x == 0) {
    if (ear_mean) *ear_mean = se[0] / static_cast<double>(T);
    if (kl_mean) *kl_mean = sk[0] / static_cast<double>(T);
  }
}

constexpr size_t kClusterSmemExtra = 16 + 2 * sizeof(SliceStat) + 8 + sizeof(SliceStat) + 64;

// Launch the cluster kernel with CS CTAs per cluster if the GPU can keep such
// clusters resident; returns the number of resident CTAs it would use (0 if
// the configuration is impossible) and launches only when `launch` is set.
template <int CS>
int64_t cluster_launch(bool launch, const uint16_t* a, const uint16_t* b, int64_t T, int64_t V,
                       float c, float inv_temp, float* ear_tok, float* kl_tok, uint32_t* flags,
                       cudaStream_t stream, cudaError_t* err) {
  const int64_t v8 = V / 8;
  const int64_t upc = (v8 + CS - 1) / CS;
  const size_t smem = static_cast<size_t>(4 * upc * 16) + kClusterSmemExtra;
  if (smem > 220 * 1024) return 0;
  if (cudaFuncSetAttribute(ear_kl_cluster_kernel<CS>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           static_cast<int>(smem)) != cudaSuccess) {
    cudaGetLastError();
    return 0;
  }
  if (CS > 8 && cudaFuncSetAttribute(ear_kl_cluster_kernel<CS>,
                                     cudaFuncAttributeNonPortableClusterSizeAllowed, 1) != cudaSuccess) {
    cudaGetLastError();
    return 0;
  }
  cudaLaunchConfig_t cfg = {};
  cfg.blockDim = dim3(kClusterThreads, 1, 1);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = CS;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  cfg.gridDim = dim3(CS * 32, 1, 1);
  int max_clusters = 0;
  if (cudaOccupancyMaxActiveClusters(&max_clusters, ear_kl_cluster_kernel<CS>, &cfg) != cudaSuccess)
    max_clusters = 0;
  cudaGetLastError();
  if (max_clusters <= 0) return 0;
  const int64_t nc = T < max_clusters ? T : max_clusters;
  if (launch) {
    cfg.gridDim = dim3(static_cast<unsigned>(CS * nc), 1, 1);
    *err = cudaLaunchKernelEx(&cfg, ear_kl_cluster_kernel<CS>, a, b, T, V, static_cast<int>(upc),
                              c, inv_temp, ear_tok, kl_tok, flags);
  }
  return static_cast<int64_t>(max_clusters) * CS;
}

}  // namespace

cudaError_t launch_ear_kl(const uint16_t* a, const uint16_t* b, int64_t T, int64_t V,
                          float temperature, float* ear_tok, float* kl_tok, double* ear_mean,
                          double* kl_mean, uint32_t* flags, cudaStream_t stream) {
  int sms = 148, dev = 0;
  if (cudaGetDevice(&dev) == cudaSuccess)
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const float inv_temp = 1.0f / temperature;
  const float c = 1.4426950408889634f * inv_temp;
  cudaError_t err = cudaSuccess;

  // Single-pass cluster kernel when rows are 16-byte aligned and the slices
  // fit in shared memory; the configuration with more resident CTAs wins
  // (16-CTA clusters halve the slice, so two CTAs can share an SM).  The row
  // kernel covers every other case.
  bool done = false;
  if (V % 8 == 0) {
    const int64_t r16 = cluster_launch<16>(false, a, b, T, V, c, inv_temp, ear_tok, kl_tok, flags, stream, &err);
    const int64_t r8 = cluster_launch<8>(false, a, b, T, V, c, inv_temp, ear_tok, kl_tok, flags, stream, &err);
    if (r16 > 0 && r16 >= r8) {
      cluster_launch<16>(true, a, b, T, V, c, inv_temp, ear_tok, kl_tok, flags, stream, &err);
      done = true;
    } else if (r8 > 0) {
      cluster_launch<8>(true, a, b, T, V, c, inv_temp, ear_tok, kl_tok, flags, stream, &err);
      done = true;
    }
    if (err != cudaSuccess) return err;
  }
  if (!done) {
    constexpr int kThreads = 1024;
    const int64_t blocks = T < static_cast<int64_t>(sms) * 2 ? T : static_cast<int64_t>(sms) * 2;
    if (V % 8 == 0)
      ear_kl_rows_kernel<kThreads, true><<<static_cast<unsigned>(blocks), kThreads, 0, stream>>>(
          a, b, T, V, c, inv_temp, ear_tok, kl_tok);
    else
      ear_kl_rows_kernel<kThreads, false><<<static_cast<unsigned>(blocks), kThreads, 0, stream>>>(
          a, b, T, V, c, inv_temp, ear_tok, kl_tok);
    err = cudaGetLastError();
    if (err != cudaSuccess) return err;
  }
  if (ear_mean || kl_mean) {
    token_mean_kernel<<<1, 1024, 0, stream>>>(ear_tok, kl_tok, T, ear_mean, kl_mean);
    err = cudaGetLastError();
  }
  return err;
}

}  // namespace slq
