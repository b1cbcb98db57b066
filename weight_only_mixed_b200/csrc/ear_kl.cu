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
#include <cuda_bf16.h>

#include "internal.h"
#include "ptx.cuh"

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

}  // namespace

cudaError_t launch_ear_kl(const uint16_t* a, const uint16_t* b, int64_t T, int64_t V,
                          float temperature, float* ear_tok, float* kl_tok, double* ear_mean,
                          double* kl_mean, uint32_t* flags, cudaStream_t stream) {
  (void)flags;
  int sms = 148, dev = 0;
  if (cudaGetDevice(&dev) == cudaSuccess)
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const float inv_temp = 1.0f / temperature;
  const float c = 1.4426950408889634f * inv_temp;
  constexpr int kThreads = 1024;
  int64_t blocks = T < static_cast<int64_t>(sms) * 2 ? T : static_cast<int64_t>(sms) * 2;
  if (V % 8 == 0)
    ear_kl_rows_kernel<kThreads, true><<<static_cast<unsigned>(blocks), kThreads, 0, stream>>>(
        a, b, T, V, c, inv_temp, ear_tok, kl_tok);
  else
    ear_kl_rows_kernel<kThreads, false><<<static_cast<unsigned>(blocks), kThreads, 0, stream>>>(
        a, b, T, V, c, inv_temp, ear_tok, kl_tok);
  cudaError_t err = cudaGetLastError();
  if (err != cudaSuccess) return err;
  if (ear_mean || kl_mean) {
    token_mean_kernel<<<1, 1024, 0, stream>>>(ear_tok, kl_tok, T, ear_mean, kl_mean);
    err = cudaGetLastError();
  }
  return err;
}

}  // namespace slq
