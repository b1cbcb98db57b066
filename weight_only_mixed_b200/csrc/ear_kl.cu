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

#include <type_traits>

#include "internal.h"
#include "ptx.cuh"

namespace slq {
namespace {

constexpr unsigned kFull = 0xffffffffu;
// Ring kernel shape: 16 consumer warps, three 16-byte units of each logit
// stream per consumer thread per stage (a 48 KiB stage), four stages
// (measured against 12-24 warps and 2-3 units on T = 4096, V = 151936).
constexpr int kEarConsumerWarps = 16;
constexpr int kEarUnits = 3;
constexpr int kEarStages = 4;

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

// The two bf16 logits of one 32-bit word as a packed binary32 pair (exact).
__device__ __forceinline__ uint64_t bf16x2_f32x2(uint32_t w) { return pk(bf16_lo(w), bf16_hi(w)); }
__device__ __forceinline__ uint64_t ex2x2(uint64_t x) { return pk(ex2(pk_lo(x)), ex2(pk_hi(x))); }

// Maximum of the bf16 logits in U 16-byte units (packed bf16 max tree).
template <int U>
__device__ __forceinline__ float units_max(const uint4 (&v)[U]) {
  uint32_t m[U];
#pragma unroll
  for (int u = 0; u < U; ++u) {
    uint32_t x, y;
    asm("max.bf16x2 %0, %1, %2;" : "=r"(x) : "r"(v[u].x), "r"(v[u].y));
    asm("max.bf16x2 %0, %1, %2;" : "=r"(y) : "r"(v[u].z), "r"(v[u].w));
    asm("max.bf16x2 %0, %1, %2;" : "=r"(m[u]) : "r"(x), "r"(y));
  }
#pragma unroll
  for (int w = 1; w < U; w *= 2)
#pragma unroll
    for (int u = 0; u + w < U; u += 2 * w) asm("max.bf16x2 %0, %1, %2;" : "=r"(m[u]) : "r"(m[u]), "r"(m[u + w]));
  return fmaxf(bf16_lo(m[0]), bf16_hi(m[0]));
}

// Per-thread statistics of the vector path.  The sums are kept relative to
// the offset o = -rn(k c), k = max(running max, -1e30), so each term is one
// packed FMA (a c + o) and one exponential; the running maximum moves at most
// once per group of units.  At the end the sums are brought to the exact
// offset -k c by the factor 2^(k c + o), whose exponent an FMA gives exactly.
struct VecStat {
  float ma, ka, mb, kb;
  uint64_t oa, ob;      // {o, o}
  uint64_t sa, sb, w;   // packed partial sums
};

__device__ __forceinline__ VecStat vec_stat_init(float c) {
  const float o = 1e30f * c;
  return VecStat{-INFINITY, -1e30f, -INFINITY, -1e30f, pk(o, o), pk(o, o), 0ull, 0ull, 0ull};
}

template <int U>
__device__ __forceinline__ void push_units(VecStat& st, const uint4 (&va)[U], const uint4 (&vb)[U],
                                           float c) {
  const uint64_t c2 = pk(c, c);
  const float mA = units_max<U>(va), mB = units_max<U>(vb);
  if (mA > st.ma) {
    st.ma = mA;
    st.ka = fmaxf(mA, -1e30f);
    const float o = -(st.ka * c);
    const float f = ex2(o - pk_lo(st.oa));
    st.sa = mul2(st.sa, pk(f, f));
    st.w = mul2(st.w, pk(f, f));
    st.oa = pk(o, o);
  }
  if (mB > st.mb) {
    st.mb = mB;
    st.kb = fmaxf(mB, -1e30f);
    const float o = -(st.kb * c);
    const float f = ex2(o - pk_lo(st.ob));
    st.sb = mul2(st.sb, pk(f, f));
    st.ob = pk(o, o);
  }
#pragma unroll
  for (int u = 0; u < U; ++u) {
    const uint32_t wa[4] = {va[u].x, va[u].y, va[u].z, va[u].w};
    const uint32_t wb[4] = {vb[u].x, vb[u].y, vb[u].z, vb[u].w};
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const uint64_t A = bf16x2_f32x2(wa[q]), B = bf16x2_f32x2(wb[q]);
      const uint64_t ea = ex2x2(fma2(A, c2, st.oa));
      st.sa = add2(st.sa, ea);
      st.w = fma2(ea, sub2(A, B), st.w);
      st.sb = add2(st.sb, ex2x2(fma2(B, c2, st.ob)));
    }
  }
}

__device__ __forceinline__ RowStat vec_stat_final(const VecStat& st, float c) {
  const float fa = ex2(-fmaf(st.ka, c, pk_lo(st.oa)));
  const float fb = ex2(-fmaf(st.kb, c, pk_lo(st.ob)));
  return RowStat{{st.ma, (pk_lo(st.sa) + pk_hi(st.sa)) * fa},
                 {st.mb, (pk_lo(st.sb) + pk_hi(st.sb)) * fb},
                 (pk_lo(st.w) + pk_hi(st.w)) * fa};
}

// EAR terms of U units: 2^min(x_a, x_b) with x = (a - m) c - log2 S; the
// shift by the row maximum is exact in binary32, so x takes one rounding.
template <int U>
__device__ __forceinline__ void ear_units(uint64_t (&acc)[2], const uint4 (&va)[U],
                                          const uint4 (&vb)[U], uint64_t c2, uint64_t ma2,
                                          uint64_t nla2, uint64_t mb2, uint64_t nlb2) {
#pragma unroll
  for (int u = 0; u < U; ++u) {
    const uint32_t wa[4] = {va[u].x, va[u].y, va[u].z, va[u].w};
    const uint32_t wb[4] = {vb[u].x, vb[u].y, vb[u].z, vb[u].w};
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const uint64_t xa = fma2(sub2(bf16x2_f32x2(wa[q]), ma2), c2, nla2);
      const uint64_t xb = fma2(sub2(bf16x2_f32x2(wb[q]), mb2), c2, nlb2);
      const float x0 = fminf(pk_lo(xa), pk_lo(xb)), x1 = fminf(pk_hi(xa), pk_hi(xb));
      acc[q & 1] = add2(acc[q & 1], pk(ex2(x0), ex2(x1)));
    }
  }
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

// Row statistics plus an EAR partial, reduced together.
struct Part {
  RowStat st;
  float ear;
};

__device__ __forceinline__ Part warp_reduce(Part v, float c) {
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) {
    merge(v.st, shfl_xor(v.st, off), c);
    v.ear += __shfl_xor_sync(kFull, v.ear, off);
  }
  return v;
}

__device__ __forceinline__ float kl_of(const RowStat& r, float inv_temp) {
  constexpr float kLn2 = 0.693147180559945309f;
  const float la = lg2(r.a.s), lb = lg2(r.b.s);
  return (r.w / r.a.s) * inv_temp - ((r.a.m - r.b.m) * inv_temp + (la - lb) * kLn2);
}

// ---------------------------------------------------------------------------
// V % 8 == 0 (16-byte aligned rows): one CTA per SM walks its rows t0,
// t0 + G, ...  A producer warp streams each row twice through a ring of
// shared-memory stages with 1-D bulk copies -- chunks of the row for the
// statistics pass (from HBM, kept in L2), then the same chunks again for the
// EAR pass (from L2) -- so loads are always in flight, independent of the
// arithmetic.  kCW consumer warps process the stages: each thread takes kU
// 16-byte units of each logit stream per stage.  Between the passes the
// consumer warps reduce the row statistics through shared memory; the EAR
// sum of a row is reduced together with the statistics of the next one.
// Every wait is bounded; a timeout raises SLQ_FLAG_TIMEOUT and the CTA stops.
// ---------------------------------------------------------------------------
template <int kCW, int kU>
struct RingCfg {
  static constexpr int kConsumers = kCW * 32;
  static constexpr int kThreads = kConsumers + 32;
  static constexpr int kChunk = kU * 8 * kConsumers;  // logits of one stream per stage
  static constexpr int kStageBytes = 2 * kChunk * 2;  // a and b
};

__device__ __forceinline__ bool ring_wait(uint64_t* bar, uint32_t parity, volatile int* abort) {
  if (mbar_try_wait(bar, parity)) return true;
  const long long t0 = clock64();
  while (true) {
#pragma unroll 1
    for (int i = 0; i < 8; ++i)
      if (mbar_try_wait(bar, parity)) return true;
    if (*abort) return false;
    if (clock64() - t0 > kWaitLimitCycles) {
      *abort = 1;
      return false;
    }
  }
}

template <int kCW, int kU, int kStages>
__global__ void __launch_bounds__(RingCfg<kCW, kU>::kThreads, 1)
    ear_kl_ring_kernel(const uint16_t* __restrict__ A, const uint16_t* __restrict__ Bq, int64_t T,
                       int64_t V, float c, float inv_temp, float* __restrict__ ear_tok,
                       float* __restrict__ kl_tok, uint32_t* __restrict__ flags) {
  using Cfg = RingCfg<kCW, kU>;
  constexpr int kChunk = Cfg::kChunk;
  extern __shared__ __align__(128) uint8_t smem[];
  uint16_t* stages = reinterpret_cast<uint16_t*>(smem);
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + kStages * Cfg::kStageBytes);
  uint64_t* empty = full + kStages;
  uint64_t* red = empty + kStages;  // [2]
  Part* parts = reinterpret_cast<Part*>(red + 2);  // [2][kCW]
  volatile int* abort = reinterpret_cast<volatile int*>(parts + 2 * kCW);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t G = gridDim.x;
  const int64_t nch = (V + kChunk - 1) / kChunk;  // chunks per pass of one row
  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], kCW);
    }
    mbar_init(&red[0], kCW);
    mbar_init(&red[1], kCW);
    *abort = 0;
    fence_mbarrier_init();
  }
  __syncthreads();

  if (warp == kCW) {
    // Producer: one lane issues every copy, in the consumers' order.
    if (lane != 0) return;
    const uint64_t keep = l2_policy_evict_last();
    const uint64_t done = l2_policy_evict_first();
    uint32_t seq = 0;
    bool ok = true;
    for (int64_t t = blockIdx.x; t < T && ok; t += G) {
      for (int pass = 0; pass < 2 && ok; ++pass) {
        for (int64_t k = 0; k < nch; ++k, ++seq) {
          const int s = static_cast<int>(seq % kStages);
          if (seq >= static_cast<uint32_t>(kStages) &&
              !ring_wait(&empty[s], ((seq / kStages) & 1u) ^ 1u, abort)) {
            ok = false;
            break;
          }
          const int64_t v0 = k * kChunk;
          const uint32_t bytes = static_cast<uint32_t>((V - v0 < kChunk ? V - v0 : kChunk) * 2);
          uint16_t* dst = stages + static_cast<size_t>(s) * (2 * kChunk);
          mbar_arrive_expect_tx(&full[s], 2 * bytes);
          bulk_load_hint(dst, A + t * V + v0, bytes, &full[s], pass ? done : keep);
          bulk_load_hint(dst + kChunk, Bq + t * V + v0, bytes, &full[s], pass ? done : keep);
        }
      }
    }
    if (!ok) {
      // Consumers stopped: let the copies already issued land before exit.
      const uint32_t first = seq > static_cast<uint32_t>(kStages) ? seq - kStages : 0u;
      for (uint32_t q = first; q < seq; ++q)
        mbar_wait_bounded(&full[q % kStages], (q / kStages) & 1u);
      if (flags) atomicOr(flags, kFlagTimeout);
    }
    return;
  }

  // Consumers.
  const int ct = threadIdx.x;  // 0 .. kConsumers-1
  const Part none{{{-INFINITY, 0.0f}, {-INFINITY, 0.0f}, 0.0f}, 0.0f};
  uint32_t seq = 0, nred = 0;
  int64_t t_prev = -1;
  float ear_part = 0.0f;
  // One stage: load this thread's units (all of them, or those inside a
  // ragged last chunk), release the stage once the loads have returned, then
  // run `f` on the loaded units.
  auto consume = [&](int64_t k, auto&& f_full, auto&& f_one) -> bool {
    const int s = static_cast<int>(seq % kStages);
    if (!ring_wait(&full[s], (seq / kStages) & 1u, abort)) return false;
    const uint16_t* a_st = stages + static_cast<size_t>(s) * (2 * kChunk);
    const uint16_t* b_st = a_st + kChunk;
    const int64_t left = V - k * kChunk;
    uint4 va[kU], vb[kU];
    uint32_t dep = 0;
    if (left >= kChunk) {
#pragma unroll
      for (int u = 0; u < kU; ++u) {
        va[u] = *reinterpret_cast<const uint4*>(a_st + 8 * (ct + u * Cfg::kConsumers));
        vb[u] = *reinterpret_cast<const uint4*>(b_st + 8 * (ct + u * Cfg::kConsumers));
        dep ^= va[u].x ^ va[u].y ^ va[u].z ^ va[u].w ^ vb[u].x ^ vb[u].y ^ vb[u].z ^ vb[u].w;
      }
    } else {
      const int units = static_cast<int>(left / 8);
#pragma unroll
      for (int u = 0; u < kU; ++u) {
        const int unit = ct + u * Cfg::kConsumers;
        if (unit < units) {
          va[u] = *reinterpret_cast<const uint4*>(a_st + 8 * unit);
          vb[u] = *reinterpret_cast<const uint4*>(b_st + 8 * unit);
          dep ^= va[u].x ^ va[u].y ^ va[u].z ^ va[u].w ^ vb[u].x ^ vb[u].y ^ vb[u].z ^ vb[u].w;
        }
      }
    }
    dep = __reduce_or_sync(kFull, dep);
    if (lane == 0) {
      fence_proxy_async_smem();
      mbar_arrive_after(&empty[s], dep);
    }
    ++seq;
    if (left >= kChunk) {
      f_full(va, vb);
    } else {
      const int units = static_cast<int>(left / 8);
#pragma unroll
      for (int u = 0; u < kU; ++u)
        if (ct + u * Cfg::kConsumers < units) f_one(va[u], vb[u]);
    }
    return true;
  };
  // Reduce (statistics, EAR part) over the consumer warps; every warp ends
  // with the same total.
  auto reduce = [&](Part mine, Part& tot) -> bool {
    mine = warp_reduce(mine, c);
    Part* slot = parts + (nred & 1u) * kCW;
    uint64_t* bar = &red[nred & 1u];
    if (lane == 0) {
      slot[warp] = mine;
      mbar_arrive(bar);
    }
    if (!ring_wait(bar, (nred >> 1) & 1u, abort)) return false;
    ++nred;
    tot = (lane < kCW) ? slot[lane] : none;
    tot = warp_reduce(tot, c);
    return true;
  };

  bool ok = true;
  for (int64_t t = blockIdx.x; t < T && ok; t += G) {
    VecStat vs = vec_stat_init(c);
    for (int64_t k = 0; k < nch && ok; ++k)
      ok = consume(
          k, [&](const uint4(&va)[kU], const uint4(&vb)[kU]) { push_units<kU>(vs, va, vb, c); },
          [&](const uint4& a1, const uint4& b1) {
            const uint4 va[1] = {a1}, vb[1] = {b1};
            push_units<1>(vs, va, vb, c);
          });
    Part tot;
    if (!ok || !reduce(Part{vec_stat_final(vs, c), ear_part}, tot)) {
      ok = false;
      break;
    }
    if (ct == 0) {
      if (t_prev >= 0) ear_tok[t_prev] = tot.ear;
      kl_tok[t] = kl_of(tot.st, inv_temp);
    }
    const uint64_t c2 = pk(c, c);
    const float nla = -lg2(tot.st.a.s), nlb = -lg2(tot.st.b.s);
    const uint64_t ma2 = pk(tot.st.a.m, tot.st.a.m), mb2 = pk(tot.st.b.m, tot.st.b.m);
    const uint64_t nla2 = pk(nla, nla), nlb2 = pk(nlb, nlb);
    uint64_t acc[2] = {0ull, 0ull};
    for (int64_t k = 0; k < nch && ok; ++k)
      ok = consume(
          k,
          [&](const uint4(&va)[kU], const uint4(&vb)[kU]) {
            ear_units<kU>(acc, va, vb, c2, ma2, nla2, mb2, nlb2);
          },
          [&](const uint4& a1, const uint4& b1) {
            const uint4 va[1] = {a1}, vb[1] = {b1};
            ear_units<1>(acc, va, vb, c2, ma2, nla2, mb2, nlb2);
          });
    ear_part = (pk_lo(acc[0]) + pk_hi(acc[0])) + (pk_lo(acc[1]) + pk_hi(acc[1]));
    t_prev = t;
  }
  if (ok && t_prev >= 0) {
    Part tot;
    if (reduce(Part{none.st, ear_part}, tot)) {
      if (ct == 0) ear_tok[t_prev] = tot.ear;
    } else {
      ok = false;
    }
  }
  if (!ok && ct == 0 && flags) atomicOr(flags, kFlagTimeout);
}

template <int kCW, int kU, int kStages>
constexpr size_t ring_smem_bytes() {
  return static_cast<size_t>(kStages) * RingCfg<kCW, kU>::kStageBytes +
         (2 * kStages + 2) * sizeof(uint64_t) + 2 * kCW * sizeof(Part) + 16;
}

// ---------------------------------------------------------------------------
// Any V (the V % 8 != 0 case): one row per CTA, scalar loads; pass 1 the
// online statistics, pass 2 the EAR terms (the row is back from L2).
// ---------------------------------------------------------------------------
template <int kThreads>
__global__ void __launch_bounds__(kThreads)
    ear_kl_rows_kernel(const uint16_t* __restrict__ A, const uint16_t* __restrict__ Bq, int64_t T,
                       int64_t V, float c, float inv_temp, float* __restrict__ ear_tok,
                       float* __restrict__ kl_tok) {
  for (int64_t t = blockIdx.x; t < T; t += gridDim.x) {
    const uint16_t* a_row = A + t * V;
    const uint16_t* b_row = Bq + t * V;
    RowStat st{{-INFINITY, 0.0f}, {-INFINITY, 0.0f}, 0.0f};
    for (int64_t v = threadIdx.x; v < V; v += kThreads)
      push(st, __uint_as_float(static_cast<uint32_t>(a_row[v]) << 16),
           __uint_as_float(static_cast<uint32_t>(b_row[v]) << 16), c);
    const RowStat tot = block_reduce<kThreads>(st, c);
    const float la = lg2(tot.a.s), lb = lg2(tot.b.s);
    const float ma = tot.a.m, mb = tot.b.m;
    float acc[4] = {0.0f, 0.0f, 0.0f, 0.0f};
    int q = 0;
    for (int64_t v = threadIdx.x; v < V; v += kThreads) {
      const float a = __uint_as_float(static_cast<uint32_t>(a_row[v]) << 16);
      const float b = __uint_as_float(static_cast<uint32_t>(b_row[v]) << 16);
      acc[q] += ex2(fminf((a - ma) * c - la, (b - mb) * c - lb));
      q = (q + 1) & 3;
    }
    const float ear = block_sum<kThreads>((acc[0] + acc[1]) + (acc[2] + acc[3]));
    if (threadIdx.x == 0) {
      ear_tok[t] = ear;
      kl_tok[t] = kl_of(tot, inv_temp);
    }
  }
}

// ---------------------------------------------------------------------------
// Top-K form (the pages' evaluation: EAR and KL restricted to the top-K
// tokens).  T = the K largest reference logits a, ties to the lower index;
// EAR = sum over T of min(p, q) with the full-vocabulary softmaxes; KL =
// KL(p_T || q_T) with p and q renormalized over T.
//
// One CTA per row, one pass over the row: every thread keeps the online
// statistics of its logits (as above).  Each warp keeps its top-K list in
// registers across its lanes and a warp-wide threshold (the list's K-th
// entry): a unit's 8 logits are offered only when the unit's maximum (packed
// bf16 max) reaches the threshold, and offered logits that still reach it
// are inserted with one shuffle.  After the row, warp 0 merges the warps'
// lists by K rounds of a shuffle arg-max (KM = the power of two >= K bounds
// the register lists), and K lanes form the terms.
// ---------------------------------------------------------------------------
constexpr int kTopMax = 16;
// Small CTAs, several per SM: a CTA's end-of-row merge (warp 0 alone, the
// others at the barrier) then overlaps the other CTAs' streaming.  One
// 512-thread CTA per SM (~100 registers a thread) left the SM idle during
// every merge.  On 4096 x 151936, K = 10: 1089 us with 512 threads (1 CTA
// per SM), 635 with 128 (4 per SM), 573 with 64 (8 per SM); with fewer rows
// than 2 per 64-thread CTA the 128-thread shape is faster (T = 512: 98
// against 130 us).
constexpr int kTopThreadsSmall = 64, kTopCtasSmall = 8;
constexpr int kTopThreadsLarge = 128, kTopCtasLarge = 4;

// (v, i) ranks before (w, j): larger logit first, lower index on ties.
__device__ __forceinline__ bool top_before(float v, int i, float w, int j) {
  return v > w || (v == w && i < j);
}

template <int KM>
struct TopList {
  float v[KM];
  int i[KM];
};

template <int KM>
__device__ __forceinline__ void top_init(TopList<KM>& t) {
#pragma unroll
  for (int j = 0; j < KM; ++j) {
    t.v[j] = -INFINITY;
    t.i[j] = 0x7fffffff;
  }
}

// Insert (v, i) into the sorted list; no-op if it ranks after the last entry.
template <int KM>
__device__ __forceinline__ void top_push(TopList<KM>& t, float v, int i) {
  if (!top_before(v, i, t.v[KM - 1], t.i[KM - 1])) return;
#pragma unroll
  for (int j = 0; j < KM; ++j) {
    if (top_before(v, i, t.v[j], t.i[j])) {
      const float tv = t.v[j];
      const int ti = t.i[j];
      t.v[j] = v;
      t.i[j] = i;
      v = tv;
      i = ti;
    }
  }
}

// K rounds of a warp arg-max over the lanes' sorted lists (each lane's head
// advances when it wins); lane r < K ends with the r-th best of the warp.
template <int KM>
__device__ __forceinline__ void top_warp_merge(const TopList<KM>& t, int K, float& out_v,
                                               int& out_i) {
  const int lane = threadIdx.x & 31;
  int h = 0;
  out_v = -INFINITY;
  out_i = 0x7fffffff;
  for (int r = 0; r < K; ++r) {
    float hv = -INFINITY;
    int hi = 0x7fffffff;
#pragma unroll
    for (int j = 0; j < KM; ++j)
      if (j == h) {
        hv = t.v[j];
        hi = t.i[j];
      }

    float bv = hv;
    int bi = hi, bl = lane;
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) {
      const float ov = __shfl_xor_sync(kFull, bv, off);
      const int oi = __shfl_xor_sync(kFull, bi, off);
      const int ol = __shfl_xor_sync(kFull, bl, off);
      if (top_before(ov, oi, bv, bi) || (ov == bv && oi == bi && ol < bl)) {
        bv = ov;
        bi = oi;
        bl = ol;
      }
    }
    if (lane == bl) ++h;
    if (lane == r) {
      out_v = bv;
      out_i = bi;
    }
  }
}

// The warp's top-K list lives in registers across the lanes: lane r < K
// holds the r-th best (a, index) seen by the warp so far, lanes >= K hold
// placeholders.  Inserting a warp-uniform (v, i) shifts the entries that rank
// after it down by one lane.
__device__ __forceinline__ void warp_list_insert(float& lv, int& li, float v, int i) {
  const int lane = threadIdx.x & 31;
  const bool after = top_before(v, i, lv, li);  // this lane's entry now ranks after (v, i)
  const float pv = __shfl_up_sync(kFull, lv, 1);
  const int pi = __shfl_up_sync(kFull, li, 1);
  const bool pafter = __shfl_up_sync(kFull, after ? 1 : 0, 1) != 0 && lane > 0;
  if (after) {
    lv = pafter ? pv : v;
    li = pafter ? pi : i;
  }
}

// The K-th largest of one value per lane (a bitonic sort over the warp).
__device__ __forceinline__ float warp_kth_largest(float m, int K) {
  const int lane = threadIdx.x & 31;
#pragma unroll
  for (int k = 2; k <= 32; k <<= 1)
#pragma unroll
    for (int j = k >> 1; j > 0; j >>= 1) {
      const float o = __shfl_xor_sync(kFull, m, j);
      const bool up = (lane & k) == 0, lower = (lane & j) == 0;
      m = (lower == up) ? fmaxf(m, o) : fminf(m, o);
    }
  return __shfl_sync(kFull, m, K - 1);
}

template <bool kVec, int KM, int kTopThreads>
__global__ void __launch_bounds__(kTopThreads)
    ear_kl_topk_kernel(const uint16_t* __restrict__ A, const uint16_t* __restrict__ Bq, int64_t T,
                       int64_t V, int K, float c, float* __restrict__ ear_tok,
                       float* __restrict__ kl_tok) {
  constexpr int kWarps = kTopThreads / 32;
  __shared__ Part parts[kWarps];
  __shared__ float wv[kWarps][KM];
  __shared__ int wi[kWarps][KM];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  constexpr float kLn2 = 0.693147180559945309f;
  for (int64_t t = blockIdx.x; t < T; t += gridDim.x) {
    const uint16_t* a_row = A + t * V;
    const uint16_t* b_row = Bq + t * V;
    // thr: the warp's K-th best so far (or a lower bound of it); a logit
    // below it cannot enter the row's top K.
    float lv = -INFINITY, thr = -INFINITY;
    int li = 0x7fffffff;
    // Lanes whose `hit` is set offer their `cnt` logits (values from `get`)
    // one at a time, in lane order; many hits first raise the threshold to
    // the K-th largest of the lanes' maxima (at least K logits reach it).
    // `sel(thr)` gives a lane's bitmask of its logits that reach thr.
    auto offer = [&](bool hit, float mx, auto&& get, auto&& sel) {
      unsigned mask = __ballot_sync(kFull, hit);
      if (!mask) return;
      if (__popc(mask) >= K && __popc(mask) > 4) {
        thr = fmaxf(thr, warp_kth_largest(hit ? mx : -INFINITY, K));
        mask = __ballot_sync(kFull, hit && mx >= thr);
      }
      const unsigned mine = (mask >> lane) & 1u ? sel(thr) : 0u;
      while (mask) {
        const int src = __ffs(mask) - 1;
        mask &= mask - 1;
        unsigned bits = __shfl_sync(kFull, mine, src);
        while (bits) {
          const int e = __ffs(bits) - 1;
          bits &= bits - 1;
          float x;
          int ix;
          get(src, e, x, ix);
          if (x >= thr) {
            warp_list_insert(lv, li, x, ix);
            thr = fmaxf(thr, __shfl_sync(kFull, lv, K - 1));
          }
        }
      }
    };
    RowStat st;
    if constexpr (kVec) {
      const int64_t nv = V / 8;
      VecStat vs = vec_stat_init(c);
      auto visit = [&](const uint4& va, int64_t unit, bool valid) {
        const uint4 one[1] = {va};
        const float mx = valid ? units_max<1>(one) : -INFINITY;
        offer(valid && mx >= thr, mx,
              [&](int src, int e, float& x, int& ix) {
                const uint32_t wsel = (e >> 1) == 0 ? va.x : (e >> 1) == 1 ? va.y : (e >> 1) == 2 ? va.z : va.w;
                const uint32_t w = __shfl_sync(kFull, wsel, src);
                x = (e & 1) ? bf16_hi(w) : bf16_lo(w);
                ix = 8 * static_cast<int>(__shfl_sync(kFull, static_cast<int>(unit), src)) + e;
              },
              [&](float th) {
                const uint32_t w[4] = {va.x, va.y, va.z, va.w};
                unsigned bits = 0;
#pragma unroll
                for (int e = 0; e < 8; ++e)
                  if (((e & 1) ? bf16_hi(w[e >> 1]) : bf16_lo(w[e >> 1])) >= th) bits |= 1u << e;
                return bits;
              });
      };
      // Loop bounds are the warp's (its last lane's), so every lane takes
      // part in every warp-wide step.
      int64_t i0 = 32 * warp;
      for (; i0 + 31 + 3 * kTopThreads < nv; i0 += 4 * kTopThreads) {
        const int64_t i = i0 + lane;
        uint4 va[4], vb[4];
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          va[u] = ld_stream_v4(a_row + 8 * (i + u * kTopThreads));
          vb[u] = ld_stream_v4(b_row + 8 * (i + u * kTopThreads));
        }
        push_units<4>(vs, va, vb, c);
#pragma unroll
        for (int u = 0; u < 4; ++u) visit(va[u], i + u * kTopThreads, true);
      }
      for (; i0 < nv; i0 += kTopThreads) {
        const int64_t u = i0 + lane;
        const bool valid = u < nv;
        uint4 va = make_uint4(0u, 0u, 0u, 0u);
        if (valid) {
          va = ld_stream_v4(a_row + 8 * u);
          const uint4 a1[1] = {va};
          const uint4 b1[1] = {ld_stream_v4(b_row + 8 * u)};
          push_units<1>(vs, a1, b1, c);
        }
        visit(va, u, valid);
      }
      st = vec_stat_final(vs, c);
    } else {
      st = RowStat{{-INFINITY, 0.0f}, {-INFINITY, 0.0f}, 0.0f};
      for (int64_t v0 = 32 * warp; v0 < V; v0 += kTopThreads) {
        const int64_t v = v0 + lane;
        const bool valid = v < V;
        float a = -INFINITY;
        if (valid) {
          a = __uint_as_float(static_cast<uint32_t>(a_row[v]) << 16);
          const float b = __uint_as_float(static_cast<uint32_t>(b_row[v]) << 16);
          push(st, a, b, c);
        }
        offer(valid && a >= thr, a,
              [&](int src, int, float& x, int& ix) {
                x = __shfl_sync(kFull, a, src);
                ix = __shfl_sync(kFull, static_cast<int>(v), src);
              },
              [&](float th) { return a >= th ? 1u : 0u; });
      }
    }
    // The warp's K best, lane r holding the r-th: its sorted list.
    TopList<KM> top;
    top_init(top);
#pragma unroll
    for (int j = 0; j < KM; ++j) {
      const float v = __shfl_sync(kFull, lv, j);
      const int ix = __shfl_sync(kFull, li, j);
      if (j < K) {
        top.v[j] = v;
        top.i[j] = ix;
      }
    }
    // Row statistics and the warps' top-K lists.
    Part mine{st, 0.0f};
    mine = warp_reduce(mine, c);
    if (lane == 0) parts[warp] = mine;
#pragma unroll
    for (int j = 0; j < KM; ++j)
      if (lane == j && j < K) {
        wv[warp][j] = top.v[j];
        wi[warp][j] = top.i[j];
      }
    __syncthreads();
    if (warp == 0) {
      Part tot = (lane < kWarps) ? parts[lane]
                                 : Part{{{-INFINITY, 0.0f}, {-INFINITY, 0.0f}, 0.0f}, 0.0f};
      tot = warp_reduce(tot, c);
      TopList<KM> wl;
      top_init(wl);
      if (lane < kWarps) {
#pragma unroll
        for (int j = 0; j < KM; ++j)
          if (j < K) {
            wl.v[j] = wv[lane][j];
            wl.i[j] = wi[lane][j];
          }
      }
      float bv;
      int bi;
      top_warp_merge(wl, K, bv, bi);
      // Lane k < K holds the k-th token of T: its terms in base 2.
      const float la = lg2(tot.st.a.s), lb = lg2(tot.st.b.s);
      float xa = -INFINITY, xb = -INFINITY;
      if (lane < K && bi < V) {  // bi < V always holds for finite logits
        const float a = __uint_as_float(static_cast<uint32_t>(a_row[bi]) << 16);
        const float b = __uint_as_float(static_cast<uint32_t>(b_row[bi]) << 16);
        xa = (a - tot.st.a.m) * c - la;  // log2 p
        xb = (b - tot.st.b.m) * c - lb;  // log2 q
      }
      const float p = lane < K ? ex2(xa) : 0.0f, q = lane < K ? ex2(xb) : 0.0f;
      float e = fminf(p, q), pt = p, qt = q;
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) {
        e += __shfl_xor_sync(kFull, e, off);
        pt += __shfl_xor_sync(kFull, pt, off);
        qt += __shfl_xor_sync(kFull, qt, off);
      }
      const float lpt = xa - lg2(pt), lqt = xb - lg2(qt);  // log2 of the renormalized p, q
      float d = lane < K ? ex2(lpt) * (lpt - lqt) : 0.0f;
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) d += __shfl_xor_sync(kFull, d, off);
      if (lane == 0) {
        ear_tok[t] = e;
        kl_tok[t] = d * kLn2;
      }
    }
    __syncthreads();
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

cudaError_t launch_ear_kl_topk(const uint16_t* a, const uint16_t* b, int64_t T, int64_t V, int K,
                               float temperature, float* ear_tok, float* kl_tok, double* ear_mean,
                               double* kl_mean, cudaStream_t stream) {
  if (K < 1 || K > kTopMax || K > V) return cudaErrorInvalidValue;
  int sms = 148, dev = 0;
  if (cudaGetDevice(&dev) == cudaSuccess)
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const float c = 1.4426950408889634f / temperature;
  const bool small = T >= 2 * kTopCtasSmall * static_cast<int64_t>(sms);
  const int64_t cap = (small ? kTopCtasSmall : kTopCtasLarge) * static_cast<int64_t>(sms);
  const unsigned blocks = static_cast<unsigned>(T < cap ? T : cap);
  const bool aligned = ((reinterpret_cast<uintptr_t>(a) | reinterpret_cast<uintptr_t>(b)) & 15u) == 0;
  const bool vec = V % 8 == 0 && aligned;
  auto run = [&](auto km) {
    constexpr int KM = decltype(km)::value;
    constexpr int NS = kTopThreadsSmall, NL = kTopThreadsLarge;
    if (vec && small)
      ear_kl_topk_kernel<true, KM, NS><<<blocks, NS, 0, stream>>>(a, b, T, V, K, c, ear_tok, kl_tok);
    else if (vec)
      ear_kl_topk_kernel<true, KM, NL><<<blocks, NL, 0, stream>>>(a, b, T, V, K, c, ear_tok, kl_tok);
    else if (small)
      ear_kl_topk_kernel<false, KM, NS><<<blocks, NS, 0, stream>>>(a, b, T, V, K, c, ear_tok, kl_tok);
    else
      ear_kl_topk_kernel<false, KM, NL><<<blocks, NL, 0, stream>>>(a, b, T, V, K, c, ear_tok, kl_tok);
  };
  if (K <= 1) run(std::integral_constant<int, 1>{});
  else if (K <= 2) run(std::integral_constant<int, 2>{});
  else if (K <= 4) run(std::integral_constant<int, 4>{});
  else if (K <= 8) run(std::integral_constant<int, 8>{});
  else run(std::integral_constant<int, 16>{});
  cudaError_t err = cudaGetLastError();
  if (err != cudaSuccess) return err;
  if (ear_mean || kl_mean) {
    token_mean_kernel<<<1, 1024, 0, stream>>>(ear_tok, kl_tok, T, ear_mean, kl_mean);
    err = cudaGetLastError();
  }
  return err;
}

int ear_kl_topk_max() { return kTopMax; }

cudaError_t launch_ear_kl(const uint16_t* a, const uint16_t* b, int64_t T, int64_t V,
                          float temperature, float* ear_tok, float* kl_tok, double* ear_mean,
                          double* kl_mean, uint32_t* flags, cudaStream_t stream) {
  int sms = 148, dev = 0;
  if (cudaGetDevice(&dev) == cudaSuccess)
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const float inv_temp = 1.0f / temperature;
  const float c = 1.4426950408889634f * inv_temp;
  cudaError_t err = cudaSuccess;

  const bool aligned = ((reinterpret_cast<uintptr_t>(a) | reinterpret_cast<uintptr_t>(b)) & 15u) == 0;
  if (V % 8 == 0 && aligned) {
    constexpr int kCW = kEarConsumerWarps, kU = kEarUnits, kS = kEarStages;
    constexpr size_t smem = ring_smem_bytes<kCW, kU, kS>();
    static_assert(smem <= 227 * 1024, "ring exceeds shared memory");
    auto kern = ear_kl_ring_kernel<kCW, kU, kS>;
    err = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               static_cast<int>(smem));
    if (err != cudaSuccess) return err;
    const int64_t cap = static_cast<int64_t>(sms);
    const int64_t blocks = T < cap ? T : cap;
    kern<<<static_cast<unsigned>(blocks), RingCfg<kCW, kU>::kThreads, smem, stream>>>(
        a, b, T, V, c, inv_temp, ear_tok, kl_tok, flags);
  } else {
    const int64_t cap = static_cast<int64_t>(sms);
    const int64_t blocks = T < cap ? T : cap;
    ear_kl_rows_kernel<1024><<<static_cast<unsigned>(blocks), 1024, 0, stream>>>(
        a, b, T, V, c, inv_temp, ear_tok, kl_tok);
  }
  err = cudaGetLastError();
  if (err != cudaSuccess) return err;
  if (ear_mean || kl_mean) {
    token_mean_kernel<<<1, 1024, 0, stream>>>(ear_tok, kl_tok, T, ear_mean, kl_mean);
    err = cudaGetLastError();
  }
  return err;
}

}  // namespace slq
