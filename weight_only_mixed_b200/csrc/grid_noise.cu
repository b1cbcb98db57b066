// grid_noise.cu -- per-group rounding noise of the asymmetric grid the format
// uses and of the symmetric grid it is compared with (the gamma^2 law).
//
// The pages' argument for an asymmetric grid (wispaper.ai blog, section on the
// gamma^2 variance law; gist.science summary, Methodology section 1
// "Theoretical Foundation"): for a group with range R = max w - min w and
// largest magnitude M = max |w|, gamma = 2 M / R, and a symmetric grid over
// [-M, M] has a step gamma times that of an asymmetric grid over [min, max],
// hence gamma^2 times its rounding-noise variance.  Per 128-weight group this
// kernel gives gamma and the sum of squared errors of each grid's nearest
// point (2^b points, min + i R / L and -M + i 2 M / L, L = 2^b - 1): the
// measurement behind the pages' ablation of the symmetric grid.
//
// Shape: a persistent CTA per resident slot.  A producer warp streams
// contiguous 32 KB chunks (128 groups) through a ring of shared-memory stages
// with 1-D bulk copies, so the loads in flight do not depend on registers.
// Eight consumer warps take sixteen groups each per stage, two lanes per
// group: lane sl of a group reads the group's 16-byte chunks 2 x + sl, x in
// 0..7, starting at x = the group's index mod 8 so that a warp's
// shared-memory reads take the minimum four wavefronts.  Group statistics are
// one shuffle between the two lanes.  HBM-bound: 2 bytes read per weight,
// 12 bytes written per group.  Every wait is bounded; a timeout raises
// SLQ_FLAG_TIMEOUT and the CTA stops.
//
// Arithmetic.  Minimum and maximum by bf16x2 min/max (exact); M is the larger
// magnitude of the two.  The group is scaled by a power of two 2^s that puts
// M in [2^-8, 4) (exact; keeps every intermediate inside binary32 range for
// subnormal and near-overflow groups; the sums scale back by 2^-2s exactly).
// Per weight and grid, in packed binary32 pairs, with d = w - start:
//   t  = fma(d, L / R, 1.5 * 2^23)   the nearest point's index i, as t - 1.5 * 2^23
//                                    (round to nearest even of d L / R)
//   iR = fma(t, R, -1.5 * 2^23 R)    = i R exactly
//   E  = fma(d, L, -iR)              = L e, rounded once (e = d - i R / L)
// and the lane sums E^2; SSE = sum / L^2.  The fmas are exact where the
// spans have at most 16 significant bits: always for the symmetric span 2 M
// (a bf16 value doubled), and for R = max - min whenever max and min are
// within 2^8 of each other in magnitude.  A warp holding a group whose R is
// longer takes the general form for the asymmetric grid: e = d - i step with
// the step as two binary32 terms (about 2^-24 of e).  Every weight lies
// inside both grids' spans, so the index needs no clamp (it rounds into
// [0, L]); a position within rounding of a half-integer may take the other
// neighbour, whose error has the same magnitude up to that rounding.  The
// group's sums are binary32 (two chains of 32 terms per lane, then the two
// lanes).
#include "internal.h"
#include "ptx.cuh"

namespace slq {
namespace {

constexpr unsigned kFull = 0xffffffffu;
constexpr float kMagic = 12582912.0f;  // 1.5 * 2^23

__device__ __forceinline__ float bf16_lo(uint32_t v) { return __uint_as_float(v << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t v) { return __uint_as_float(v & 0xffff0000u); }
__device__ __forceinline__ uint64_t bf16x2_pair(uint32_t v) { return pk(bf16_lo(v), bf16_hi(v)); }

__device__ __forceinline__ uint32_t bf16x2_min(uint32_t a, uint32_t b) {
  uint32_t d;
  asm("min.bf16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
  return d;
}
__device__ __forceinline__ uint32_t bf16x2_max(uint32_t a, uint32_t b) {
  uint32_t d;
  asm("max.bf16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
  return d;
}
__device__ __forceinline__ float rcp_approx(float x) {
  float r;
  asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(r) : "f"(x));
  return r;
}

// floor(log2 x) of a finite x > 0 (normal or subnormal binary32).
__device__ __forceinline__ int ilog2f(float x) {
  const uint32_t u = __float_as_uint(x);
  return (u >> 23) ? static_cast<int>(u >> 23) - 127 : (31 - __clz(static_cast<int>(u))) - 149;
}

// Per-grid constants of the packed loop: d = w 2^s - start, index by
// t = fma(d, L / span, 1.5 * 2^23).  The exact form also holds -span and
// 1.5 * 2^23 span; the general form the step as hi + lo.
struct GridC {
  uint64_t nst, inv, a, b;  // exact: a = -span, b = 1.5 * 2^23 span; general: a = -hi, b = -lo
};

__device__ __forceinline__ GridC grid_exact(float start, float span, float L) {
  const float inv = span > 0.0f ? L * rcp_approx(span) : 0.0f;
  return {pk(-start, -start), pk(inv, inv), pk(-span, -span), pk(kMagic * span, kMagic * span)};
}

__device__ __forceinline__ GridC grid_general(float start, double step) {
  const float hi = static_cast<float>(step);
  const float lo = static_cast<float>(step - static_cast<double>(hi));
  const float inv = hi > 0.0f ? rcp_approx(hi) : 0.0f;
  return {pk(-start, -start), pk(inv, inv), pk(-hi, -hi), pk(-lo, -lo)};
}

// Both grids over the lane's weights (kWords packed pairs) in one pass.  The
// symmetric grid always takes the exact form (sum of (L e)^2); the
// asymmetric one the exact form when kExactA, else the general form (sum of
// e^2).  Two accumulators per grid halve the dependent chain.
template <int kWords, bool kExactA>
__device__ __forceinline__ float2 grid_sums(const uint32_t (&wds)[kWords], float f, float L, const GridC& ga,
                                            const GridC& gs) {
  const uint64_t f2 = pk(f, f), L2 = pk(L, L), magic = pk(kMagic, kMagic);
  uint64_t acc_a[2] = {0ull, 0ull}, acc_s[2] = {0ull, 0ull};
#pragma unroll
  for (int k = 0; k < kWords; ++k) {
    const uint64_t w = bf16x2_pair(wds[k]);
    const uint64_t ds = fma2(w, f2, gs.nst);
    const uint64_t ts = fma2(ds, gs.inv, magic);
    const uint64_t Es = fma2(ds, L2, fma2(ts, gs.a, gs.b));  // L d - i span
    acc_s[k & 1] = fma2(Es, Es, acc_s[k & 1]);
    const uint64_t da = fma2(w, f2, ga.nst);
    const uint64_t ta = fma2(da, ga.inv, magic);
    if constexpr (kExactA) {
      const uint64_t Ea = fma2(da, L2, fma2(ta, ga.a, ga.b));
      acc_a[k & 1] = fma2(Ea, Ea, acc_a[k & 1]);
    } else {
      const uint64_t i = sub2(ta, magic);
      const uint64_t e = fma2(i, ga.b, fma2(i, ga.a, da));
      acc_a[k & 1] = fma2(e, e, acc_a[k & 1]);
    }
  }
  const uint64_t sa = add2(acc_a[0], acc_a[1]), ss = add2(acc_s[0], acc_s[1]);
  return make_float2(pk_lo(sa) + pk_hi(sa), pk_lo(ss) + pk_hi(ss));
}

// One group, kLanes lanes (the lane's weights in wds): gamma and both SSEs,
// written by the group's first lane.
template <int kLanes, int kWords>
__device__ __forceinline__ void noise_group(const uint32_t (&wds)[kWords], int64_t grp, bool valid, int levels,
                                            double inv_l2,
                                            float* __restrict__ gamma, float* __restrict__ sse_asym,
                                            float* __restrict__ sse_sym, uint32_t* __restrict__ flags) {
  const int sl = threadIdx.x & (kLanes - 1);
  uint32_t vmin = wds[0], vmax = wds[0];
#pragma unroll
  for (int i = 1; i < kWords; ++i) {
    vmin = bf16x2_min(vmin, wds[i]);
    vmax = bf16x2_max(vmax, wds[i]);
  }
  float mn = fminf(bf16_lo(vmin), bf16_hi(vmin));
  float mx = fmaxf(bf16_lo(vmax), bf16_hi(vmax));
#pragma unroll
  for (int off = kLanes / 2; off > 0; off >>= 1) {
    mn = fminf(mn, __shfl_xor_sync(kFull, mn, off));
    mx = fmaxf(mx, __shfl_xor_sync(kFull, mx, off));
  }
  const float am = fmaxf(fabsf(mn), fabsf(mx));
  const bool finite = am <= 3.40282347e38f;  // false for inf and NaN
  // Scale 2^s with am 2^s in [2^-8, 4); s in [-126, 125] keeps 2^s normal.
  int s = (am > 0.0f && finite) ? -8 - ilog2f(am) : 0;
  s = max(-126, min(125, s));
  const float f = __uint_as_float(static_cast<uint32_t>(s + 127) << 23);
  const float L = static_cast<float>(levels);
  const float r32 = mx - mn;
  // r32 is exact and has at most 16 significant bits.
  const bool short_range = (__float_as_uint(r32) & 0xffu) == 0u &&
                           static_cast<double>(r32) == static_cast<double>(mx) - static_cast<double>(mn);
  const float ams = am * f, mns = mn * f;
  const GridC gs = grid_exact(-ams, 2.0f * ams, L);
  float2 sums;
  double sa_scale;  // 1 / L^2 (inv_l2) for the exact form, 1 for the general one
  if (__all_sync(kFull, short_range || !finite)) {
    sums = grid_sums<kWords, true>(wds, f, L, grid_exact(mns, r32 * f, L), gs);
    sa_scale = inv_l2;
  } else {
    const double range = static_cast<double>(mx) - static_cast<double>(mn);
    sums = grid_sums<kWords, false>(wds, f, L, grid_general(mns, range * static_cast<double>(f) / levels), gs);
    sa_scale = 1.0;
  }
#pragma unroll
  for (int off = kLanes / 2; off > 0; off >>= 1) {
    sums.x += __shfl_xor_sync(kFull, sums.x, off);
    sums.y += __shfl_xor_sync(kFull, sums.y, off);
  }
  if (valid && sl == 0) {
    const double range = static_cast<double>(mx) - static_cast<double>(mn);  // exact
    const double back = __longlong_as_double(static_cast<long long>(1023 - 2 * s) << 52);  // 2^-2s
    gamma[grp] = range > 0.0 ? static_cast<float>(2.0 * am / range) : 1.0f;
    sse_asym[grp] = static_cast<float>(static_cast<double>(sums.x) * sa_scale * back);
    sse_sym[grp] = static_cast<float>(static_cast<double>(sums.y) * inv_l2 * back);
    if (flags && (!finite || isnan(sums.x) || isnan(sums.y))) atomicOr(flags, kFlagNonfinite);
  }
}

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

constexpr int kWarps = 4;
constexpr int kThreads = kWarps * 32;
constexpr int kLanes = 2;                          // lanes per group
constexpr int kWords = 64 / kLanes;                // bf16 pairs per lane
constexpr int kLoads = 16 / kLanes;                // 16-byte shared-memory reads per lane
constexpr int kGroupsPerWarp = 32 / kLanes;
constexpr int kChunkGroups = kWarps * kGroupsPerWarp;  // groups per stage
constexpr int kStageBytes = kChunkGroups * kGroup * 2;
constexpr int kStages = 2;
constexpr int kCtasPerSm = 5;
constexpr size_t kSmemBytes =
    static_cast<size_t>(kStages) * kStageBytes + kStages * (sizeof(uint64_t) + sizeof(uint32_t)) + 16;

__device__ __forceinline__ void issue_chunk(uint8_t* dst, const uint16_t* W, int64_t c, int64_t total_groups,
                                            uint64_t* full, uint64_t policy) {
  const int64_t g0 = c * kChunkGroups;
  const int64_t ng = total_groups - g0 < kChunkGroups ? total_groups - g0 : kChunkGroups;
  const uint32_t bytes = static_cast<uint32_t>(ng * kGroup * 2);
  mbar_arrive_expect_tx(full, bytes);
  bulk_load_hint(dst, W + g0 * kGroup, bytes, full, policy);
}

// Chunks c = blockIdx.x + G q (q = 0, 1, ...) pass through stage q mod kStages.
// Thread 0 issues the first kStages copies; afterwards the warp that finishes
// reading a stage last (a per-stage counter) issues the stage's next chunk,
// so no warp waits to refill.
__global__ void __launch_bounds__(kThreads, kCtasPerSm)
    grid_noise_kernel(const uint16_t* __restrict__ W, int64_t total_groups, int levels, double inv_l2,
                      float* __restrict__ gamma, float* __restrict__ sse_asym,
                      float* __restrict__ sse_sym, uint32_t* __restrict__ flags) {
  extern __shared__ __align__(128) uint8_t smem[];
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + kStages * kStageBytes);
  uint32_t* done = reinterpret_cast<uint32_t*>(full + kStages);
  volatile int* abort = reinterpret_cast<volatile int*>(done + kStages);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t nchunks = (total_groups + kChunkGroups - 1) / kChunkGroups;
  const int64_t G = gridDim.x;
  const uint64_t policy = l2_policy_evict_first();
  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&full[s], 1);
      done[s] = 0;
    }
    *abort = 0;
    fence_mbarrier_init();
  }
  __syncthreads();
  if (threadIdx.x == 0)
    for (int s = 0; s < kStages; ++s) {
      const int64_t c = blockIdx.x + G * s;
      if (c < nchunks) issue_chunk(smem + s * kStageBytes, W, c, total_groups, &full[s], policy);
    }

  // Warp w takes groups [w kGroupsPerWarp, (w + 1) kGroupsPerWarp) of each
  // stage; lane sl of a group reads the group's 16-byte chunks kLanes x + sl,
  // x = (r + sub) mod kLoads for r = 0 .. kLoads - 1.
  const int sub = lane / kLanes, sl = lane % kLanes;
  const int gi = warp * kGroupsPerWarp + sub;  // group index inside the stage
  uint32_t seq = 0;
  for (int64_t c = blockIdx.x; c < nchunks; c += G, ++seq) {
    const int s = static_cast<int>(seq % kStages);
    if (!ring_wait(&full[s], (seq / kStages) & 1u, abort)) {
      // Let every copy of this CTA land before it exits.
      if (lane == 0) {
        for (int t = 0; t < kStages; ++t) {
          const uint32_t q = seq + static_cast<uint32_t>((t - s + kStages) % kStages);  // next use of stage t
          mbar_wait_bounded(&full[t], (q / kStages) & 1u);
        }
        if (flags) atomicOr(flags, kFlagTimeout);
      }
      return;
    }
    const int64_t grp = c * kChunkGroups + gi;
    const bool valid = grp < total_groups;
    uint8_t* stage = smem + static_cast<size_t>(s) * kStageBytes;
    const uint8_t* src = stage + gi * (kGroup * 2);
    uint32_t wds[kWords];
    uint32_t dep = 0;
#pragma unroll
    for (int r = 0; r < kLoads; ++r) {
      const int chunk = kLanes * ((r + sub) & (kLoads - 1)) + sl;
      uint4 v = make_uint4(0, 0, 0, 0);
      if (valid) v = *reinterpret_cast<const uint4*>(src + 16 * chunk);
      wds[4 * r] = v.x;
      wds[4 * r + 1] = v.y;
      wds[4 * r + 2] = v.z;
      wds[4 * r + 3] = v.w;
      dep ^= v.x;
    }
    dep = __reduce_or_sync(kFull, dep);
    if (lane == 0 && smem_inc_after(&done[s], dep) % kWarps == kWarps - 1) {
      const int64_t next = c + G * kStages;
      if (next < nchunks) issue_chunk(stage, W, next, total_groups, &full[s], policy);
    }
    noise_group<kLanes, kWords>(wds, grp, valid, levels, inv_l2, gamma, sse_asym, sse_sym, flags);
  }
}

}  // namespace

cudaError_t launch_grid_noise(const uint16_t* W, int64_t N, int64_t K, int bits, float* gamma,
                              float* sse_asym, float* sse_sym, uint32_t* flags, cudaStream_t stream) {
  static SmemAttr smem_attr;
  const int64_t total_groups = N * (K / kGroup);
  int sms = 148, dev = 0;
  if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  cudaError_t e = smem_attr.ensure(grid_noise_kernel, static_cast<int>(kSmemBytes));
  if (e != cudaSuccess) return e;
  const int64_t nchunks = (total_groups + kChunkGroups - 1) / kChunkGroups;
  int64_t blocks = static_cast<int64_t>(sms) * kCtasPerSm;
  if (blocks > nchunks) blocks = nchunks;
  grid_noise_kernel<<<static_cast<unsigned>(blocks), kThreads, kSmemBytes, stream>>>(
      W, total_groups, (1 << bits) - 1, 1.0 / (static_cast<double>((1 << bits) - 1) * ((1 << bits) - 1)),
      gamma, sse_asym, sse_sym, flags);
  return cudaGetLastError();
}

}  // namespace slq
