// quantize.cu -- round-to-nearest asymmetric INT-b encode + LSB-first packing.
//
// Format (pages on "Statistically-Lossless Quantization of Large Language
// Models": gist.science summary, Methodology section 3 "The SLQ Pipeline" --
// asymmetric integer grid, group size 128; GitHub README "Pipeline" -- b in
// {2..8} per layer; GitHub README "4. Build and serve a checkpoint" -- the
// weights are packed to the per-layer bitwidth when loaded).  The encode is
// the plain round-to-nearest baseline the reddit excerpt names (RTN).
//
// Kernel shape: one warp per 128-weight group.  Lane l holds weights
// [4l, 4l+4) (one 8-byte load), the min/max are warp reductions, every
// lane derives the same fp16 scale and zero point, and the 4 codes of a lane
// form a 4b-bit chunk at stream bit 4b*l.  Lane j < 4b then gathers word j of
// the group from the (at most five) lanes whose chunks overlap it and stores
// it, so a group's 4b words leave as one coalesced store.  HBM-bound: 2 bytes
// read and b/8 + 3/128 bytes written per weight.
//
// Bit-exactness with the binary32 definition: IEEE division (__fdiv_rn) for
// the scale and zero point and wherever the reciprocal product could round
// differently (rne_quotient), rintf (round half to even), __float2half_rn
// (round to nearest even, fp16 subnormals kept), no flush-to-zero and no FMA
// contraction on these paths.
#include <cuda_fp16.h>

#include "internal.h"
#include "ptx.cuh"

namespace slq {
namespace {

constexpr unsigned kFull = 0xffffffffu;
constexpr int kWarpsPerBlock = 8;
constexpr int kUnroll = 4;  // groups per warp per iteration (loads in flight)

__device__ __forceinline__ float bf16_lo(uint32_t v) { return __uint_as_float(v << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t v) { return __uint_as_float(v & 0xffff0000u); }

// Warp-wide float min / max in one instruction (sm_100a redux.sync); a NaN
// input is ignored, as with fminf / fmaxf.
__device__ __forceinline__ float warp_min(float v) {
  float r;
  asm volatile("redux.sync.min.f32 %0, %1, 0xffffffff;" : "=f"(r) : "f"(v));
  return r;
}
__device__ __forceinline__ float warp_max(float v) {
  float r;
  asm volatile("redux.sync.max.f32 %0, %1, 0xffffffff;" : "=f"(r) : "f"(v));
  return r;
}

// rne(fl32(w / s)) for the encode.  With r = RN(1/s), t = RN(w r) differs from
// the IEEE quotient fl32(w / s) by at most 1.5 * 2^-23 * |t| (< 1.9e-4 for
// |t| < 1024), so the two round to the same integer unless t lies within that
// distance of a half-integer; those rare elements (exact ties among them) take
// the IEEE division.  Beyond |t| = 1024 the code clamps to an end of the grid
// (|z| <= 255) whichever way the quotient rounds.
__device__ __forceinline__ float rne_quotient(float w, float s, float r) {
  const float t = __fmul_rn(w, r);
  float k = rintf(t);
  if (fabsf(t) < 1024.0f && fabsf(fabsf(t - k) - 0.5f) < 2.5e-4f) k = rintf(__fdiv_rn(w, s));
  return k;
}

template <int B>
__device__ __forceinline__ void encode_group(uint2 raw, int64_t grp, int lane,
                                             uint32_t* __restrict__ packed,
                                             uint16_t* __restrict__ scales,
                                             uint8_t* __restrict__ zeros,
                                             uint32_t* __restrict__ flags) {
  const float w[4] = {bf16_lo(raw.x), bf16_hi(raw.x), bf16_lo(raw.y), bf16_hi(raw.y)};
  const bool nonfinite =
      !(isfinite(w[0]) && isfinite(w[1]) && isfinite(w[2]) && isfinite(w[3]));
  const bool any_nonfinite = __any_sync(kFull, nonfinite);

  // Group statistics: min and max (exact in binary32).
  const float mn = warp_min(fminf(fminf(w[0], w[1]), fminf(w[2], w[3])));
  const float mx = warp_max(fmaxf(fmaxf(w[0], w[1]), fmaxf(w[2], w[3])));

  // A constant group is widened to include 0.
  float lo = mn, hi = mx;
  if (hi == lo) {
    if (lo > 0.0f) lo = 0.0f;
    if (hi < 0.0f) hi = 0.0f;
  }
  constexpr float maxq = static_cast<float>((1 << B) - 1);
  const float s32 = __fdiv_rn(__fsub_rn(hi, lo), maxq);

  // Scale stored in fp16; the encode uses the stored value.
  uint16_t s16;
  bool overflow = false;
  if (s32 == 0.0f) {
    s16 = 0x3C00u;  // all-zero group: 1.0
  } else {
    s16 = __half_as_ushort(__float2half_rn(s32));
    if ((s16 & 0x7FFFu) == 0u) {
      s16 = 0x0001u;  // nonzero step below fp16 range: 2^-24
    } else if (s16 == 0x7C00u) {
      s16 = 0x7BFFu;  // above fp16 range: 65504, flagged
      overflow = true;
    }
  }
  const float s = __half2float(__ushort_as_half(s16));
  const float zf = fminf(fmaxf(rintf(__fdiv_rn(-lo, s)), 0.0f), maxq);

  const float r = __frcp_rn(s);
  uint32_t chunk = 0;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const float v = fminf(fmaxf(__fadd_rn(rne_quotient(w[i], s, r), zf), 0.0f), maxq);
    chunk |= static_cast<uint32_t>(v) << (B * i);
  }

  // Assemble word j = lane of the group's 4B words from the overlapping chunks.
  constexpr int kChunkBits = 4 * B;
  constexpr int kMaxSources = (32 + kChunkBits - 1) / kChunkBits + 1;
  const int j = lane;
  const int first = (32 * j) / kChunkBits;
  uint32_t word = 0;
#pragma unroll
  for (int i = 0; i < kMaxSources; ++i) {
    const int src = first + i;
    const uint32_t v = __shfl_sync(kFull, chunk, src & 31);
    const int off = kChunkBits * src - 32 * j;  // chunk start relative to word start
    if (j < kChunkBits && src < 32 && off < 32 && off > -kChunkBits)
      word |= (off >= 0) ? (v << off) : (v >> (-off));
  }
  if (j < kChunkBits) packed[grp * kChunkBits + j] = word;
  if (lane == 0) {
    scales[grp] = s16;
    zeros[grp] = static_cast<uint8_t>(zf);
    uint32_t f = (any_nonfinite ? kFlagNonfinite : 0u) | (overflow ? kFlagScaleOverflow : 0u);
    if (f && flags) atomicOr(flags, f);
  }
}

template <int B>
__global__ void __launch_bounds__(kWarpsPerBlock * 32)
    quantize_kernel(const uint16_t* __restrict__ W, int64_t total_groups,
                    uint32_t* __restrict__ packed, uint16_t* __restrict__ scales,
                    uint8_t* __restrict__ zeros, uint32_t* __restrict__ flags) {
  const int lane = threadIdx.x & 31;
  const int64_t warp = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  const int64_t nwarps = (static_cast<int64_t>(gridDim.x) * blockDim.x) >> 5;
  for (int64_t base = warp * kUnroll; base < total_groups; base += nwarps * kUnroll) {
    uint2 raw[kUnroll];
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) {
      const int64_t grp = base + u;
      raw[u] = (grp < total_groups) ? ld_stream_v2(W + grp * kGroup + lane * 4) : make_uint2(0, 0);
    }
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) {
      const int64_t grp = base + u;
      if (grp < total_groups) encode_group<B>(raw[u], grp, lane, packed, scales, zeros, flags);
    }
  }
}

template <int B>
cudaError_t launch_b(const uint16_t* W, int64_t total_groups, uint32_t* packed,
                     uint16_t* scales, uint8_t* zeros, uint32_t* flags, cudaStream_t stream) {
  int sms = 148;
  int dev = 0;
  if (cudaGetDevice(&dev) == cudaSuccess)
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const int64_t per_block = kWarpsPerBlock * kUnroll;
  int64_t blocks = (total_groups + per_block - 1) / per_block;
  const int64_t cap = static_cast<int64_t>(sms) * 8;  // 8 resident blocks of 256 threads
  if (blocks > cap) blocks = cap;
  quantize_kernel<B><<<static_cast<unsigned>(blocks), kWarpsPerBlock * 32, 0, stream>>>(
      W, total_groups, packed, scales, zeros, flags);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_quantize(const uint16_t* W, int64_t N, int64_t K, int bits, uint32_t* packed,
                            uint16_t* scales, uint8_t* zeros, uint32_t* flags,
                            cudaStream_t stream) {
  const int64_t total_groups = N * (K / kGroup);
  switch (bits) {
    case 2: return launch_b<2>(W, total_groups, packed, scales, zeros, flags, stream);
    case 3: return launch_b<3>(W, total_groups, packed, scales, zeros, flags, stream);
    case 4: return launch_b<4>(W, total_groups, packed, scales, zeros, flags, stream);
    case 5: return launch_b<5>(W, total_groups, packed, scales, zeros, flags, stream);
    case 6: return launch_b<6>(W, total_groups, packed, scales, zeros, flags, stream);
    case 7: return launch_b<7>(W, total_groups, packed, scales, zeros, flags, stream);
    case 8: return launch_b<8>(W, total_groups, packed, scales, zeros, flags, stream);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace slq
