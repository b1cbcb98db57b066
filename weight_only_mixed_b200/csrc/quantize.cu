// quantize.cu -- round-to-nearest asymmetric INT-b encode + LSB-first packing.
//
// Format (pages on "Statistically-Lossless Quantization of Large Language
// Models": gist.science summary, Methodology section 3 "The SLQ Pipeline" --
// asymmetric integer grid, group size 128; GitHub README "Pipeline" -- b in
// {2..8} per layer; GitHub README "4. Build and serve a checkpoint" -- the
// weights are packed to the per-layer bitwidth when loaded).  The encode is
// the plain round-to-nearest baseline the reddit excerpt names (RTN).
//
// Kernel shape: eight lanes per 128-weight group, four groups per warp.
// Lane sl of a group holds weights [16 sl, 16 sl + 16) (two 16-byte loads),
// the min/max are shuffle reductions inside the eight lanes, and the scale and
// zero point are formed once per lane for its 16 weights.  The 16 codes of a
// lane are 16b consecutive stream bits: whole words for even b, half of a
// lane pair's b words for odd b.  HBM-bound on paper: 2 bytes read and
// b/8 + 3/128 bytes written per weight.
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

// One group per 8 lanes (a warp encodes four groups at once): lane sl of the
// group holds weights [16 sl, 16 sl + 16).  min / max are shuffle reductions
// inside the 8 lanes; the scale and zero point are formed once per lane and
// serve 16 weights.  The 16 codes of a lane are 16b stream bits: for even b
// whole words (b/2 per lane, stored as they are); for odd b a lane pair
// joins its 32b bits into b words with one shuffle.
template <int B>
__device__ __forceinline__ void encode_group8(const uint4 (&raw)[2], int64_t grp, bool valid,
                                              uint32_t* __restrict__ packed,
                                              uint16_t* __restrict__ scales,
                                              uint8_t* __restrict__ zeros,
                                              uint32_t* __restrict__ flags) {
  const int lane = threadIdx.x & 31;
  const int sl = lane & 7;
  const unsigned seg = 0xFFu << (lane & 24);
  const uint32_t wds[8] = {raw[0].x, raw[0].y, raw[0].z, raw[0].w, raw[1].x, raw[1].y, raw[1].z, raw[1].w};
  float w[16];
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    w[2 * i] = bf16_lo(wds[i]);
    w[2 * i + 1] = bf16_hi(wds[i]);
  }
  bool nonfinite = false;
  float mn = w[0], mx = w[0];
#pragma unroll
  for (int i = 0; i < 16; ++i) {
    nonfinite |= !isfinite(w[i]);
    mn = fminf(mn, w[i]);
    mx = fmaxf(mx, w[i]);
  }
  const bool any_nonfinite = (__ballot_sync(kFull, nonfinite) & seg) != 0;
  // Group statistics: min and max (exact in binary32), inside the 8 lanes.
#pragma unroll
  for (int off = 4; off > 0; off >>= 1) {
    mn = fminf(mn, __shfl_xor_sync(kFull, mn, off));
    mx = fmaxf(mx, __shfl_xor_sync(kFull, mx, off));
  }

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

  // The lane's 16 codes as a little-endian bit string of 16b bits.
  constexpr int kLaneWords = (16 * B + 31) / 32;
  uint32_t words[kLaneWords];
#pragma unroll
  for (int k = 0; k < kLaneWords; ++k) words[k] = 0u;
#pragma unroll
  for (int i = 0; i < 16; ++i) {
    const uint32_t q = static_cast<uint32_t>(fminf(fmaxf(__fadd_rn(rne_quotient(w[i], s, r), zf), 0.0f), maxq));
    const int bit = i * B, wi = bit >> 5, sh = bit & 31;
    words[wi] |= q << sh;
    if (sh + B > 32) words[wi + 1] |= q >> (32 - sh);
  }
  uint32_t* out = packed + grp * (4 * B);
  if constexpr (B % 2 == 0) {
    if (valid) {
#pragma unroll
      for (int k = 0; k < B / 2; ++k) out[sl * (B / 2) + k] = words[k];
    }
  } else {
    // Lane pair (even e, odd o): word k of its b words is
    // E[k] | O[k - h] << 16 | O[k - h - 1] >> 16, h = (b - 1) / 2.
    uint32_t other[kLaneWords];
#pragma unroll
    for (int k = 0; k < kLaneWords; ++k) other[k] = __shfl_xor_sync(kFull, words[k], 1);
    const bool odd = sl & 1;
    constexpr int h = (B - 1) / 2;
    constexpr int kEven = (B + 1) / 2;  // words the even lane stores
    auto E = [&](int k) { return (k >= 0 && k < kLaneWords) ? (odd ? other[k] : words[k]) : 0u; };
    auto O = [&](int k) { return (k >= 0 && k < kLaneWords) ? (odd ? words[k] : other[k]) : 0u; };
    if (valid) {
      uint32_t* pw = out + (sl >> 1) * B;
#pragma unroll
      for (int k = 0; k < B; ++k) {
        if ((k < kEven) != odd) pw[k] = E(k) | (O(k - h) << 16) | (O(k - h - 1) >> 16);
      }
    }
  }
  if (valid && sl == 0) {
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
  const int sub = lane >> 3, sl = lane & 7;
  const int64_t warp = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  const int64_t nwarps = (static_cast<int64_t>(gridDim.x) * blockDim.x) >> 5;
  for (int64_t base = warp * 4 * kUnroll; base < total_groups; base += nwarps * 4 * kUnroll) {
    uint4 raw[kUnroll][2];
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) {
      const int64_t grp = base + 4 * u + sub;
      const uint16_t* src = W + grp * kGroup + 16 * sl;
      raw[u][0] = (grp < total_groups) ? ld_stream_v4(src) : make_uint4(0, 0, 0, 0);
      raw[u][1] = (grp < total_groups) ? ld_stream_v4(src + 8) : make_uint4(0, 0, 0, 0);
    }
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) {
      const int64_t grp = base + 4 * u + sub;
      encode_group8<B>(raw[u], grp, grp < total_groups, packed, scales, zeros, flags);
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
  const int64_t per_block = kWarpsPerBlock * 4 * kUnroll;
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
