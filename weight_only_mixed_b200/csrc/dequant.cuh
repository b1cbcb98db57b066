// dequant.cuh -- device helpers shared by the GEMM kernels: reading one
// lane's 32 codes of a packed group out of a TMA-staged (and, for b = 2, 4, 8,
// swizzled) shared-memory tile, turning them into exact bf16 (q - z) pairs,
// and the UMMA shared-memory descriptor.
#pragma once

#include <cuda_bf16.h>
#include <stdint.h>

namespace slq {
namespace dq {

constexpr int kBM = 128;  // W rows per packed tile

// Physical byte offset of a logical offset inside a packed-W stage, for the
// swizzle mode its tensor map uses (128/64/32-byte rows for b = 8/4/2).
template <int B>
__device__ __forceinline__ uint32_t p_swz(uint32_t off) {
  if constexpr (B == 8) return off ^ (((off >> 7) & 7u) << 4);
  else if constexpr (B == 4) return off ^ (((off >> 7) & 3u) << 4);
  else if constexpr (B == 2) return off ^ (((off >> 7) & 1u) << 4);
  else return off;
}

// 2b words (64 codes: units 2h and 2h + 1) of row `row` of a stage, with the
// widest loads the row's alignment allows: when the 32 lanes of a warp read
// 32 consecutive rows, b = 2, 4, 8 are conflict free and the other widths
// at most two-way conflicted.
template <int B>
__device__ __forceinline__ void load_half(const uint8_t* st, int row, int h, uint32_t (&w)[2][B]) {
  uint32_t* f = &w[0][0];
  if constexpr (B == 8 || B == 4 || B == 2 || B == 6) {
    const uint32_t off = row * 16 * B + 8 * B * h;  // 16-byte aligned
#pragma unroll
    for (int i = 0; i < B / 2; ++i) {
      const uint4 v = *reinterpret_cast<const uint4*>(st + p_swz<B>(off + 16 * i));
      f[4 * i] = v.x; f[4 * i + 1] = v.y; f[4 * i + 2] = v.z; f[4 * i + 3] = v.w;
    }
  } else {
    const uint2* p = reinterpret_cast<const uint2*>(st + row * 16 * B + 8 * B * h);  // 8-byte aligned
#pragma unroll
    for (int i = 0; i < B; ++i) {
      const uint2 v = p[i];
      f[2 * i] = v.x; f[2 * i + 1] = v.y;
    }
  }
}

template <int B>
__device__ __forceinline__ uint32_t code_at(const uint32_t (&w)[B], int i) {
  const int o = B * i;
  const int wi = o >> 5;
  const int sh = o & 31;
  constexpr uint32_t mask = (1u << B) - 1u;
  if (sh + B <= 32) return (w[wi] >> sh) & mask;
  return __funnelshift_r(w[wi], w[wi + 1], sh) & mask;
}

__device__ __forceinline__ uint32_t bf16x2_sub(uint32_t a, uint32_t b) {
  __nv_bfloat162 r = __hsub2(*reinterpret_cast<__nv_bfloat162*>(&a),
                             *reinterpret_cast<__nv_bfloat162*>(&b));
  return *reinterpret_cast<uint32_t*>(&r);
}

// The 32 codes of a unit as 16 bf16x2 registers (q_{2p} - z, q_{2p+1} - z),
// consecutive k, exact.  For b <= 7 each code is ORed into the mantissa of
// bf16 128.0 and (128 + z) is subtracted in bf16; b = 8 goes through binary32
// (2^23 + q) - (2^23 + z).  For b = 4 and b = 2 one byte is isolated with a
// byte permute and a multiply by 0x1001 / 0x4001 places its two codes 16 bits
// apart, so a single AND/OR forms the pair.
template <int B>
__device__ __forceinline__ void unit_pairs(const uint32_t (&w)[B], uint32_t z, uint32_t (&out)[16]) {
  if constexpr (B == 8) {
    const float zf = __uint_as_float(0x4B000000u | z);
#pragma unroll
    for (int i = 0; i < 8; ++i) {
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const float lo = __uint_as_float(__byte_perm(w[i], 0x4B000000u, 0x7540 | (2 * h)));
        const float hi = __uint_as_float(__byte_perm(w[i], 0x4B000000u, 0x7540 | (2 * h + 1)));
        __nv_bfloat162 v = __floats2bfloat162_rn(__fsub_rn(lo, zf), __fsub_rn(hi, zf));
        out[2 * i + h] = *reinterpret_cast<uint32_t*>(&v);
      }
    }
  } else {
    const uint32_t z2 = (0x4300u | z) * 0x00010001u;  // bf16x2 (128 + z, 128 + z)
    if constexpr (B == 4) {
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          const uint32_t y = __byte_perm(w[i], 0u, 0x4440 | k) * 0x1001u;
          out[4 * i + k] = bf16x2_sub((y & 0x000F000Fu) | 0x43004300u, z2);
        }
    } else if constexpr (B == 2) {
#pragma unroll
      for (int i = 0; i < 2; ++i)
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          const uint32_t y = __byte_perm(w[i], 0u, 0x4440 | k) * 0x4001u;
          out[8 * i + 2 * k] = bf16x2_sub((y & 0x00030003u) | 0x43004300u, z2);
          out[8 * i + 2 * k + 1] = bf16x2_sub(((y >> 4) & 0x00030003u) | 0x43004300u, z2);
        }
    } else {
#pragma unroll
      for (int p = 0; p < 16; ++p)
        out[p] = bf16x2_sub(code_at<B>(w, 2 * p) | (code_at<B>(w, 2 * p + 1) << 16) | 0x43004300u, z2);
    }
  }
}

// UMMA shared-memory descriptor: K-major, 128-byte swizzle, 8-row groups
// 1024 bytes apart (SBO), descriptor version 1 (sm_100).
__device__ __forceinline__ uint64_t sw128_desc(uint32_t saddr) {
  return static_cast<uint64_t>((saddr >> 4) & 0x3FFFu) | (static_cast<uint64_t>(1) << 16) |
         (static_cast<uint64_t>(1024 >> 4) << 32) | (static_cast<uint64_t>(1) << 46) |
         (static_cast<uint64_t>(2) << 61);
}

}  // namespace dq
}  // namespace slq
