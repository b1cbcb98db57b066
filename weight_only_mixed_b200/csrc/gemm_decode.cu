// gemm_decode.cu -- dequantize-GEMM for decode batches (M <= 16): packed
// weights streamed by TMA, dequantized in registers straight into tensor-core
// fragments, and a persistent stream-K split over the SMs.
//
// Y = X W^T, w = s * (q - z) (the weight-only linear layer of the pages'
// serving path; gist.science summary, Key Results "Inference Speedup").  At
// decode sizes the layer must stream the packed weights at HBM speed, so the
// kernel is built around the weight stream:
//
//   * warp 0 streams chunks of the layer (128 weight rows x GS consecutive
//     128-code groups, 16b*GS bytes per row -- 128 bytes where b allows, with
//     the 128-byte swizzle) into a shared-memory ring with TMA.  Short row
//     segments make a slow stream: on this B200 a TMA box of 128 rows x 32
//     bytes moves under 1.4 TB/s over the GPU, one of 128 rows x 128 bytes
//     about 3.5x that;
//   * warp 1 stages the activations of the group (M <= 16 rows x 128 k) with
//     8-byte cp.async copies, already laid out as mma B fragments;
//   * eight consumer warps own 16 weight rows each.  A thread reads its 32
//     codes of two rows (b words each), turns them into exact bf16 (q - z)
//     pairs in registers, and issues mma.sync.m16n8k16 with those registers
//     as the A fragment -- the dequantized weights never touch shared or
//     tensor memory.  The group's fp32 product is scaled by the fp16 group
//     scale and added to fp32 accumulators, so the only rounding is fp32
//     accumulation.
//
// Why mma.sync and not tcgen05 here: on this B200 a tcgen05.mma of
// M = 128, K = 16 occupies the tensor pipe for about 40 cycles whatever N is,
// and N = 16 is the smallest N with M = 128, so a decode product runs at
// about 800 MAC/clk/SM and needs a TMEM round trip per group; mma.sync
// m16n8k16 sustains about 1000 MAC/clk/SM with the A operand in registers,
// which bounds this kernel at 128 (M <= 8) or 64 (M <= 16) weights per clock
// per SM -- above the rate at which HBM delivers packed weights.
//
// The thread-to-k mapping.  Within a group, thread t (= lane % 4) of a row
// quad owns codes [32t, 32t + 32) -- one contiguous 4b-byte unit of the packed
// row -- and its k-step j uses codes 32t + 4j .. 32t + 4j + 3.  The mma's k
// order is a permutation of the group's k; the activation fragments are
// staged with the same permutation (b0 = X[m][32t + 4j + 0..1], b1 =
// X[m][32t + 4j + 2..3]), so the product is the plain dot product.
//
// Work split.  The layer is ceil(N/128) row tiles x G/GS chunks; each CTA
// (two per SM) takes a contiguous share of the row-major list of chunks
// (stream-K), so every SM streams the same number of bytes whatever N and K
// are.  A row tile whose groups fall in one CTA is
// written straight to Y.  A row tile shared by several CTAs is reduced
// deterministically: each CTA writes its fp32 partial to slot (CTA - first CTA
// of the tile) of a caller-provided workspace and increments the tile's
// counter; the CTA that completes the count adds the slots in slot order,
// writes Y and resets the counter to zero.  The result does not depend on
// which CTA finishes first.
//
// Every hand-over is an mbarrier; every wait gives up after about 2 s,
// raises SLQ_FLAG_TIMEOUT and lets the CTA drain its copies and exit.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include <mutex>

#include "dequant.cuh"
#include "internal.h"
#include "ptx.cuh"

namespace slq {
namespace {


constexpr int kRows = 256;       // weight rows per tile
constexpr int kMaxM = 16;        // activation rows (two n8 mma tiles)
constexpr int kConsumers = 8;    // consumer warps, 32 rows (two m16 mma tiles) each
constexpr int kWarpW = 0, kWarpX = 1, kWarpC0 = 2;
constexpr int kThreads = (kWarpC0 + kConsumers) * 32;
constexpr int kCtasPerSm = 2;
constexpr int kSX = 6;                 // activation fragment stages (one group each)
constexpr int kXFrag = 8 * 32 * 8;     // one n8 tile of a group: 8 k-steps x 32 lanes x 8 B
constexpr int kMaxPending = 4;         // shared tiles per CTA (at most 2 occur)
constexpr int kMinChunksPerCta = 2;  // fewer CTAs rather than one-chunk slivers
// Workspace layout: tile counters in a fixed region at the front, partial sums
// after it.  The counter region is the same for every layer, so partial sums
// of one layer can never land on another layer's counters when callers reuse
// one workspace for layers of different sizes.
constexpr size_t kCounterBytes = size_t{64} << 10;
constexpr int64_t kMaxRowTiles = kCounterBytes / sizeof(int);

template <int B>
constexpr int p_stage_bytes() {
  return kRows * 16 * B;
}

struct Pending {
  int rb, ncover, last;
};

// Groups per chunk: rows of 128 bytes (the 128-byte swizzle span) for
// b = 2, 4, 8; the widest row up to 128 bytes otherwise.
template <int B>
constexpr int chunk_groups() {
  return B == 2 ? 4 : (B == 3 || B == 4) ? 2 : 1;
}

template <int B>
constexpr bool chunk_swizzled() {
  return 16 * B * chunk_groups<B>() == 128;
}

template <int B, int NT, int GS>
struct Cfg {
  static constexpr int kXStage = NT * kXFrag;
  static constexpr int kStage = GS * p_stage_bytes<B>();
  static constexpr int kSZStage = kRows * 12;  // per row: GS fp16 scales (8 B) + GS zeros (4 B)
  static constexpr int kFixed = 1024 /* alignment slack */ + kSX * kXStage +
                                1024 /* barriers, pending list */;
  static constexpr int kBudget = 227 * 1024 / kCtasPerSm - 1024 /* static + reserved */;
  static constexpr int kSPRaw = (kBudget - kFixed) / (kStage + kSZStage);
  static constexpr int kSP = kSPRaw > 16 ? 16 : kSPRaw;
  static constexpr int kSmem = kFixed + kSP * (kStage + kSZStage);
  static_assert(kSPRaw >= 2, "shared memory budget");
};

// The b words (32 codes) of unit t of group gs of row `row` in a chunk stage
// (rows of 16*B*GS bytes; 128-byte swizzle when the row is 128 bytes).
template <int B, int GS>
__device__ __forceinline__ void load_codes(const uint8_t* st, int row, int gs, int t,
                                           uint32_t (&w)[B]) {
  constexpr int kRowBytes = 16 * B * GS;
  const uint32_t off = row * kRowBytes + gs * 16 * B + 4 * B * t;
  if constexpr (kRowBytes == 128) {
    auto phys = [](uint32_t o) { return o ^ (((o >> 7) & 7u) << 4); };
    if constexpr (B == 8) {
      const uint4 v0 = *reinterpret_cast<const uint4*>(st + phys(off));
      const uint4 v1 = *reinterpret_cast<const uint4*>(st + phys(off + 16));
      w[0] = v0.x; w[1] = v0.y; w[2] = v0.z; w[3] = v0.w;
      w[4] = v1.x; w[5] = v1.y; w[6] = v1.z; w[7] = v1.w;
    } else if constexpr (B == 4) {
      const uint4 v = *reinterpret_cast<const uint4*>(st + phys(off));
      w[0] = v.x; w[1] = v.y; w[2] = v.z; w[3] = v.w;
    } else {
      static_assert(B == 2, "128-byte rows are used for b = 2, 4, 8");
      const uint2 v = *reinterpret_cast<const uint2*>(st + phys(off));
      w[0] = v.x; w[1] = v.y;
    }
  } else if constexpr (B == 6) {
    // 24 bytes at an 8-byte aligned offset.
#pragma unroll
    for (int i = 0; i < 3; ++i) {
      const uint2 v = *reinterpret_cast<const uint2*>(st + off + 8 * i);
      w[2 * i] = v.x; w[2 * i + 1] = v.y;
    }
  } else {
    const uint32_t* p = reinterpret_cast<const uint32_t*>(st + off);
#pragma unroll
    for (int i = 0; i < B; ++i) w[i] = p[i];
  }
}

struct Bars {
  uint64_t* p_full;   // [kSP] packed stage landed (TMA)
  uint64_t* p_empty;  // [kSP] packed stage read (kConsumers warps)
  uint64_t* x_full;   // [kSX] activation fragments landed (32 cp.async lanes)
  uint64_t* x_empty;  // [kSX] activation fragments read (kConsumers warps)
  uint64_t* seg_bar;  // consumers' partials of a shared tile written (kConsumers)
  uint64_t* end_bar;  // the leader has recorded every shared tile (1)
  volatile int* abort_flag;
  Pending* pending;
  int* npending;
};

__device__ __forceinline__ bool wait_or_abort(uint64_t* bar, uint32_t parity, const Bars& sh,
                                              uint32_t* flags) {
  if (mbar_try_wait(bar, parity)) return true;
  const long long t0 = clock64();
  while (true) {
#pragma unroll 1
    for (int i = 0; i < 8; ++i)
      if (mbar_try_wait(bar, parity)) return true;
    if (*sh.abort_flag) return false;
    if (clock64() - t0 > kWaitLimitCycles) {
      *sh.abort_flag = 1;
      if (flags) atomicOr(flags, kFlagTimeout);
      return false;
    }
  }
}

__device__ __forceinline__ uint32_t atom_add_acq_rel(int* p, int v) {
  uint32_t old;
  asm volatile("atom.acq_rel.gpu.global.add.u32 %0, [%1], %2;" : "=r"(old) : "l"(p), "r"(v) : "memory");
  return old;
}

__device__ __forceinline__ uint2 lds_v2(const void* p) {
  uint2 r;
  asm volatile("ld.shared.v2.u32 {%0, %1}, [%2];" : "=r"(r.x), "=r"(r.y) : "r"(smem_u32(p)));
  return r;
}

// Pair p (0..15) of a thread's unit as exact bf16 (q - z, q' - z) for the
// consecutive codes 2p, 2p + 1; pair p feeds k-step p / 2 (even p: mma k 2t,
// 2t+1; odd p: 2t+8, 2t+9).  z2 is bf16x2 (128 + z, 128 + z) for b <= 7, zf
// the binary32 2^23 + z for b = 8.  For b = 4 (b = 2) a byte with the pair
// (two pairs) is isolated with a byte permute and a multiply by 0x1001
// (0x4001) places its codes 16 bits apart, so one LOP3 forms the pair.
template <int B>
__device__ __forceinline__ uint32_t pair_of(const uint32_t (&w)[B], uint32_t z2, float zf, int p) {
  if constexpr (B == 4) {
    const uint32_t y = __byte_perm(w[p >> 2], 0u, 0x4440 | (p & 3)) * 0x1001u;
    return dq::bf16x2_sub((y & 0x000F000Fu) | 0x43004300u, z2);
  } else if constexpr (B == 2) {
    const uint32_t y = __byte_perm(w[p >> 3], 0u, 0x4440 | ((p >> 1) & 3)) * 0x4001u;
    return dq::bf16x2_sub(((y >> (4 * (p & 1))) & 0x00030003u) | 0x43004300u, z2);
  } else if constexpr (B == 8) {
    const uint32_t word = w[p >> 1];
    const int h = p & 1;
    const float lo = __uint_as_float(__byte_perm(word, 0x4B000000u, 0x7540 | (2 * h)));
    const float hi = __uint_as_float(__byte_perm(word, 0x4B000000u, 0x7540 | (2 * h + 1)));
    __nv_bfloat162 v = __floats2bfloat162_rn(__fsub_rn(lo, zf), __fsub_rn(hi, zf));
    return *reinterpret_cast<uint32_t*>(&v);
  } else {
    return dq::bf16x2_sub(dq::code_at<B>(w, 2 * p) | (dq::code_at<B>(w, 2 * p + 1) << 16) | 0x43004300u,
                          z2);
  }
}

// GS consecutive fp16 scales / uint8 zeros of one row (aligned: G % GS == 0).
template <int GS>
__device__ __forceinline__ uint2 ld_scales(const uint16_t* p) {
  if constexpr (GS == 4) return ld_ro_v2(p);
  else if constexpr (GS == 2) return make_uint2(ld_ro_u32(p), 0u);
  else return make_uint2(static_cast<uint32_t>(*p), 0u);
}
template <int GS>
__device__ __forceinline__ uint32_t ld_zeros(const uint8_t* p) {
  if constexpr (GS == 4) return ld_ro_u32(p);
  else if constexpr (GS == 2) return static_cast<uint32_t>(*reinterpret_cast<const uint16_t*>(p));
  else return static_cast<uint32_t>(*p);
}
__device__ __forceinline__ float scale_at(uint2 v, int gs) {
  const uint32_t w = gs < 2 ? v.x : v.y;
  return __half2float(__ushort_as_half(static_cast<uint16_t>(w >> (16 * (gs & 1)))));
}

// Stream-K geometry shared by every CTA of a launch.
struct Split {
  int G;        // chunks per row tile (groups / GS)
  int per;      // chunks per CTA
  int nctas;    // CTAs launched
  int s_max;    // partial slots per row tile in the workspace
};

__device__ __forceinline__ int first_cta(const Split& sp, int rb) {
  return static_cast<int>((static_cast<int64_t>(rb) * sp.G) / sp.per);
}
__device__ __forceinline__ int last_cta(const Split& sp, int rb) {
  const int c = static_cast<int>((static_cast<int64_t>(rb) * sp.G + sp.G - 1) / sp.per);
  return c < sp.nctas - 1 ? c : sp.nctas - 1;
}

__device__ __forceinline__ void store_y(void* Y, int y_f32, int64_t o, float v) {
  if (y_f32)
    static_cast<float*>(Y)[o] = v;
  else
    static_cast<__nv_bfloat16*>(Y)[o] = __float2bfloat16_rn(v);
}

template <int B, int NT, int GS>
__global__ void __launch_bounds__(kThreads, kCtasPerSm)
    gemm_decode_kernel(const __grid_constant__ CUtensorMap tmap_w, const uint16_t* __restrict__ X,
                       int M, int N, int K, const uint16_t* __restrict__ scales,
                       const uint8_t* __restrict__ zeros, void* __restrict__ Y, int y_f32, Split sp,
                       int* __restrict__ counters, float* __restrict__ partials,
                       uint32_t* __restrict__ flags) {
  using C = Cfg<B, NT, GS>;
  constexpr int kSP = C::kSP;
  constexpr int kStage = C::kStage;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw_addr = smem_u32(smem_raw);
  uint8_t* smem = smem_raw + (((raw_addr + 1023u) & ~1023u) - raw_addr);
  uint8_t* pbuf = smem;                  // [kSP][128 rows][16 B GS bytes], TMA layout
  uint8_t* xbuf = pbuf + kSP * kStage;   // [kSX][NT][8 k-steps][32 lanes][8 B]
  uint8_t* szbuf = xbuf + kSX * C::kXStage;  // [kSP][kRows] uint2 scales, then [kSP][kRows] u32 zeros
  uint2* sc_st = reinterpret_cast<uint2*>(szbuf);
  uint32_t* zc_st = reinterpret_cast<uint32_t*>(szbuf + kSP * kRows * 8);
  uint64_t* bars = reinterpret_cast<uint64_t*>(szbuf + kSP * C::kSZStage);
  Bars sh;
  sh.p_full = bars;
  sh.p_empty = sh.p_full + kSP;
  sh.x_full = sh.p_empty + kSP;
  sh.x_empty = sh.x_full + kSX;
  sh.seg_bar = sh.x_empty + kSX;
  sh.end_bar = sh.seg_bar + 1;
  sh.abort_flag = reinterpret_cast<volatile int*>(sh.end_bar + 1);
  sh.npending = const_cast<int*>(sh.abort_flag) + 1;
  sh.pending = reinterpret_cast<Pending*>(sh.npending + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int G = sp.G * GS;  // groups per row
  const int Gc = sp.G;      // chunks per row
  const int rbs = (N + kRows - 1) / kRows;
  const int64_t total = static_cast<int64_t>(rbs) * Gc;
  const int64_t t0 = static_cast<int64_t>(blockIdx.x) * sp.per;
  const int64_t t1 = (t0 + sp.per) < total ? (t0 + sp.per) : total;
  const int nc = static_cast<int>(t1 - t0);  // chunks of this CTA
  const int ng = nc * GS;                    // groups of this CTA
  const int rb0 = static_cast<int>(t0 / Gc), gk0 = static_cast<int>(t0 % Gc) * GS;

  if (threadIdx.x == 0) {
    for (int i = 0; i < kSP; ++i) {
      mbar_init(&sh.p_full[i], 1);
      mbar_init(&sh.p_empty[i], kConsumers);
    }
    for (int i = 0; i < kSX; ++i) {
      mbar_init(&sh.x_full[i], 32);
      mbar_init(&sh.x_empty[i], kConsumers);
    }
    mbar_init(sh.seg_bar, kConsumers);
    mbar_init(sh.end_bar, 1);
    *sh.abort_flag = 0;
    *sh.npending = 0;
    fence_mbarrier_init();
  }
  // Launched as a programmatic dependent of the previous kernel on the stream:
  // everything above overlapped its tail.  Before waiting for it, the first
  // chunks of packed weights are prefetched into L2 (a prefetch cannot make
  // a later read stale: L2 is where writes land); no global memory is read
  // into the SM or written before the previous kernel has completed.
  if (warp == kWarpW && lane == 0) {
    int rb = rb0, gc = gk0 / GS;
    for (int ci = 0; ci < nc && ci < kSP; ++ci) {
      tma_prefetch_l2_2d(&tmap_w, gc * 4 * B * GS, rb * kRows);
      if (++gc == Gc) {
        gc = 0;
        ++rb;
      }
    }
  }
  grid_dependency_wait();
  __syncthreads();

  if (warp == kWarpW) {
    // ---------------- packed-W producer (TMA) + scale / zero staging ----------------
    // Lane 0 issues the chunk's TMA; every lane stages the GS scales and GS
    // zeros of rows 8l..8l+7 of the chunk into the stage's slot (one vector
    // load per row, loaded one chunk ahead; rows past N and chunks past the
    // range read clamped, valid addresses).  The stage is published by one
    // arrival after the stores, with the TMA bytes on the same phase.
    if (lane == 0) prefetch_tmap(&tmap_w);
    int rb = rb0, gc = gk0 / GS;
    int frb = rb0, fgc = gc;
    // Two chunks of scales / zeros in flight (ring slot = chunk parity, so
    // the loop is unrolled by two to keep the slot a compile-time index).
    uint2 ns[2][8];
    uint32_t nz[2][8];
    auto sz_fetch = [&](uint2 (&ds)[8], uint32_t (&dz)[8]) {
      const int rbc = min(frb, rbs - 1) * kRows;
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const int64_t gi = static_cast<int64_t>(min(rbc + 8 * lane + i, N - 1)) * G + fgc * GS;
        ds[i] = ld_scales<GS>(scales + gi);
        dz[i] = ld_zeros<GS>(zeros + gi);
      }
      if (++fgc == Gc) {
        fgc = 0;
        ++frb;
      }
    };
    sz_fetch(ns[0], nz[0]);
    sz_fetch(ns[1], nz[1]);
    int issued = 0;
    bool run = true;
    for (int c0 = 0; c0 < nc && run; c0 += 2) {
#pragma unroll
      for (int jj = 0; jj < 2; ++jj) {
        const int ci = c0 + jj;
        if (ci < nc && run) {
          const int s = ci % kSP;
          if (__all_sync(0xffffffffu, wait_or_abort(&sh.p_empty[s], ((ci / kSP) & 1) ^ 1, sh, flags))) {
            if (lane == 0) {
              mbar_expect_tx(&sh.p_full[s], kStage);
              tma_load_2d(pbuf + s * kStage, &tmap_w, &sh.p_full[s], gc * 4 * B * GS, rb * kRows);
            }
#pragma unroll
            for (int i = 0; i < 8; ++i) {
              sc_st[s * kRows + 8 * lane + i] = ns[jj][i];
              zc_st[s * kRows + 8 * lane + i] = nz[jj][i];
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&sh.p_full[s]);
            sz_fetch(ns[jj], nz[jj]);  // chunk ci + 2
            ++issued;
            if (++gc == Gc) {
              gc = 0;
              ++rb;
            }
          } else {
            run = false;
          }
        }
      }
    }
    grid_launch_dependents();
    if (lane == 0)  // every issued copy lands before exit
      for (int i = issued - kSP; i < issued; ++i)
        if (i >= 0) mbar_wait_bounded(&sh.p_full[i % kSP], (i / kSP) & 1);
    __syncwarp();
  } else if (warp == kWarpX) {
    // ---------------- activation fragments (rows >= M are zero) ----------------
    // Fragment slot (nt, j, l), m = 8nt + l / 4, t = l % 4, holds
    // X[m][k0 + 32t + 4j .. + 3]: the B fragment of k-step j for activation
    // rows 8nt..8nt+7.  One instruction copies one activation row of the group
    // (256 contiguous bytes): lane L takes bytes [8L, 8L + 8), i.e. t = L / 8,
    // j = L % 8.  Rows >= M are not copied -- they only reach output columns
    // >= M, which are never stored.  Each lane's arrival fires when its copies
    // have landed, so this warp never waits for data, only for free stages.
    int gk = gk0;
    const int jl = lane & 7, tl = lane >> 3;
    for (int g = 0; g < ng; ++g, gk = (gk + 1 == G) ? 0 : gk + 1) {
      const int s = g % kSX;
      if (!__all_sync(0xffffffffu,
                      wait_or_abort(&sh.x_empty[s], ((g / kSX) & 1) ^ 1, sh, flags)))
        break;
      uint8_t* stage = xbuf + s * C::kXStage;
      const uint16_t* src = X + gk * kGroup + 4 * lane;
      for (int m = 0; m < M; ++m) {
        const int nt = m >> 3, n = m & 7;
        cp_async_8(stage + (nt * 8 + jl) * 256 + (4 * n + tl) * 8, src + static_cast<int64_t>(m) * K, 8u);
      }
      cp_async_mbar_arrive(&sh.x_full[s]);
    }
    grid_launch_dependents();
    cp_async_wait<0>();  // nothing in flight past this point
    __syncwarp();
  } else {
    // ---------------- consumers: rows 32c + lane / 4 + {0, 8, 16, 24} of the tile ----------------
    // Rows 0, 1 of the thread form the m16 tile "A" of the warp, rows 2, 3
    // tile "B"; both share each activation fragment.
    const int c = warp - kWarpC0;
    const int t = lane & 3;
    int rr[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) rr[i] = 32 * c + (lane >> 2) + 8 * i;
    const bool leader = threadIdx.x == kWarpC0 * 32;
    float acc[2][NT][4];
#pragma unroll
    for (int h = 0; h < 2; ++h)
#pragma unroll
      for (int nt = 0; nt < NT; ++nt)
#pragma unroll
        for (int e = 0; e < 4; ++e) acc[h][nt][e] = 0.0f;

    bool ok = true;
    int nseg = 0;  // shared row tiles met so far (the same count in every consumer warp)
    int rb = rb0, gk = gk0;
    for (int ci = 0; ci < nc && ok; ++ci) {
      const int sp_ = ci % kSP;
      ok = __all_sync(0xffffffffu, wait_or_abort(&sh.p_full[sp_], (ci / kSP) & 1, sh, flags));
      if (!ok) break;
      // This chunk's scales and zeros of the four rows (staged with the codes).
      uint2 cs[4];
      uint32_t cz[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        cs[i] = sc_st[sp_ * kRows + rr[i]];
        cz[i] = zc_st[sp_ * kRows + rr[i]];
      }
      const uint8_t* pst = pbuf + sp_ * kStage;
#pragma unroll
      for (int gs = 0; gs < GS; ++gs) {
        const int g = ci * GS + gs;
        const int sx = g % kSX;
        if (ok)
          ok = __all_sync(0xffffffffu, wait_or_abort(&sh.x_full[sx], (g / kSX) & 1, sh, flags));
        if (ok) {
          // ---- codes of the four rows ----
          uint32_t w[4][B];
#pragma unroll
          for (int i = 0; i < 4; ++i) load_codes<B, GS>(pst, rr[i], gs, t, w[i]);
          if (gs == GS - 1) {
            // Release the stage only after every code word of this warp has
            // arrived in registers (the TMA refill may overwrite it at once),
            // ordered before the async proxy's writes.
            uint32_t dep = 0;
#pragma unroll
            for (int i = 0; i < 4; ++i) {
              dep ^= cs[i].x ^ cs[i].y ^ cz[i];
#pragma unroll
              for (int k = 0; k < B; ++k) dep ^= w[i][k];
            }
            fence_proxy_async_smem();
            __syncwarp();
            dep = __any_sync(0xffffffffu, dep != 0);
            if (lane == 0) mbar_arrive_after(&sh.p_empty[sp_], dep);
          }
          uint32_t z2[4];
          float zf[4];
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            const uint32_t z = (cz[i] >> (8 * gs)) & 0xFFu;
            z2[i] = (0x4300u | z) * 0x00010001u;
            zf[i] = __uint_as_float(0x4B000000u | z);
          }

          // ---- 8 k-steps x 2 m16 tiles; pairs made as they are used ----
          float d[2][NT][4];
#pragma unroll
          for (int h = 0; h < 2; ++h)
#pragma unroll
            for (int nt = 0; nt < NT; ++nt)
#pragma unroll
              for (int e = 0; e < 4; ++e) d[h][nt][e] = 0.0f;
          const uint8_t* xs = xbuf + sx * C::kXStage + lane * 8;
#pragma unroll
          for (int ks = 0; ks < 8; ++ks) {
            uint2 bfr[NT];
#pragma unroll
            for (int nt = 0; nt < NT; ++nt) bfr[nt] = lds_v2(xs + (nt * 8 + ks) * 256);
#pragma unroll
            for (int h = 0; h < 2; ++h) {
              const int ra = 2 * h, rb_ = 2 * h + 1;
              const uint32_t a0 = pair_of<B>(w[ra], z2[ra], zf[ra], 2 * ks);
              const uint32_t a1 = pair_of<B>(w[rb_], z2[rb_], zf[rb_], 2 * ks);
              const uint32_t a2 = pair_of<B>(w[ra], z2[ra], zf[ra], 2 * ks + 1);
              const uint32_t a3 = pair_of<B>(w[rb_], z2[rb_], zf[rb_], 2 * ks + 1);
#pragma unroll
              for (int nt = 0; nt < NT; ++nt)
                mma_bf16_16816(d[h][nt], a0, a1, a2, a3, bfr[nt].x, bfr[nt].y);
            }
          }
          {
            // Release the activation stage once every mma that read it has
            // consumed its fragments (a dependency on all the accumulators).
            uint32_t dep = 0;
#pragma unroll
            for (int h = 0; h < 2; ++h)
#pragma unroll
              for (int nt = 0; nt < NT; ++nt) dep ^= __float_as_uint(d[h][nt][0]);
            __syncwarp();
            dep = __any_sync(0xffffffffu, dep != 0);
            if (lane == 0) mbar_arrive_after(&sh.x_empty[sx], dep);
          }
#pragma unroll
          for (int h = 0; h < 2; ++h) {
            const float sa = scale_at(cs[2 * h], gs), sb = scale_at(cs[2 * h + 1], gs);
#pragma unroll
            for (int nt = 0; nt < NT; ++nt) {
              acc[h][nt][0] = fmaf(sa, d[h][nt][0], acc[h][nt][0]);
              acc[h][nt][1] = fmaf(sa, d[h][nt][1], acc[h][nt][1]);
              acc[h][nt][2] = fmaf(sb, d[h][nt][2], acc[h][nt][2]);
              acc[h][nt][3] = fmaf(sb, d[h][nt][3], acc[h][nt][3]);
            }
          }

          // ---- end of this CTA's part of a row tile: write it out ----
          if (gk == G - 1 || g == ng - 1) {
            const int c0 = first_cta(sp, rb);  // in chunks: sp.G = Gc
            const int ncover = last_cta(sp, rb) - c0 + 1;
            if (ncover == 1) {
#pragma unroll
              for (int h = 0; h < 2; ++h)
#pragma unroll
                for (int nt = 0; nt < NT; ++nt)
#pragma unroll
                  for (int e = 0; e < 4; ++e) {
                    const int m = 8 * nt + 2 * t + (e & 1);
                    const int n = rb * kRows + rr[2 * h + (e >> 1)];
                    if (m < M && n < N) store_y(Y, y_f32, static_cast<int64_t>(m) * N + n, acc[h][nt][e]);
                  }
            } else {
              const int slot = static_cast<int>(blockIdx.x) - c0;
              float* part = partials + (static_cast<int64_t>(rb) * sp.s_max + slot) * (kMaxM * kRows);
#pragma unroll
              for (int h = 0; h < 2; ++h)
#pragma unroll
                for (int nt = 0; nt < NT; ++nt)
#pragma unroll
                  for (int e = 0; e < 4; ++e) {
                    const int m = 8 * nt + 2 * t + (e & 1);
                    if (m < M) part[m * kRows + rr[2 * h + (e >> 1)]] = acc[h][nt][e];
                  }
              // Each writer makes its partial visible at GPU scope before the
              // tile's counter can be advanced (the CTA barrier below is CTA
              // scope only).
              __threadfence();
              __syncwarp();
              if (lane == 0) mbar_arrive(sh.seg_bar);
              if (leader && wait_or_abort(sh.seg_bar, nseg & 1, sh, flags)) {
                // Every consumer's partial is written and fenced; the atomic
                // orders the count after them.
                const uint32_t old = atom_add_acq_rel(counters + rb, 1);
                const int np = *sh.npending;
                if (np < kMaxPending) {
                  sh.pending[np] = Pending{rb, ncover, static_cast<int>(old) == ncover - 1 ? 1 : 0};
                  *sh.npending = np + 1;
                }
              }
              ++nseg;
            }
#pragma unroll
            for (int h = 0; h < 2; ++h)
#pragma unroll
              for (int nt = 0; nt < NT; ++nt)
#pragma unroll
                for (int e = 0; e < 4; ++e) acc[h][nt][e] = 0.0f;
          }
          if (++gk == G) {
            gk = 0;
            ++rb;
          }
        }
      }
    }

    // The next kernel on the stream may be scheduled once every CTA is here.
    grid_launch_dependents();
    // Shared row tiles this CTA completed last: add the slots in slot order.
    if (leader) mbar_arrive(sh.end_bar);
    ok = __all_sync(0xffffffffu, ok && wait_or_abort(sh.end_bar, 0, sh, flags));
    if (ok) {
      const int np = *sh.npending;
      const int ct = threadIdx.x - kWarpC0 * 32;  // 0 .. 32 * kConsumers - 1 == kRows - 1
      static_assert(32 * kConsumers == kRows, "one reducing thread per tile row");
      for (int e = 0; e < np; ++e) {
        const Pending pe = sh.pending[e];
        if (!pe.last) continue;
        __threadfence();
        // Thread ct owns row ct of the tile for every activation row m < M.
        // The slots are added in slot order; the loads of four slots x all m
        // are issued together so that the L2 latency is paid once per four
        // slots, not once per value.
        const float* base = partials + static_cast<int64_t>(pe.rb) * sp.s_max * (kMaxM * kRows) + ct;
        float v[kMaxM];
#pragma unroll
        for (int m = 0; m < kMaxM; ++m) v[m] = m < M ? __ldcg(base + m * kRows) : 0.0f;
        for (int c0 = 1; c0 < pe.ncover; c0 += 4) {
          float u[4][kMaxM];
#pragma unroll
          for (int cc = 0; cc < 4; ++cc)
#pragma unroll
            for (int m = 0; m < kMaxM; ++m)
              u[cc][m] = (c0 + cc < pe.ncover && m < M)
                             ? __ldcg(base + (c0 + cc) * (kMaxM * kRows) + m * kRows)
                             : 0.0f;
#pragma unroll
          for (int cc = 0; cc < 4; ++cc)
#pragma unroll
            for (int m = 0; m < kMaxM; ++m)
              if (c0 + cc < pe.ncover) v[m] += u[cc][m];
        }
        const int n = pe.rb * kRows + ct;
        if (n < N) {
#pragma unroll
          for (int m = 0; m < kMaxM; ++m)
            if (m < M) store_y(Y, y_f32, static_cast<int64_t>(m) * N + n, v[m]);
        }
        if (leader) counters[pe.rb] = 0;  // ready for the next call
      }
    }
  }
  __syncthreads();
}

// ---------------------------------------------------------------------------
// Split-K GEMV (M <= 16) without workspace.  A CTA owns 16 * RT consecutive
// weight rows; its S warps split the rows' groups into S contiguous K ranges.
// Each warp streams its rows' groups (16b bytes per row and group) through a
// private D-stage shared-memory ring with 16-byte cp.async copies, GB groups
// per stage, so D - 1 stages are in flight per warp without holding
// registers.  A thread then reads its 4b-byte unit of each of its 2 * RT rows
// and feeds the pairs to mma.sync as above; the activation fragments come
// through L1; the S partial tiles are added in shared memory in warp order
// (deterministic, no cross-CTA step).
//
// The zero point leaves the inner loop: the A pairs are the codes themselves
// as exact bf16 values code * 2^(c - 133) (pair_sub), the activation pairs
// that meet them are x * 2^(E - c) for one exponent E per group, one more mma
// per k-step with A = 2^(c - 133) gives Sx = sum_k x 2^(E - 133), and the
// group's product is s * 2^(133 - E) * (sum q x 2^(E - 133) - z Sx), every
// scaling a power of two.  For b = 2 and 4 a pair takes two codes 16 bits
// apart in one word (one mask; one shift by 8 per word for the codes in the
// upper bytes) and the activation pairs are permuted to the same k order.
// ---------------------------------------------------------------------------
template <int B>
__device__ __forceinline__ void lds_unit(const uint8_t* p, uint32_t (&w)[B]) {
  if constexpr (B == 4 || B == 8) {
#pragma unroll
    for (int i = 0; i < B / 4; ++i) {
      const uint4 v = *reinterpret_cast<const uint4*>(p + 16 * i);
      w[4 * i] = v.x; w[4 * i + 1] = v.y; w[4 * i + 2] = v.z; w[4 * i + 3] = v.w;
    }
  } else if constexpr (B == 2 || B == 6) {
#pragma unroll
    for (int i = 0; i < B / 2; ++i) {
      const uint2 v = *reinterpret_cast<const uint2*>(p + 8 * i);
      w[2 * i] = v.x; w[2 * i + 1] = v.y;
    }
  } else {
#pragma unroll
    for (int i = 0; i < B; ++i) w[i] = reinterpret_cast<const uint32_t*>(p)[i];
  }
}

__device__ __forceinline__ uint32_t u4_comp(const uint4& v, int c) {
  return c == 0 ? v.x : c == 1 ? v.y : c == 2 ? v.z : v.w;
}

// Activation fragments (b0, b1) of k-step j for the pair order of pair_nib:
// xv holds the thread's 32 consecutive activations, 8 per uint4.
template <int B>
__device__ __forceinline__ void xpair_nib(const uint4 (&xv)[4], int j, uint32_t& b0, uint32_t& b1) {
  uint32_t lo, hi;
  if constexpr (B == 4) {
    lo = u4_comp(xv[j >> 1], (j & 1));
    hi = u4_comp(xv[j >> 1], (j & 1) + 2);
  } else {
    lo = u4_comp(xv[2 * (j >> 2)], j & 3);
    hi = u4_comp(xv[2 * (j >> 2) + 1], j & 3);
  }
  b0 = __byte_perm(lo, hi, 0x5410);
  b1 = __byte_perm(lo, hi, 0x7632);
}

// Pair p of a unit with its two codes as bf16 values code * 2^(c - 133): a
// bf16 bit pattern whose high byte is zero is the integer in its low byte
// times 2^-133 (the subnormals join the smallest binade without a gap), so
// codes masked to bits [c, c + b) of the low byte of each 16-bit half need no
// offset, no conversion and no zero point.  b = 4 and b = 2 take the pair
// order of pair_nib (two codes 16 bits apart in one word; the upper byte's
// codes after one shift by 8 per word), so c = pair_class<B>(p) varies with
// p; b = 8 places bytes 2h, 2h + 1 of a word with one byte permute; the other
// widths take consecutive codes at c = 0.
template <int B>
__host__ __device__ constexpr int pair_class(int p) {
  return B == 4 ? 4 * (p & 1) : B == 2 ? 2 * (p & 3) : 0;
}
template <int B>
__device__ __forceinline__ uint32_t pair_sub(const uint32_t (&w)[B], int p) {
  if constexpr (B == 4) {
    const uint32_t v = (p & 2) ? (w[p >> 2] >> 8) : w[p >> 2];
    return v & (0x000F000Fu << pair_class<4>(p));
  } else if constexpr (B == 2) {
    const uint32_t v = (p & 4) ? (w[p >> 3] >> 8) : w[p >> 3];
    return v & (0x00030003u << pair_class<2>(p));
  } else if constexpr (B == 8) {
    const int h = p & 1;
    return __byte_perm(w[p >> 1], 0u, 0x4040 | (2 * h) | ((2 * h + 1) << 8));
  } else if constexpr (B == 3 || B == 5) {
    const int bit = 2 * B * p, wi = bit >> 5, sh = bit & 31;
    const uint32_t x = sh + 2 * B <= 32 ? (w[wi] >> sh) : __funnelshift_r(w[wi], w[wi + 1], sh);
    const uint32_t t = x & ((1u << (2 * B)) - 1u);
    constexpr uint32_t mask = ((1u << B) - 1u) * 0x00010001u;
    return (t * (1u + (1u << (16 - B)))) & mask;
  } else {
    return dq::code_at<B>(w, 2 * p) | (dq::code_at<B>(w, 2 * p + 1) << 16);
  }
}

// bf16x2 (2^e, 2^e), e in [-126, 127].
__device__ __forceinline__ uint32_t bf16x2_pow2(int e) { return static_cast<uint32_t>(e + 127) * 0x00800080u; }

__device__ __forceinline__ uint32_t bf16x2_mul(uint32_t a, uint32_t b) {
  uint32_t r;
  asm("mul.rn.bf16x2 %0, %1, %2;" : "=r"(r) : "r"(a), "r"(b));
  return r;
}
// max(|a|, |b|) per half; the sign bit of the result is sign(a) ^ sign(b).
__device__ __forceinline__ uint32_t bf16x2_maxabs(uint32_t a, uint32_t b) {
  uint32_t r;
  asm("max.xorsign.abs.bf16x2 %0, %1, %2;" : "=r"(r) : "r"(a), "r"(b));
  return r;
}

__device__ __forceinline__ uint32_t ld_ro_u16(const void* p) {
  unsigned short r;
  asm volatile("ld.global.nc.u16 %0, [%1];" : "=h"(r) : "l"(p));
  return r;
}
__device__ __forceinline__ uint32_t ld_ro_u8(const void* p) {
  unsigned short r;
  asm volatile("ld.global.nc.u8 %0, [%1];" : "=h"(r) : "l"(p));
  return r & 0xFFu;
}

template <int B, int RT, int GB>
constexpr int gemv_stage_bytes() {  // one warp's stage
  return GB * RT * 2 * 8 * 16 * B;
}

template <int B, int RT, int S>
constexpr int gemv_depth() {  // stages per warp: about 12 KiB of ring per warp, 3..8
  constexpr int d = 12 * 1024 / gemv_stage_bytes<B, RT, 2>();
  return d < 3 ? 3 : d > 8 ? 8 : d;
}

template <int B, int RT, int S>
constexpr bool gemv_fits() {  // the CTA's rings within 192 KiB
  return S * gemv_depth<B, RT, S>() * gemv_stage_bytes<B, RT, 2>() <= 192 * 1024;
}


// One layer of a GEMV launch (all device pointers; gmax = the most groups a
// warp takes, ceil(G / S)).
struct GemvLayer {
  const uint16_t* X;
  const uint8_t* packed;
  const uint16_t* scales;
  const uint8_t* zeros;
  void* Y;
  int N, K, gmax, bits;
};

// Row tile `tile` of one layer, computed by the whole CTA.
template <int B, int NT, int RT, int S, int GB, int D>
__device__ __forceinline__ void gemv_tile(const GemvLayer& L, int M, int y_f32, int tile,
                                          uint8_t* smem) {
  const uint16_t* __restrict__ X = L.X;
  const uint8_t* __restrict__ packed = L.packed;
  const uint16_t* __restrict__ scales = L.scales;
  const uint8_t* __restrict__ zeros = L.zeros;
  void* __restrict__ Y = L.Y;
  const int N = L.N, K = L.K, gmax = L.gmax;
  constexpr int kTile = 16 * RT;
  constexpr int kRowG = 16 * B;  // bytes of one row's group
  constexpr int kStage = gemv_stage_bytes<B, RT, GB>();
  constexpr bool kNib = B == 2 || B == 4;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int t = lane & 3, q = lane >> 2;
  const int G = K / kGroup;
  const int64_t row_bytes = static_cast<int64_t>(G) * kRowG;
  const int tile0 = tile * kTile;
  const int g0 = static_cast<int>(static_cast<int64_t>(G) * warp / S);
  const int g1 = static_cast<int>(static_cast<int64_t>(G) * (warp + 1) / S);
  const int ng = g1 - g0;
  uint8_t* ring = smem + warp * (D * kStage);
  uint32_t* szs = reinterpret_cast<uint32_t*>(smem + S * D * kStage) + warp * (kTile * gmax);

  // Rows of this thread: 16 rt + q + 8 h of the tile (clamped for loads).
  // Stage layout: [group i][rt][h][q][16b bytes]; the quad (same q) copies
  // its row's group as b 16-byte chunks, chunk c by lane t = c % 4.
  const uint8_t* wrow[RT][2];
#pragma unroll
  for (int rt = 0; rt < RT; ++rt)
#pragma unroll
    for (int h = 0; h < 2; ++h)
      wrow[rt][h] = packed + min(tile0 + 16 * rt + q + 8 * h, N - 1) * row_bytes;
  auto issue = [&](int stage, int gb) {
    uint8_t* st = ring + stage * kStage + q * kRowG;
#pragma unroll
    for (int i = 0; i < GB; ++i)
      if (gb + i < g1) {
#pragma unroll
        for (int rt = 0; rt < RT; ++rt)
#pragma unroll
          for (int h = 0; h < 2; ++h)
#pragma unroll
            for (int c = t; c < B; c += 4)
              cp_async_16(st + ((i * RT + rt) * 2 + h) * 8 * kRowG + 16 * c,
                          wrow[rt][h] + (gb + i) * kRowG + 16 * c, 16u);
      }
  };

  // The first stage's weights go to L2 while the previous kernel finishes;
  // nothing is read into the SM before it has completed.
  // So do this warp's scales and zeros: lane r < 16 RT takes row r.
  if (ng > 0) {
#pragma unroll
    for (int rt = 0; rt < RT; ++rt)
#pragma unroll
      for (int h = 0; h < 2; ++h) asm volatile("prefetch.global.L2 [%0];" ::"l"(wrow[rt][h] + g0 * kRowG));
    if (lane < kTile) {
      const int64_t o = static_cast<int64_t>(min(tile0 + lane, N - 1)) * G + g0;
      asm volatile("prefetch.global.L2 [%0];" ::"l"(scales + o));
      asm volatile("prefetch.global.L2 [%0];" ::"l"(zeros + o));
    }
  }
  grid_dependency_wait();
  const int nb = (ng + GB - 1) / GB;
#pragma unroll
  for (int d = 0; d < D - 1; ++d) {
    if (d < nb) issue(d, g0 + d * GB);
    cp_async_commit();
  }
  // Activation fragments X[n][128 g + 32 t + 4 j .. + 3] (k-step j) of one
  // group; loaded one group ahead, alternating between two register sets.
  auto load_x = [&](int g, uint4 (&xv)[NT][4]) {
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
      const int n = q + 8 * nt;
      const uint16_t* xp = X + static_cast<int64_t>(n) * K + g * kGroup + 32 * t;
#pragma unroll
      for (int v = 0; v < 4; ++v) xv[nt][v] = n < M ? ld_ro_v4(xp + 8 * v) : make_uint4(0u, 0u, 0u, 0u);
    }
  };
  // The first group's activations are in flight with the weights' first
  // stages while the scales and zeros are staged.
  constexpr bool kAhead = NT == 1;
  uint4 xa[NT][4], xb[NT][4];
  if (kAhead && ng > 0) load_x(g0, xa);
  // This warp's scales and zeros, (scale | zero << 16) per (row, group).
  // Each lane issues up to kSzBatch loads of each kind before its first
  // store, so a batch costs one memory latency rather than one per entry.
  constexpr int kSzBatch = 8;
  for (int base = 0; base < kTile * ng; base += 32 * kSzBatch) {
    uint32_t sv[kSzBatch], zv[kSzBatch];
    int at[kSzBatch];
#pragma unroll
    for (int u = 0; u < kSzBatch; ++u) {
      const int idx = base + 32 * u + lane;
      at[u] = -1;
      if (idx < kTile * ng) {
        const int r = idx / ng, gg = idx - r * ng;
        const int64_t o = static_cast<int64_t>(min(tile0 + r, N - 1)) * G + g0 + gg;
        sv[u] = ld_ro_u16(scales + o);
        zv[u] = ld_ro_u8(zeros + o);
        at[u] = r * gmax + gg;
      }
    }
#pragma unroll
    for (int u = 0; u < kSzBatch; ++u)
      if (at[u] >= 0) szs[at[u]] = sv[u] | (zv[u] << 16);
  }
  __syncwarp();

  float acc[RT][NT][4];
#pragma unroll
  for (int rt = 0; rt < RT; ++rt)
#pragma unroll
    for (int nt = 0; nt < NT; ++nt)
#pragma unroll
      for (int e = 0; e < 4; ++e) acc[rt][nt][e] = 0.0f;

  auto group = [&](const uint8_t* st, int i, int gl, const uint4 (&xpre)[NT][4]) {
    // M <= 8: the fragments came one group ahead; M > 8: loaded here (two
    // register sets of 32 would spill next to two row tiles).
    uint4 xj[NT][4];
    if constexpr (NT == 2) load_x(g0 + gl, xj);
    const uint4(*xv)[4] = (NT == 2) ? xj : xpre;
    uint32_t w[RT][2][B];
    uint32_t sz[RT][2];
#pragma unroll
    for (int rt = 0; rt < RT; ++rt)
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        lds_unit<B>(st + ((i * RT + rt) * 2 + h) * 8 * kRowG, w[rt][h]);
        sz[rt][h] = szs[(16 * rt + q + 8 * h) * gmax + gl];
      }
    float d[RT][NT][4], dsum[NT][4];
#pragma unroll
    for (int nt = 0; nt < NT; ++nt)
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        dsum[nt][e] = 0.0f;
#pragma unroll
        for (int rt = 0; rt < RT; ++rt) d[rt][nt][e] = 0.0f;
      }
    // The group's activation exponent: with 2^e <= max |x| < 2^(e + 1),
    // E = 126 - e puts every x 2^E below 2^127 (clamped to [6, 127]: 2^(E - c)
    // stays a normal bf16 for c <= 6, and 2^(133 - E) a normal binary32).
    uint32_t xm = 0u;
#pragma unroll
    for (int nt = 0; nt < NT; ++nt)
#pragma unroll
      for (int v = 0; v < 4; ++v)
        xm = bf16x2_maxabs(bf16x2_maxabs(xm, xv[nt][v].x), bf16x2_maxabs(xv[nt][v].y,
                           bf16x2_maxabs(xv[nt][v].z, xv[nt][v].w)));
    xm &= 0x7FFF7FFFu;
    xm = __reduce_max_sync(0xFFFFFFFFu, max(xm & 0xFFFFu, xm >> 16));
    const int E = min(127, max(6, 126 - (static_cast<int>(xm >> 7) - 127)));
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const int c0 = pair_class<B>(2 * j), c1 = pair_class<B>(2 * j + 1);
      const uint32_t sc0 = bf16x2_pow2(E - c0), sc1 = bf16x2_pow2(E - c1);
      uint32_t b0[NT], b1[NT];
#pragma unroll
      for (int nt = 0; nt < NT; ++nt) {
        if constexpr (kNib) {
          xpair_nib<B>(xv[nt], j, b0[nt], b1[nt]);
        } else {
          b0[nt] = (j & 1) ? xv[nt][j >> 1].z : xv[nt][j >> 1].x;
          b1[nt] = (j & 1) ? xv[nt][j >> 1].w : xv[nt][j >> 1].y;
        }
        b0[nt] = bf16x2_mul(b0[nt], sc0);
        b1[nt] = bf16x2_mul(b1[nt], sc1);
        // Sx = sum_k x_k 2^(E - 133) in the accumulator layout (A = 2^(c - 133)).
        const uint32_t o0 = 0x00010001u << c0, o1 = 0x00010001u << c1;
        mma_bf16_16816(dsum[nt], o0, o0, o1, o1, b0[nt], b1[nt]);
      }
#pragma unroll
      for (int rt = 0; rt < RT; ++rt) {
        const uint32_t a0 = pair_sub<B>(w[rt][0], 2 * j);
        const uint32_t a1 = pair_sub<B>(w[rt][1], 2 * j);
        const uint32_t a2 = pair_sub<B>(w[rt][0], 2 * j + 1);
        const uint32_t a3 = pair_sub<B>(w[rt][1], 2 * j + 1);
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) mma_bf16_16816(d[rt][nt], a0, a1, a2, a3, b0[nt], b1[nt]);
      }
    }
    // y += s 2^(133 - E) (D - z Sx): D = sum_k q x 2^(E - 133).
    const float pw = __uint_as_float(static_cast<uint32_t>(260 - E) << 23);
#pragma unroll
    for (int rt = 0; rt < RT; ++rt) {
      const float s0 = __half2float(__ushort_as_half(static_cast<uint16_t>(sz[rt][0] & 0xFFFFu))) * pw;
      const float s1 = __half2float(__ushort_as_half(static_cast<uint16_t>(sz[rt][1] & 0xFFFFu))) * pw;
      const float zb0 = -static_cast<float>(sz[rt][0] >> 16);
      const float zb1 = -static_cast<float>(sz[rt][1] >> 16);
#pragma unroll
      for (int nt = 0; nt < NT; ++nt) {
        acc[rt][nt][0] = fmaf(s0, fmaf(zb0, dsum[nt][0], d[rt][nt][0]), acc[rt][nt][0]);
        acc[rt][nt][1] = fmaf(s0, fmaf(zb0, dsum[nt][1], d[rt][nt][1]), acc[rt][nt][1]);
        acc[rt][nt][2] = fmaf(s1, fmaf(zb1, dsum[nt][2], d[rt][nt][2]), acc[rt][nt][2]);
        acc[rt][nt][3] = fmaf(s1, fmaf(zb1, dsum[nt][3], d[rt][nt][3]), acc[rt][nt][3]);
      }
    }
  };

  // Two groups per stage (GB = 2): for M <= 8 the first computes from xa
  // while xb is loaded for the second, which loads xa for the next stage's
  // first.
  static_assert(GB == 2, "the activation double buffer alternates within a stage");
  for (int bi = 0; bi < nb; ++bi) {
    const int nx = bi + D - 1;
    if (nx < nb) issue(nx % D, g0 + nx * GB);
    cp_async_commit();
    cp_async_wait<D - 1>();
    __syncwarp();  // the quad's chunks of every row are in
    const uint8_t* st = ring + (bi % D) * kStage + q * kRowG + 4 * B * t;
    const int gl = bi * GB;
    if (kAhead && gl + 1 < ng) load_x(g0 + gl + 1, xb);
    group(st, 0, gl, xa);
    if (gl + 1 < ng) {
      if (kAhead && gl + 2 < ng) load_x(g0 + gl + 2, xa);
      group(st, 1, gl + 1, xb);
    }
    __syncwarp();  // the stage is read before the quad may refill it
  }
  cp_async_wait<0>();
  grid_launch_dependents();

  // Add the S warps' partial tiles in warp order (the rings are free now).
  __syncthreads();
  float* part = reinterpret_cast<float*>(smem);  // [S][kTile][8 NT + 1]
  constexpr int kLd = 8 * NT + 1;
#pragma unroll
  for (int rt = 0; rt < RT; ++rt)
#pragma unroll
    for (int nt = 0; nt < NT; ++nt)
#pragma unroll
      for (int e = 0; e < 4; ++e)
        part[(warp * kTile + 16 * rt + q + 8 * (e >> 1)) * kLd + 8 * nt + 2 * t + (e & 1)] = acc[rt][nt][e];
  __syncthreads();
  for (int idx = threadIdx.x; idx < kTile * M; idx += 32 * S) {
    const int m = idx / kTile, r = idx - m * kTile;
    const int n = tile0 + r;
    if (n < N) {
      float v = part[r * kLd + m];
#pragma unroll
      for (int w = 1; w < S; ++w) v += part[(w * kTile + r) * kLd + m];
      store_y(Y, y_f32, static_cast<int64_t>(m) * N + n, v);
    }
  }
}

template <int B, int NT, int RT, int S, int GB, int D>
__global__ void __launch_bounds__(32 * S)
    gemm_gemv_kernel(const __grid_constant__ GemvLayer L, int M, int y_f32) {
  extern __shared__ __align__(16) uint8_t smem[];
  gemv_tile<B, NT, RT, S, GB, D>(L, M, y_f32, static_cast<int>(blockIdx.x), smem);
}

// Several layers (any mix of b, N, K) in one launch: the CTAs are the
// layers' row tiles in order; each finds its layer and runs that layer's b.
constexpr int kMaxGroup = 8;
struct GemvGroup {
  GemvLayer layer[kMaxGroup];
  int tile_end[kMaxGroup];  // prefix sums of the layers' row tiles
  int count;
};

template <int NT, int RT, int S>
__global__ void __launch_bounds__(32 * S)
    gemm_gemv_group_kernel(const __grid_constant__ GemvGroup grp, int M, int y_f32) {
  extern __shared__ __align__(16) uint8_t smem[];
  const int cta = static_cast<int>(blockIdx.x);
  int i = 0;
  while (i + 1 < grp.count && cta >= grp.tile_end[i]) ++i;
  const int tile = cta - (i ? grp.tile_end[i - 1] : 0);
  const GemvLayer& L = grp.layer[i];
  switch (L.bits) {
    case 2: gemv_tile<2, NT, RT, S, 2, gemv_depth<2, RT, S>()>(L, M, y_f32, tile, smem); break;
    case 3: gemv_tile<3, NT, RT, S, 2, gemv_depth<3, RT, S>()>(L, M, y_f32, tile, smem); break;
    case 4: gemv_tile<4, NT, RT, S, 2, gemv_depth<4, RT, S>()>(L, M, y_f32, tile, smem); break;
    case 5: gemv_tile<5, NT, RT, S, 2, gemv_depth<5, RT, S>()>(L, M, y_f32, tile, smem); break;
    case 6: gemv_tile<6, NT, RT, S, 2, gemv_depth<6, RT, S>()>(L, M, y_f32, tile, smem); break;
    case 7: gemv_tile<7, NT, RT, S, 2, gemv_depth<7, RT, S>()>(L, M, y_f32, tile, smem); break;
    default: gemv_tile<8, NT, RT, S, 2, gemv_depth<8, RT, S>()>(L, M, y_f32, tile, smem); break;
  }
}

// ---------------------------------------------------------------------------
// Host side
// ---------------------------------------------------------------------------

// Groups per chunk for a layer: the preferred chunk when it divides the
// groups of a row, else single groups.
int groups_per_chunk(int64_t K, int bits) {
  const int G = static_cast<int>(K / kGroup);
  int gs = 1;
  switch (bits) {
    case 2: gs = chunk_groups<2>(); break;
    case 3: gs = chunk_groups<3>(); break;
    case 4: gs = chunk_groups<4>(); break;
    default: gs = 1;
  }
  return G % gs == 0 ? gs : 1;
}

// Stream-K geometry for a layer over at most `ctas_max` resident CTAs.
Split make_split(int64_t N, int64_t K, int gs, int ctas_max) {
  Split sp;
  sp.G = static_cast<int>(K / kGroup) / gs;
  const int64_t rbs = (N + kRows - 1) / kRows;
  const int64_t total = rbs * sp.G;
  const int64_t ctas = total < ctas_max ? total : ctas_max;
  sp.per = static_cast<int>((total + ctas - 1) / ctas);
  if (sp.per < kMinChunksPerCta) sp.per = kMinChunksPerCta;
  sp.nctas = static_cast<int>((total + sp.per - 1) / sp.per);
  // A row tile of G groups meets at most ceil((G - 1) / per) + 1 CTA ranges.
  int s = (sp.G - 1 + sp.per - 1) / sp.per + 1;
  sp.s_max = s < sp.nctas ? s : sp.nctas;
  return sp;
}

int resident_ctas() {
  int dev = 0, sms = 148;
  if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  return sms * kCtasPerSm;
}

template <int B, int NT, int GS>
cudaError_t launch_cfg(const uint16_t* X, int M, int N, int K, const uint32_t* packed,
                       const uint16_t* scales, const uint8_t* zeros, void* Y, bool y_f32,
                       void* workspace, uint32_t* flags, cudaStream_t stream) {
  using C = Cfg<B, NT, GS>;
  CUtensorMap tw;
  const CUtensorMapSwizzle swz =
      16 * B * GS == 128 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_NONE;
  if (!encode_tensor_map_2d(&tw, CU_TENSOR_MAP_DATA_TYPE_UINT32, packed,
                            static_cast<uint64_t>(K) * B / 32, static_cast<uint64_t>(N),
                            static_cast<uint64_t>(K) * B / 8, 4 * B * GS, kRows, swz))
    return cudaErrorInvalidValue;
  static SmemAttr smem_attr;  // per template instance
  const cudaError_t ea = smem_attr.ensure(gemm_decode_kernel<B, NT, GS>, C::kSmem);
  if (ea != cudaSuccess) return ea;
  const Split sp = make_split(N, K, GS, resident_ctas());
  int* counters = static_cast<int*>(workspace);
  float* partials = reinterpret_cast<float*>(static_cast<uint8_t*>(workspace) + kCounterBytes);
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(sp.nctas), 1, 1);
  cfg.blockDim = dim3(kThreads, 1, 1);
  cfg.dynamicSmemBytes = C::kSmem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, gemm_decode_kernel<B, NT, GS>, tw, X, M, N, K, scales, zeros, Y,
                            y_f32 ? 1 : 0, sp, counters, partials, flags);
}

template <int B>
cudaError_t launch_b(const uint16_t* X, int M, int N, int K, const uint32_t* packed,
                     const uint16_t* scales, const uint8_t* zeros, void* Y, bool y_f32,
                     void* workspace, uint32_t* flags, cudaStream_t stream) {
  constexpr int kGS = chunk_groups<B>();
  if (groups_per_chunk(K, B) == kGS) {
    if (M <= 8)
      return launch_cfg<B, 1, kGS>(X, M, N, K, packed, scales, zeros, Y, y_f32, workspace, flags, stream);
    return launch_cfg<B, 2, kGS>(X, M, N, K, packed, scales, zeros, Y, y_f32, workspace, flags, stream);
  }
  if constexpr (kGS != 1) {
    if (M <= 8)
      return launch_cfg<B, 1, 1>(X, M, N, K, packed, scales, zeros, Y, y_f32, workspace, flags, stream);
    return launch_cfg<B, 2, 1>(X, M, N, K, packed, scales, zeros, Y, y_f32, workspace, flags, stream);
  }
  return cudaErrorInvalidValue;
}

}  // namespace

size_t gemm_decode_workspace_bytes(int64_t N, int64_t K, int bits) {
  const Split sp = make_split(N, K, groups_per_chunk(K, bits), resident_ctas());
  const int64_t rbs = (N + kRows - 1) / kRows;
  if (sp.s_max <= 1) return 0;
  return kCounterBytes + static_cast<size_t>(rbs) * sp.s_max * kMaxM * kRows * sizeof(float);
}

int64_t gemm_decode_max_n() { return kMaxRowTiles * kRows; }

cudaError_t launch_gemm_decode(const uint16_t* X, int64_t M, int64_t N, int64_t K, int bits,
                               const uint32_t* packed, const uint16_t* scales,
                               const uint8_t* zeros, void* Y, bool y_f32, void* workspace,
                               uint32_t* flags, cudaStream_t stream) {
  const int m = static_cast<int>(M), n = static_cast<int>(N), k = static_cast<int>(K);
  switch (bits) {
    case 2: return launch_b<2>(X, m, n, k, packed, scales, zeros, Y, y_f32, workspace, flags, stream);
    case 3: return launch_b<3>(X, m, n, k, packed, scales, zeros, Y, y_f32, workspace, flags, stream);
    case 4: return launch_b<4>(X, m, n, k, packed, scales, zeros, Y, y_f32, workspace, flags, stream);
    case 5: return launch_b<5>(X, m, n, k, packed, scales, zeros, Y, y_f32, workspace, flags, stream);
    case 6: return launch_b<6>(X, m, n, k, packed, scales, zeros, Y, y_f32, workspace, flags, stream);
    case 7: return launch_b<7>(X, m, n, k, packed, scales, zeros, Y, y_f32, workspace, flags, stream);
    case 8: return launch_b<8>(X, m, n, k, packed, scales, zeros, Y, y_f32, workspace, flags, stream);
    default: return cudaErrorInvalidValue;
  }
}

namespace {

template <int B, int NT, int RT, int S>
cudaError_t launch_gemv_cfg(const uint16_t* X, int M, int N, int K, const uint32_t* packed,
                            const uint16_t* scales, const uint8_t* zeros, void* Y, bool y_f32,
                            cudaStream_t stream) {
  constexpr int kGB = 2;
  constexpr int kD = gemv_depth<B, RT, S>();
  auto kern = gemm_gemv_kernel<B, NT, RT, S, kGB, kD>;
  const int G = K / kGroup;
  const int gmax = (G + S - 1) / S;
  const size_t rings = static_cast<size_t>(S) * kD * gemv_stage_bytes<B, RT, kGB>();
  const size_t szb = static_cast<size_t>(S) * 16 * RT * gmax * 4;
  const size_t partb = static_cast<size_t>(S) * 16 * RT * (8 * NT + 1) * 4;
  const size_t smem = (rings + szb) > partb ? rings + szb : partb;
  if (smem > 227 * 1024) return cudaErrorInvalidValue;
  static SmemAttr smem_attr;  // per template instance
  const cudaError_t ea = smem_attr.ensure(kern, static_cast<int>(smem));
  if (ea != cudaSuccess) return ea;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>((N + 16 * RT - 1) / (16 * RT)), 1, 1);
  cfg.blockDim = dim3(32 * S, 1, 1);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  const GemvLayer L{X, reinterpret_cast<const uint8_t*>(packed), scales, zeros, Y, N, K, gmax, B};
  return cudaLaunchKernelEx(&cfg, kern, L, M, y_f32 ? 1 : 0);
}

// Tile shape of a GEMV launch over `rows` weight rows with G groups each
// (measured on this B200 over the Qwen3-8B block's layers and 8192 x 8192,
// graph-timed, M = 1, 4, 16):
//  * RT: the CTAs of a launch run concurrently, so an SM's time follows the
//    rows it gets, ceil(tiles / SMs) * 16 RT.  Two m16 tiles per warp share
//    the per-group activation work, so RT = 2 unless one tile per warp puts
//    at least a fifth fewer rows on the busiest SM (or rt2 is not allowed).
//  * S (warps splitting K): 16 when the tiles leave SMs idle and K is long,
//    4 once there are two tiles per SM or more, else 8.
struct GemvShape {
  int rt, s;
};
GemvShape gemv_shape(int64_t rows, int G, bool rt2, int sms) {
  const int64_t t1 = (rows + 15) / 16, t2 = (rows + 31) / 32;
  const int64_t w1 = (t1 + sms - 1) / sms, w2 = 2 * ((t2 + sms - 1) / sms);
  const int rt = (!rt2 || 5 * w1 < 4 * w2) ? 1 : 2;
  const int64_t tiles = rt == 1 ? t1 : t2;
  int s = 8;
  if (tiles < sms && G >= 32) s = 16;
  else if (tiles >= 2 * sms || G < 16) s = 4;
  return {rt, s};
}

int device_sms() {
  int dev = 0, sms = 148;
  if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  return sms;
}

template <int B, int NT, int RT>
cudaError_t launch_gemv_rt(int s, const uint16_t* X, int M, int N, int K, const uint32_t* packed,
                           const uint16_t* scales, const uint8_t* zeros, void* Y, bool y_f32,
                           cudaStream_t stream) {
  // A shape whose rings do not fit falls back to fewer warps.
  if constexpr (gemv_fits<B, RT, 16>()) {
    if (s == 16) return launch_gemv_cfg<B, NT, RT, 16>(X, M, N, K, packed, scales, zeros, Y, y_f32, stream);
  }
  if constexpr (gemv_fits<B, RT, 8>()) {
    if (s >= 8) return launch_gemv_cfg<B, NT, RT, 8>(X, M, N, K, packed, scales, zeros, Y, y_f32, stream);
  }
  return launch_gemv_cfg<B, NT, RT, 4>(X, M, N, K, packed, scales, zeros, Y, y_f32, stream);
}

template <int B>
cudaError_t launch_gemv_b(const uint16_t* X, int M, int N, int K, const uint32_t* packed,
                          const uint16_t* scales, const uint8_t* zeros, void* Y, bool y_f32,
                          cudaStream_t stream) {
  // At M <= 8, b = 7 and 8, the doubled unit registers of RT = 2 cost more
  // than the shared activation work saves.
  const GemvShape sh = gemv_shape(N, K / kGroup, M > 8 || B <= 6, device_sms());
  if (M <= 8) {
    if (sh.rt == 2) return launch_gemv_rt<B, 1, 2>(sh.s, X, M, N, K, packed, scales, zeros, Y, y_f32, stream);
    return launch_gemv_rt<B, 1, 1>(sh.s, X, M, N, K, packed, scales, zeros, Y, y_f32, stream);
  }
  if (sh.rt == 2) return launch_gemv_rt<B, 2, 2>(sh.s, X, M, N, K, packed, scales, zeros, Y, y_f32, stream);
  return launch_gemv_rt<B, 2, 1>(sh.s, X, M, N, K, packed, scales, zeros, Y, y_f32, stream);
}

}  // namespace

cudaError_t launch_gemm_gemv(const uint16_t* X, int64_t M, int64_t N, int64_t K, int bits,
                             const uint32_t* packed, const uint16_t* scales, const uint8_t* zeros,
                             void* Y, bool y_f32, uint32_t* flags, cudaStream_t stream) {
  (void)flags;  // the GEMV kernel has no bounded waits (cp.async groups only)
  const int m = static_cast<int>(M), n = static_cast<int>(N), k = static_cast<int>(K);
  switch (bits) {
    case 2: return launch_gemv_b<2>(X, m, n, k, packed, scales, zeros, Y, y_f32, stream);
    case 3: return launch_gemv_b<3>(X, m, n, k, packed, scales, zeros, Y, y_f32, stream);
    case 4: return launch_gemv_b<4>(X, m, n, k, packed, scales, zeros, Y, y_f32, stream);
    case 5: return launch_gemv_b<5>(X, m, n, k, packed, scales, zeros, Y, y_f32, stream);
    case 6: return launch_gemv_b<6>(X, m, n, k, packed, scales, zeros, Y, y_f32, stream);
    case 7: return launch_gemv_b<7>(X, m, n, k, packed, scales, zeros, Y, y_f32, stream);
    case 8: return launch_gemv_b<8>(X, m, n, k, packed, scales, zeros, Y, y_f32, stream);
    default: return cudaErrorInvalidValue;
  }
}

namespace {

// Shared memory a layer of b bits needs in a CTA of the (NT, RT, S) shape,
// and whether two ring stages per warp fit at all.
template <int NT, int RT, int S>
size_t gemv_group_smem(int b, int gmax, bool* fits) {
  size_t stage = 0;
  int d = 0;
  bool f = false;
  switch (b) {
#define SLQ_GEMV_CASE(BB)                                    \
  case BB:                                                   \
    stage = gemv_stage_bytes<BB, RT, 2>();                   \
    d = gemv_depth<BB, RT, S>();                             \
    f = gemv_fits<BB, RT, S>();                              \
    break;
    SLQ_GEMV_CASE(2) SLQ_GEMV_CASE(3) SLQ_GEMV_CASE(4) SLQ_GEMV_CASE(5)
    SLQ_GEMV_CASE(6) SLQ_GEMV_CASE(7) SLQ_GEMV_CASE(8)
#undef SLQ_GEMV_CASE
    default: break;
  }
  *fits = f;
  const size_t rings = static_cast<size_t>(S) * d * stage;
  const size_t szb = static_cast<size_t>(S) * 16 * RT * gmax * 4;
  const size_t partb = static_cast<size_t>(S) * 16 * RT * (8 * NT + 1) * 4;
  return (rings + szb) > partb ? rings + szb : partb;
}

template <int NT, int RT, int S>
cudaError_t launch_group_cfg(const GemvLayer* layers, int count, int M, bool y_f32,
                             cudaStream_t stream, bool* fits) {
  GemvGroup grp = {};
  grp.count = count;
  size_t smem = 0;
  int tiles = 0;
  *fits = true;
  for (int i = 0; i < count; ++i) {
    grp.layer[i] = layers[i];
    const int G = layers[i].K / kGroup;
    grp.layer[i].gmax = (G + S - 1) / S;
    bool f = false;
    const size_t need = gemv_group_smem<NT, RT, S>(layers[i].bits, grp.layer[i].gmax, &f);
    if (!f || need > 227 * 1024) {
      *fits = false;
      return cudaSuccess;
    }
    smem = need > smem ? need : smem;
    tiles += (layers[i].N + 16 * RT - 1) / (16 * RT);
    grp.tile_end[i] = tiles;
  }
  auto kern = gemm_gemv_group_kernel<NT, RT, S>;
  static SmemAttr smem_attr;  // per template instance
  const cudaError_t ea = smem_attr.ensure(kern, static_cast<int>(smem));
  if (ea != cudaSuccess) return ea;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(tiles), 1, 1);
  cfg.blockDim = dim3(32 * S, 1, 1);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, grp, M, y_f32 ? 1 : 0);
}

// The same shape rules as a single layer, applied to the group's totals.
template <int NT, int RT>
cudaError_t launch_group_rt(int s, const GemvLayer* layers, int count, int M, bool y_f32,
                            cudaStream_t stream) {
  bool fits = false;
  cudaError_t e = cudaSuccess;
  if (s == 16) {
    e = launch_group_cfg<NT, RT, 16>(layers, count, M, y_f32, stream, &fits);
    if (fits || e != cudaSuccess) return e;
  }
  if (s >= 8) {
    e = launch_group_cfg<NT, RT, 8>(layers, count, M, y_f32, stream, &fits);
    if (fits || e != cudaSuccess) return e;
  }
  e = launch_group_cfg<NT, RT, 4>(layers, count, M, y_f32, stream, &fits);
  if (e != cudaSuccess) return e;
  return fits ? cudaSuccess : cudaErrorInvalidValue;
}

}  // namespace

int gemm_gemv_group_max() { return kMaxGroup; }

cudaError_t launch_gemm_gemv_group(const GemvCall* calls, int count, int64_t M, bool y_f32,
                                   uint32_t* flags, cudaStream_t stream) {
  (void)flags;
  if (count < 1 || count > kMaxGroup) return cudaErrorInvalidValue;
  GemvLayer layers[kMaxGroup];
  int64_t rows = 0;
  int bmax = 0;
  for (int i = 0; i < count; ++i) {
    const GemvCall& c = calls[i];
    layers[i] = GemvLayer{c.X, reinterpret_cast<const uint8_t*>(c.packed), c.scales, c.zeros, c.Y,
                          static_cast<int>(c.N), static_cast<int>(c.K), 0, c.bits};
    rows += c.N;
    bmax = c.bits > bmax ? c.bits : bmax;
  }
  const int m = static_cast<int>(M);
  // The single-layer shape rule over all the layers' rows (each layer's
  // tiles are whole; the shortest K decides the warp split).
  int gmin = 1 << 30;
  for (int i = 0; i < count; ++i) gmin = layers[i].K / kGroup < gmin ? layers[i].K / kGroup : gmin;
  const GemvShape sh = gemv_shape(rows, gmin, m > 8 || bmax <= 6, device_sms());
  if (m <= 8) {
    if (sh.rt == 2) return launch_group_rt<1, 2>(sh.s, layers, count, m, y_f32, stream);
    return launch_group_rt<1, 1>(sh.s, layers, count, m, y_f32, stream);
  }
  if (sh.rt == 2) return launch_group_rt<2, 2>(sh.s, layers, count, m, y_f32, stream);
  return launch_group_rt<2, 1>(sh.s, layers, count, m, y_f32, stream);
}

// ---------------------------------------------------------------------------
// Allocation-free variant: the split-K workspace lives in a fixed device
// array of this file instead of caller memory.
// ---------------------------------------------------------------------------
namespace {

constexpr size_t kStaticScratchBytes = size_t{8} << 20;  // 8 MiB per device

// Zero-initialized when the library is loaded on a device; every device that
// loads the library keeps it until the process exits.
static __device__ __align__(256) uint8_t g_static_scratch[kStaticScratchBytes];

constexpr int kMaxDevices = 64;
std::mutex g_static_mu;
void* g_static_ptr[kMaxDevices] = {};
void* g_static_ctx[kMaxDevices] = {};

// The current context (the device's primary context under the runtime), from
// the driver entry point looked up through the runtime.
void* current_context() {
  using GetCtx = int (*)(void**);
  static GetCtx fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<GetCtx>(p);
  });
  void* ctx = nullptr;
  if (fn) fn(&ctx);
  return ctx;
}

// The device address of g_static_scratch on the current device.  In host
// code the array's name is only a host-side stand-in, so the address is
// looked up with that device current and cached per device, together with
// the context it belongs to: after a cudaDeviceReset the device gets a new
// primary context (and a new copy of the array), and the address is looked
// up again.
cudaError_t static_scratch(void** out) {
  int dev = -1;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  void* ctx = current_context();
  std::lock_guard<std::mutex> lock(g_static_mu);
  if (!g_static_ptr[dev] || g_static_ctx[dev] != ctx) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_static_scratch);
    if (e != cudaSuccess) return e;
    g_static_ptr[dev] = p;
    g_static_ctx[dev] = ctx;
  }
  *out = g_static_ptr[dev];
  return cudaSuccess;
}

}  // namespace

size_t gemm_decode_static_scratch_bytes() { return kStaticScratchBytes; }

cudaError_t launch_gemm_decode_static(const uint16_t* X, int64_t M, int64_t N, int64_t K, int bits,
                                      const uint32_t* packed, const uint16_t* scales,
                                      const uint8_t* zeros, void* Y, bool y_f32, uint32_t* flags,
                                      cudaStream_t stream) {
  const size_t need = gemm_decode_workspace_bytes(N, K, bits);
  if (need > kStaticScratchBytes) return cudaErrorInvalidValue;
  void* ws = nullptr;
  cudaError_t e = static_scratch(&ws);
  if (e != cudaSuccess) return e;
  if (need > 0) {
    // The tile counters must start at zero; the partial sums need not.
    const int64_t rbs = (N + kRows - 1) / kRows;
    e = cudaMemsetAsync(ws, 0, static_cast<size_t>(rbs) * sizeof(int), stream);
    if (e != cudaSuccess) return e;
  }
  return launch_gemm_decode(X, M, N, K, bits, packed, scales, zeros, Y, y_f32, ws, flags, stream);
}

}  // namespace slq
