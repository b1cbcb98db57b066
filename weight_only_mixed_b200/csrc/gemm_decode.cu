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

using dq::unit_pairs;

constexpr int kRows = 128;       // weight rows per tile
constexpr int kMaxM = 16;        // activation rows (two n8 mma tiles)
constexpr int kConsumers = 8;    // consumer warps, 16 rows each
constexpr int kWarpW = 0, kWarpX = 1, kWarpC0 = 2;
constexpr int kThreads = (kWarpC0 + kConsumers) * 32;
constexpr int kCtasPerSm = 2;
constexpr int kSX = 6;                 // activation fragment stages (one group each)
constexpr int kXFrag = 8 * 32 * 8;     // one n8 tile of a group: 8 k-steps x 32 lanes x 8 B
constexpr int kLook = 4;               // scale / zero loads in flight (groups)
constexpr int kMaxPending = 4;         // shared tiles per CTA (at most 2 occur)
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
  static constexpr int kFixed = 1024 /* alignment slack */ + kSX * kXStage +
                                1024 /* barriers, pending list */;
  static constexpr int kBudget = 227 * 1024 / kCtasPerSm - 1024 /* static + reserved */;
  static constexpr int kSPRaw = (kBudget - kFixed) / kStage;
  static constexpr int kSP = kSPRaw > 16 ? 16 : kSPRaw;
  static constexpr int kSmem = kFixed + kSP * kStage;
  static_assert(kSPRaw >= 3, "shared memory budget");
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
  uint64_t* bars = reinterpret_cast<uint64_t*>(xbuf + kSX * C::kXStage);
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
  __syncthreads();

  if (warp == kWarpW) {
    // ---------------- packed-W producer (TMA) ----------------
    if (lane == 0) {
      prefetch_tmap(&tmap_w);
      int rb = rb0, gc = gk0 / GS;
      int issued = 0;
      for (int ci = 0; ci < nc; ++ci) {
        const int s = ci % kSP;
        if (!wait_or_abort(&sh.p_empty[s], ((ci / kSP) & 1) ^ 1, sh, flags)) break;
        mbar_arrive_expect_tx(&sh.p_full[s], kStage);
        tma_load_2d(pbuf + s * kStage, &tmap_w, &sh.p_full[s], gc * 4 * B * GS, rb * kRows);
        ++issued;
        if (++gc == Gc) {
          gc = 0;
          ++rb;
        }
      }
      for (int i = issued - kSP; i < issued; ++i)  // every issued copy lands before exit
        if (i >= 0) mbar_wait_bounded(&sh.p_full[i % kSP], (i / kSP) & 1);
    }
    __syncwarp();
  } else if (warp == kWarpX) {
    // ---------------- activation fragments (cp.async, rows >= M zero) ----------------
    // Slot (nt, j, lane) holds X[m][k0 + 32t + 4j .. + 3], m = 8nt + lane / 4,
    // t = lane % 4: the B fragment of k-step j for activation rows 8nt..8nt+7.
    const int t = lane & 3;
    int gk = gk0;
    for (int g = 0; g < ng; ++g, gk = (gk + 1 == G) ? 0 : gk + 1) {
      const int s = g % kSX;
      if (!__all_sync(0xffffffffu,
                      wait_or_abort(&sh.x_empty[s], ((g / kSX) & 1) ^ 1, sh, flags)))
        break;
      uint8_t* dst = xbuf + s * C::kXStage + lane * 8;
#pragma unroll
      for (int nt = 0; nt < NT; ++nt) {
        const int m = 8 * nt + (lane >> 2);
        const bool in = m < M;
        const uint16_t* src = X + static_cast<int64_t>(in ? m : 0) * K + gk * kGroup + 32 * t;
#pragma unroll
        for (int j = 0; j < 8; ++j) cp_async_8(dst + (nt * 8 + j) * 256, src + 4 * j, in ? 8u : 0u);
      }
      cp_async_mbar_arrive(&sh.x_full[s]);
    }
    cp_async_wait<0>();  // nothing in flight past this point
    __syncwarp();
  } else {
    // ---------------- consumers: rows 16c + lane / 4 and + 8 of the tile ----------------
    const int c = warp - kWarpC0;
    const int t = lane & 3;
    const int r0 = 16 * c + (lane >> 2), r1 = r0 + 8;
    const bool leader = threadIdx.x == kWarpC0 * 32;
    float acc[NT][4];
#pragma unroll
    for (int nt = 0; nt < NT; ++nt)
#pragma unroll
      for (int e = 0; e < 4; ++e) acc[nt][e] = 0.0f;

    // Scales and zeros of both rows, kLook groups ahead.  Rows past N and
    // groups past the range read clamped (valid, unused) addresses, so the
    // loads are unconditional and nothing waits on them until they are used.
    int frb = rb0, fgk = gk0;
    auto sz_load = [&](uint32_t& s0, uint32_t& s1, uint32_t& z0, uint32_t& z1) {
      const int rbc = min(frb, rbs - 1) * kRows;
      const int64_t i0 = static_cast<int64_t>(min(rbc + r0, N - 1)) * G + fgk;
      const int64_t i1 = static_cast<int64_t>(min(rbc + r1, N - 1)) * G + fgk;
      s0 = scales[i0];
      s1 = scales[i1];
      z0 = zeros[i0];
      z1 = zeros[i1];
      if (++fgk == G) {
        fgk = 0;
        ++frb;
      }
    };
    uint32_t rs0[kLook], rs1[kLook], rz0[kLook], rz1[kLook];
#pragma unroll
    for (int j = 0; j < kLook; ++j) sz_load(rs0[j], rs1[j], rz0[j], rz1[j]);

    bool ok = true;
    int nseg = 0;  // shared row tiles met so far (the same count in every consumer warp)
    int rb = rb0, gk = gk0;
    // The ring index j must stay a compile-time constant (the ring lives in
    // registers), so the unrolled body is predicated instead of exited.
    for (int g0 = 0; g0 < ng && ok; g0 += kLook) {
#pragma unroll
      for (int j = 0; j < kLook; ++j) {
        const int g = g0 + j;
        const int ci = g / GS, gs = g % GS;  // chunk, group within the chunk
        const int sp_ = ci % kSP, sx = g % kSX;
        if (g < ng && ok)
          ok = __all_sync(0xffffffffu,
                          (gs != 0 || wait_or_abort(&sh.p_full[sp_], (ci / kSP) & 1, sh, flags)) &&
                              wait_or_abort(&sh.x_full[sx], (g / kSX) & 1, sh, flags));
        if (g < ng && ok) {
          // ---- codes of both rows -> exact bf16 (q - z) pairs ----
          const uint8_t* pst = pbuf + sp_ * kStage;
          uint32_t w0[B], w1[B];
          load_codes<B, GS>(pst, r0, gs, t, w0);
          load_codes<B, GS>(pst, r1, gs, t, w1);
          if (gs == GS - 1) {
            // Release the stage only after every code word of this warp has
            // arrived in registers (the TMA refill may overwrite it at once),
            // ordered before the async proxy's writes.
            uint32_t dep = 0;
#pragma unroll
            for (int i = 0; i < B; ++i) dep ^= w0[i] ^ w1[i];
            fence_proxy_async_smem();
            __syncwarp();
            dep = __shfl_sync(0xffffffffu, dep, 0) | __any_sync(0xffffffffu, dep != 0);
            if (lane == 0) mbar_arrive_after(&sh.p_empty[sp_], dep);
          }
          const float s0 = __half2float(__ushort_as_half(static_cast<uint16_t>(rs0[j])));
          const float s1 = __half2float(__ushort_as_half(static_cast<uint16_t>(rs1[j])));
          const uint32_t z0 = rz0[j], z1 = rz1[j];
          sz_load(rs0[j], rs1[j], rz0[j], rz1[j]);
          uint32_t p0[16], p1[16];
          unit_pairs<B>(w0, z0, p0);
          unit_pairs<B>(w1, z1, p1);

          // ---- 8 k-steps; even and odd steps in separate accumulators ----
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
#pragma unroll
            for (int nt = 0; nt < NT; ++nt) {
              const uint2 bfr = lds_v2(xs + (nt * 8 + ks) * 256);
              mma_bf16_16816(d[ks & 1][nt], p0[2 * ks], p1[2 * ks], p0[2 * ks + 1], p1[2 * ks + 1],
                             bfr.x, bfr.y);
            }
          }
          {
            // Release the activation stage once every mma that read it has
            // consumed its fragments (a dependency on all the accumulators).
            uint32_t dep = 0;
#pragma unroll
            for (int nt = 0; nt < NT; ++nt)
              dep ^= __float_as_uint(d[0][nt][0]) ^ __float_as_uint(d[1][nt][0]);
            __syncwarp();
            dep = __any_sync(0xffffffffu, dep != 0);
            if (lane == 0) mbar_arrive_after(&sh.x_empty[sx], dep);
          }
#pragma unroll
          for (int nt = 0; nt < NT; ++nt) {
            acc[nt][0] = fmaf(s0, d[0][nt][0] + d[1][nt][0], acc[nt][0]);
            acc[nt][1] = fmaf(s0, d[0][nt][1] + d[1][nt][1], acc[nt][1]);
            acc[nt][2] = fmaf(s1, d[0][nt][2] + d[1][nt][2], acc[nt][2]);
            acc[nt][3] = fmaf(s1, d[0][nt][3] + d[1][nt][3], acc[nt][3]);
          }

          // ---- end of this CTA's part of a row tile: write it out ----
          if (gk == G - 1 || g == ng - 1) {
            const int c0 = first_cta(sp, rb);  // in chunks: sp.G = Gc
            const int ncover = last_cta(sp, rb) - c0 + 1;
            if (ncover == 1) {
#pragma unroll
              for (int nt = 0; nt < NT; ++nt)
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                  const int m = 8 * nt + 2 * t + (e & 1);
                  const int n = rb * kRows + (e < 2 ? r0 : r1);
                  if (m < M && n < N) store_y(Y, y_f32, static_cast<int64_t>(m) * N + n, acc[nt][e]);
                }
            } else {
              const int slot = static_cast<int>(blockIdx.x) - c0;
              float* part = partials + (static_cast<int64_t>(rb) * sp.s_max + slot) * (kMaxM * kRows);
#pragma unroll
              for (int nt = 0; nt < NT; ++nt)
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                  const int m = 8 * nt + 2 * t + (e & 1);
                  if (m < M) part[m * kRows + (e < 2 ? r0 : r1)] = acc[nt][e];
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
            for (int nt = 0; nt < NT; ++nt)
#pragma unroll
              for (int e = 0; e < 4; ++e) acc[nt][e] = 0.0f;
          }
          if (++gk == G) {
            gk = 0;
            ++rb;
          }
        }
      }
    }

    // Shared row tiles this CTA completed last: add the slots in slot order.
    if (leader) mbar_arrive(sh.end_bar);
    ok = __all_sync(0xffffffffu, ok && wait_or_abort(sh.end_bar, 0, sh, flags));
    if (ok) {
      const int np = *sh.npending;
      const int ct = threadIdx.x - kWarpC0 * 32;  // 0 .. 32 * kConsumers - 1
      for (int e = 0; e < np; ++e) {
        const Pending pe = sh.pending[e];
        if (!pe.last) continue;
        __threadfence();
        const float* base = partials + static_cast<int64_t>(pe.rb) * sp.s_max * (kMaxM * kRows);
        for (int idx = ct; idx < M * kRows; idx += 32 * kConsumers) {
          float v = __ldcg(base + idx);
          for (int cc = 1; cc < pe.ncover; ++cc) v += __ldcg(base + cc * (kMaxM * kRows) + idx);
          const int m = idx / kRows, n = pe.rb * kRows + idx % kRows;
          if (n < N) store_y(Y, y_f32, static_cast<int64_t>(m) * N + n, v);
        }
        if (leader) counters[pe.rb] = 0;  // ready for the next call
      }
    }
  }
  __syncthreads();
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

size_t align256(size_t x) { return (x + 255) & ~static_cast<size_t>(255); }

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
  static bool attr_set = false;  // per template instance
  if (!attr_set) {
    cudaError_t e = cudaFuncSetAttribute(gemm_decode_kernel<B, NT, GS>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, C::kSmem);
    if (e != cudaSuccess) return e;
    e = cudaFuncSetAttribute(gemm_decode_kernel<B, NT, GS>,
                             cudaFuncAttributePreferredSharedMemoryCarveout,
                             static_cast<int>(cudaSharedmemCarveoutMaxShared));
    if (e != cudaSuccess) return e;
    attr_set = true;
  }
  const Split sp = make_split(N, K, GS, resident_ctas());
  int* counters = static_cast<int*>(workspace);
  float* partials = reinterpret_cast<float*>(static_cast<uint8_t*>(workspace) + kCounterBytes);
  gemm_decode_kernel<B, NT, GS><<<sp.nctas, kThreads, C::kSmem, stream>>>(
      tw, X, M, N, K, scales, zeros, Y, y_f32 ? 1 : 0, sp, counters, partials, flags);
  return cudaGetLastError();
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

// The device address of g_static_scratch on the current device.  In host
// code the array's name is only a host-side stand-in, so the address is
// looked up (once per device, with that device current) and cached.
cudaError_t static_scratch(void** out) {
  int dev = -1;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lock(g_static_mu);
  if (!g_static_ptr[dev]) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_static_scratch);
    if (e != cudaSuccess) return e;
    g_static_ptr[dev] = p;
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
