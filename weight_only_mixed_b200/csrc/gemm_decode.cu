// gemm_decode.cu -- dequantize-GEMM for decode batches (M <= 16) on tcgen05,
// with the weight operand in tensor memory and a persistent stream-K split.
//
// Y = X W^T, w = s * (q - z) (the weight-only linear layer of the pages'
// serving path; gist.science summary, Key Results "Inference Speedup").  At
// decode sizes the layer must stream the packed weights at HBM speed.  Each
// dequant thread owns one weight row -- one TMEM lane -- turns 64 of its codes
// per group into exact bf16 (q - z) in registers and stores them straight into
// TMEM (tcgen05.st); tcgen05.mma reads that A operand from TMEM and the
// activation tile (M <= 16 rows, TMA-loaded) from shared memory.  The fp16
// group scale multiplies the fp32 group product when it is folded into the
// accumulators, so the only rounding is fp32 accumulation.
//
// Work split.  The layer is ceil(N/128) row tiles x G groups ("group tiles").
// One CTA runs per SM and takes a contiguous range of the row-major list of
// group tiles (stream-K), so every SM streams the same number of bytes
// whatever N and K are.  A row tile whose groups fall in one CTA's range is
// written straight to Y.  A row tile shared by several CTAs is reduced
// deterministically: each CTA writes its fp32 partial to slot (CTA - first
// CTA of the tile) of a caller-provided workspace and increments the tile's
// counter; the CTA that sees the count complete adds the slots in slot order,
// writes Y and resets the counter to zero.  The result therefore does not
// depend on which CTA finishes first.
//
// CTA (768 threads, 1 per SM):
//   warp 0      TMA producer of packed W (one 128-code group x 128 rows per stage).
//   warps 1, 3  MMA issuers (warp 1 also allocates the 512 TMEM columns);
//               issuer h takes groups h, h + 2, ...
//   warp 2      TMA producer of the activation tile (M rows x 128 k per group).
//   warps 4-19  dequant, four sets of four warps: warp w owns TMEM lane
//               quarter w % 4 (one weight row per thread, all 128 codes of
//               the group, and that row's zero point, loaded one group
//               ahead); set (w - 4) / 4 takes every fourth group, so four
//               groups are dequantized at once.
//   warps 20-23 fold: lane quarter w % 4; acc[m] += s[n, g] * P_g[n, m] for
//               the activation rows (scales loaded eight groups ahead), then
//               the tile's output / partial.
// A group's eight K = 16 MMAs go to four independent accumulators (MMA k into
// chain k % 4): an N = 16 MMA is short, and MMAs that accumulate into the
// same TMEM columns wait for each other, so a single chain would run at the
// tensor core's latency.  The fold adds the four chains in a fixed order.
// TMEM: a ring of 4 A buffers (64 columns: 128 bf16 codes per row) and a ring
// of 4 product buffers (4 chains x 16 fp32 columns).  Every hand-over is an
// mbarrier; every wait gives up after about 2 s, raises SLQ_FLAG_TIMEOUT and
// lets the CTA drain its copies and free TMEM.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include "dequant.cuh"
#include "internal.h"
#include "ptx.cuh"

namespace slq {
namespace {

using dq::load_unit;
using dq::sw128_desc;
using dq::unit_pairs;

constexpr int kRows = 128;   // weight rows per tile (MMA M, TMEM lanes)
constexpr int kBN = 16;      // activation rows per MMA (MMA N); M <= 16
constexpr int kNA = 4;       // A buffers in TMEM
constexpr int kNP = 4;       // product buffers in TMEM
constexpr int kChains = 4;   // independent accumulators per group
constexpr int kColP = kNA * 64;
constexpr int kCols = 512;
constexpr int kSX = 6;                  // activation stages (one group each)
constexpr int kXStage = 2 * kBN * 128;  // two 64-k swizzle atoms of 16 rows
constexpr int kSLook = 8;               // fold: scale loads in flight (groups)
// Dequant warps come in sets of four (one per TMEM lane quarter); set k
// dequantizes groups k, k + kSets, ... so that kSets groups are in flight.
constexpr int kSets = 4;
constexpr int kWarpW = 0, kWarpMma = 1, kWarpX = 2, kWarpMma2 = 3, kWarpDq0 = 4;
// One tcgen05.commit per group, on done[g % kDone]: it frees the group's A
// buffer and activation stage and publishes its product.  kDone is larger
// than every distance at which a consumer waits behind the MMAs (and a
// multiple of kSets), so no wait can confuse two phases of one barrier.
constexpr int kDone = 16;
constexpr int kNumDq = 4 * kSets;
constexpr int kWarpFold0 = kWarpDq0 + kNumDq;
constexpr int kNumFold = 4;
constexpr int kThreads = (kWarpFold0 + kNumFold) * 32;
constexpr int kMaxPending = 4;  // shared tiles per CTA (at most 2 occur)

static_assert(kColP + kNP * kChains * kBN == kCols, "TMEM budget");
static_assert(kDone > kSX && kDone > kNA && kDone > kNP && kDone % kSets == 0, "done ring");

template <int B>
constexpr int p_stage_bytes() {
  return kRows * 16 * B;
}

struct Pending {
  int rb, ncover, last;
};

template <int B>
struct Cfg {
  static constexpr int kFixed = 1024 /* alignment slack */ + kSX * kXStage +
                                1024 /* barriers, TMEM address, pending list */;
  static constexpr int kSPRaw = (227 * 1024 - kFixed) / p_stage_bytes<B>();
  static constexpr int kSP = kSPRaw > 32 ? 32 : kSPRaw;
  static constexpr int kSmem = kFixed + kSP * p_stage_bytes<B>();
  static_assert(kSmem <= 232448, "shared memory budget");
};

// Instruction descriptor, kind::f16: bf16 A and B (K-major), fp32 D, M = 128, N = 16.
constexpr uint32_t kIdesc = (1u << 4) | (1u << 7) | (1u << 10) |
                            (static_cast<uint32_t>(kBN >> 3) << 17) |
                            (static_cast<uint32_t>(kRows >> 4) << 24);

struct Bars {
  uint64_t* p_full;   // [kSP] packed stage landed (TMA)
  uint64_t* p_empty;  // [kSP] packed stage read by the dequant warps of its set (4)
  uint64_t* x_full;   // [kSX] activation stage landed (TMA)
  uint64_t* a_full;   // [kNA] A buffer written (the 4 dequant warps of a set)
  uint64_t* done;     // [kDone] MMAs of group g complete (one commit)
  uint64_t* d_empty;  // [kNP] product read by the fold (4 fold warps)
  uint64_t* mma_done; // both issuers' MMAs complete (2 commits)
  uint64_t* seg_bar;  // fold warps' partials of a shared tile written (4 fold warps)
  uint64_t* end_bar;  // fold thread 0 has recorded every shared tile (1)
  uint32_t* tmem_base;
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

// One fold step for MB activation rows: acc[m] += s * (c0 + c1 + c2 + c3)[m],
// the four accumulator chains of the group's product at TMEM address p (lane
// quarter already applied), added in a fixed order.  Releases the product
// buffer (d_empty) as soon as the loads have completed.
template <int MB>
__device__ __forceinline__ void tmem_ld_cols(uint32_t taddr, uint32_t (&r)[MB]) {
  if constexpr (MB == 1)
    asm volatile("tcgen05.ld.sync.aligned.32x32b.x1.b32 {%0}, [%1];" : "=r"(r[0]) : "r"(taddr));
  else if constexpr (MB == 2)
    asm volatile("tcgen05.ld.sync.aligned.32x32b.x2.b32 {%0, %1}, [%2];"
                 : "=r"(r[0]), "=r"(r[1]) : "r"(taddr));
  else if constexpr (MB == 4)
    asm volatile("tcgen05.ld.sync.aligned.32x32b.x4.b32 {%0, %1, %2, %3}, [%4];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]) : "r"(taddr));
  else if constexpr (MB == 8)
    tmem_ld_32x32b_x8(taddr, r);
  else
    tmem_ld_32x32b_x16(taddr, r);
}

template <int MB>
__device__ __forceinline__ void fold_cols(uint32_t p, float s, float* acc) {
  uint32_t r0[MB], r1[MB], r2[MB], r3[MB];
  tmem_ld_cols<MB>(p + 0 * kBN, r0);
  tmem_ld_cols<MB>(p + 1 * kBN, r1);
  tmem_ld_cols<MB>(p + 2 * kBN, r2);
  tmem_ld_cols<MB>(p + 3 * kBN, r3);
  tmem_wait_ld();
#pragma unroll
  for (int i = 0; i < MB; ++i) {
    const float v = (__uint_as_float(r0[i]) + __uint_as_float(r1[i])) +
                    (__uint_as_float(r2[i]) + __uint_as_float(r3[i]));
    acc[i] = fmaf(s, v, acc[i]);
  }
}

// Columns 0..MB-1 of the product; 16 columns go in two halves of 8 to bound
// the registers held at once.
template <int MB>
__device__ __forceinline__ void fold_group(uint32_t p, float s, float (&acc)[kBN]) {
  if constexpr (MB == 16) {
    fold_cols<8>(p, s, acc);
    fold_cols<8>(p + 8, s, acc + 8);
  } else {
    fold_cols<MB>(p, s, acc);
  }
}

// Stream-K geometry shared by every CTA of a launch.
struct Split {
  int G;        // groups per row tile
  int per;      // group tiles per CTA
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

template <int B>
__global__ void __launch_bounds__(kThreads, 1)
    gemm_decode_kernel(const __grid_constant__ CUtensorMap tmap_w,
                       const __grid_constant__ CUtensorMap tmap_x, int M, int N, int K,
                       const uint16_t* __restrict__ scales, const uint8_t* __restrict__ zeros,
                       void* __restrict__ Y, int y_f32, Split sp, int* __restrict__ counters,
                       float* __restrict__ partials, uint32_t* __restrict__ flags) {
  using C = Cfg<B>;
  constexpr int kSP = C::kSP;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw_addr = smem_u32(smem_raw);
  uint8_t* smem = smem_raw + (((raw_addr + 1023u) & ~1023u) - raw_addr);
  uint8_t* xbuf = smem;                  // [kSX][2][16 rows][128 B], swizzled
  uint8_t* pbuf = xbuf + kSX * kXStage;  // [kSP][128 rows][16B B]
  uint64_t* bars = reinterpret_cast<uint64_t*>(pbuf + kSP * p_stage_bytes<B>());
  Bars sh;
  sh.p_full = bars;
  sh.p_empty = sh.p_full + kSP;
  sh.x_full = sh.p_empty + kSP;
  sh.a_full = sh.x_full + kSX;
  sh.done = sh.a_full + kNA;
  sh.d_empty = sh.done + kDone;
  sh.mma_done = sh.d_empty + kNP;
  sh.seg_bar = sh.mma_done + 1;
  sh.end_bar = sh.seg_bar + 1;
  sh.tmem_base = reinterpret_cast<uint32_t*>(sh.end_bar + 1);
  sh.abort_flag = reinterpret_cast<volatile int*>(sh.tmem_base + 1);
  sh.npending = const_cast<int*>(sh.abort_flag) + 1;
  sh.pending = reinterpret_cast<Pending*>(sh.npending + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int G = sp.G;
  const int rbs = (N + kRows - 1) / kRows;
  const int64_t total = static_cast<int64_t>(rbs) * G;
  const int64_t t0 = static_cast<int64_t>(blockIdx.x) * sp.per;
  const int64_t t1 = (t0 + sp.per) < total ? (t0 + sp.per) : total;
  const int ng = static_cast<int>(t1 - t0);  // group tiles of this CTA
  const int mr = M < kBN ? M : kBN;          // activation rows the TMA brings in
  const int rb0 = static_cast<int>(t0 / G), gk0 = static_cast<int>(t0 % G);

  if (threadIdx.x == 0) {
    for (int i = 0; i < kSP; ++i) {
      mbar_init(&sh.p_full[i], 1);
      mbar_init(&sh.p_empty[i], 4);
    }
    for (int i = 0; i < kSX; ++i) mbar_init(&sh.x_full[i], 1);
    for (int i = 0; i < kNA; ++i) mbar_init(&sh.a_full[i], 4);
    for (int i = 0; i < kDone; ++i) mbar_init(&sh.done[i], 1);
    for (int i = 0; i < kNP; ++i) mbar_init(&sh.d_empty[i], kNumFold);
    mbar_init(sh.mma_done, 2);
    mbar_init(sh.seg_bar, kNumFold);
    mbar_init(sh.end_bar, 1);
    *sh.abort_flag = 0;
    *sh.npending = 0;
    fence_mbarrier_init();
  }
  __syncwarp();
  if (warp == kWarpMma) {
    tmem_alloc(sh.tmem_base, kCols);
    tmem_relinquish();
  }
  tc_fence_before_sync();
  __syncthreads();
  tc_fence_after_sync();
  const uint32_t tmem = *sh.tmem_base;

  if (warp == kWarpW) {
    // ---------------- packed-W producer (TMA) ----------------
    if (lane == 0) {
      prefetch_tmap(&tmap_w);
      int rb = rb0, gk = gk0;
      int issued = 0;
      for (int g = 0; g < ng; ++g) {
        const int s = g % kSP;
        if (!wait_or_abort(&sh.p_empty[s], ((g / kSP) & 1) ^ 1, sh, flags)) break;
        mbar_arrive_expect_tx(&sh.p_full[s], p_stage_bytes<B>());
        tma_load_2d(pbuf + s * p_stage_bytes<B>(), &tmap_w, &sh.p_full[s], gk * 4 * B, rb * kRows);
        ++issued;
        if (++gk == G) {
          gk = 0;
          ++rb;
        }
      }
      for (int i = issued - kSP; i < issued; ++i)  // every issued copy lands before exit
        if (i >= 0) mbar_wait_bounded(&sh.p_full[i % kSP], (i / kSP) & 1);
    }
    __syncwarp();
  } else if (warp == kWarpX) {
    // ---------------- activation producer (TMA, rows >= M not loaded) ----------------
    if (lane == 0) {
      prefetch_tmap(&tmap_x);
      int issued = 0;
      int gk = gk0;
      for (int g = 0; g < ng; ++g, gk = (gk + 1 == G) ? 0 : gk + 1) {
        const int s = g % kSX;
        const int gp = g - kSX;  // the group that last used this stage
        if (gp >= 0 && !wait_or_abort(&sh.done[gp % kDone], (gp / kDone) & 1, sh, flags)) break;
        uint8_t* dst = xbuf + s * kXStage;
        mbar_arrive_expect_tx(&sh.x_full[s], 2 * mr * 128);
        tma_load_2d(dst, &tmap_x, &sh.x_full[s], gk * kGroup, 0);
        tma_load_2d(dst + kBN * 128, &tmap_x, &sh.x_full[s], gk * kGroup + 64, 0);
        ++issued;
      }
      for (int i = issued - kSX; i < issued; ++i)
        if (i >= 0) mbar_wait_bounded(&sh.x_full[i % kSX], (i / kSX) & 1);
    }
    __syncwarp();
  } else if (warp == kWarpMma || warp == kWarpMma2) {
    // ---------------- MMA issuers: issuer h takes groups h, h + 2, ...; group g -> product g % kNP ----------------
    // Two issuing threads: one thread's tcgen05.mma issue rate is below the
    // tensor pipe's rate for these short (N = 16) MMAs.
    if (lane == 0) {
      const int h = warp == kWarpMma ? 0 : 1;
      bool ok = true;
      for (int g = h; g < ng && ok; g += 2) {
        const int ia = g % kNA, ix = g % kSX, ip = g % kNP;
        ok = wait_or_abort(&sh.a_full[ia], (g / kNA) & 1, sh, flags) &&
             wait_or_abort(&sh.x_full[ix], (g / kSX) & 1, sh, flags) &&
             wait_or_abort(&sh.d_empty[ip], ((g / kNP) & 1) ^ 1, sh, flags);
        if (!ok) break;
        tc_fence_after_sync();
        const uint32_t a = tmem + static_cast<uint32_t>(ia * 64);
        const uint32_t d = tmem + static_cast<uint32_t>(kColP + ip * kChains * kBN);
        const uint32_t xs = smem_u32(xbuf + ix * kXStage);
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {  // K = 16 per MMA: 8 TMEM columns of A, 32 bytes of X
          const uint64_t bd = sw128_desc(xs + (kk >> 2) * kBN * 128) + 2 * (kk & 3);
          umma_bf16_ts(d + static_cast<uint32_t>((kk % kChains) * kBN),
                       a + static_cast<uint32_t>(8 * kk), bd, kIdesc, kk >= kChains ? 1u : 0u);
        }
        umma_commit(&sh.done[g % kDone]);
      }
      umma_commit(sh.mma_done);
      mbar_wait_bounded(sh.mma_done, 0);  // no MMA in flight past this point
    }
    __syncwarp();
  } else if (warp >= kWarpDq0 && warp < kWarpDq0 + kNumDq) {
    // ---------------- dequant: all 128 codes of row 32q + lane; groups set, set + kSets, ... ----------------
    const int q = warp & 3;
    const int set = (warp - kWarpDq0) >> 2;
    const int row = 32 * q + lane;
    const uint32_t lane_addr = static_cast<uint32_t>(32 * q) << 16;
    // Cursor (rb, gk) of group `set`, and of the next group of this set.
    int rb = rb0, gk = gk0 + set;
    while (gk >= G) {
      gk -= G;
      ++rb;
    }
    auto zaddr = [&](int rb_, int gk_) -> const uint8_t* {
      const int n = min(min(rb_, rbs - 1) * kRows + row, N - 1);  // clamped: always a valid address
      return zeros + static_cast<int64_t>(n) * G + gk_;
    };
    uint32_t z_next = *zaddr(rb, gk);
    for (int g = set; g < ng; g += kSets) {
      const uint32_t z = z_next;
      gk += kSets;
      while (gk >= G) {
        gk -= G;
        ++rb;
      }
      z_next = *zaddr(rb, gk);  // next group of this set, consumed one iteration later
      const int ia = g % kNA, sp_ = g % kSP;
      const int gp = g - kNA;  // the group that last used this A buffer
      bool ok = (gp < 0 || wait_or_abort(&sh.done[gp % kDone], (gp / kDone) & 1, sh, flags)) &&
                wait_or_abort(&sh.p_full[sp_], (g / kSP) & 1, sh, flags);
      if (!__all_sync(0xffffffffu, ok)) break;
      tc_fence_after_sync();
      const uint8_t* pst = pbuf + sp_ * p_stage_bytes<B>();
      const uint32_t a = tmem + lane_addr + static_cast<uint32_t>(ia * 64);
#pragma unroll
      for (int u = 0; u < 4; ++u) {  // 32 codes per unit -> 16 TMEM columns
        uint32_t w[B];
        load_unit<B>(pst, row, u, w);
        uint32_t pr[16];
        unit_pairs<B>(w, z, pr);
        tmem_st_32x32b_x16(a + static_cast<uint32_t>(16 * u), pr);
      }
      tmem_wait_st();
      tc_fence_before_sync();
      __syncwarp();
      if (lane == 0) {
        mbar_arrive(&sh.a_full[ia]);
        mbar_arrive(&sh.p_empty[sp_]);
      }
    }
  } else if (warp >= kWarpFold0) {
    // ---------------- fold + output: row 32q + lane, activation rows 0..M-1 ----------------
    // Hand-overs among the four fold warps use mbarriers with bounded waits
    // (not bar.sync), so a warp that gives up after a timeout cannot leave the
    // others blocked.
    const int q = warp & 3;
    const int row = 32 * q + lane;
    const bool leader = threadIdx.x == kWarpFold0 * 32;
    const uint32_t lane_addr = static_cast<uint32_t>(32 * q) << 16;
    const int mb = M <= 1 ? 1 : M <= 2 ? 2 : M <= 4 ? 4 : M <= 8 ? 8 : 16;
    float acc[kBN];
#pragma unroll
    for (int i = 0; i < kBN; ++i) acc[i] = 0.0f;
    // Scales of this row, kSLook groups ahead (clamped addresses, always valid).
    int frb = rb0, fgk = gk0;
    auto sload = [&]() -> uint32_t {
      const int n = min(min(frb, rbs - 1) * kRows + row, N - 1);
      const uint32_t v = scales[static_cast<int64_t>(n) * G + fgk];
      if (++fgk == G) {
        fgk = 0;
        ++frb;
      }
      return v;
    };
    uint32_t sr[kSLook];
#pragma unroll
    for (int j = 0; j < kSLook; ++j) sr[j] = sload();
    bool ok = true;
    int nseg = 0;  // shared row tiles met so far (the same count in every fold warp)
    int rb = rb0, gk = gk0;
    // The ring slot index j must stay a compile-time constant (the ring lives
    // in registers), so the unrolled body is predicated instead of exited.
    for (int g0 = 0; g0 < ng && ok; g0 += kSLook) {
#pragma unroll
      for (int j = 0; j < kSLook; ++j) {
        const int g = g0 + j;
        if (g < ng && ok)
          ok = __all_sync(0xffffffffu, wait_or_abort(&sh.done[g % kDone], (g / kDone) & 1, sh, flags));
        if (g < ng && ok) {
        const int ip = g % kNP;
        tc_fence_after_sync();
        const float s = __half2float(__ushort_as_half(static_cast<uint16_t>(sr[j])));
        sr[j] = sload();
        const uint32_t p = tmem + lane_addr + static_cast<uint32_t>(kColP + ip * kChains * kBN);
        switch (mb) {
          case 1: fold_group<1>(p, s, acc); break;
          case 2: fold_group<2>(p, s, acc); break;
          case 4: fold_group<4>(p, s, acc); break;
          case 8: fold_group<8>(p, s, acc); break;
          default: fold_group<16>(p, s, acc); break;
        }
        tc_fence_before_sync();
        __syncwarp();
        if (lane == 0) mbar_arrive(&sh.d_empty[ip]);

        // End of this CTA's part of a row tile: write it out.
        if (gk == G - 1 || g == ng - 1) {
          const int c0 = first_cta(sp, rb);
          const int ncover = last_cta(sp, rb) - c0 + 1;
          const int n = rb * kRows + row;
          if (ncover == 1) {
            if (n < N) {
#pragma unroll
              for (int m = 0; m < kBN; ++m) {
                if (m < M) {
                  const int64_t o = static_cast<int64_t>(m) * N + n;
                  if (y_f32)
                    static_cast<float*>(Y)[o] = acc[m];
                  else
                    static_cast<__nv_bfloat16*>(Y)[o] = __float2bfloat16_rn(acc[m]);
                }
              }
            }
          } else {
            const int slot = static_cast<int>(blockIdx.x) - c0;
            float* part = partials + (static_cast<int64_t>(rb) * sp.s_max + slot) * (kBN * kRows);
#pragma unroll
            for (int m = 0; m < kBN; ++m)
              if (m < M) part[m * kRows + row] = acc[m];
            __syncwarp();
            if (lane == 0) mbar_arrive(sh.seg_bar);
            if (leader && wait_or_abort(sh.seg_bar, nseg & 1, sh, flags)) {
              // Every fold warp's partial is written (mbarrier acquire); the
              // release half of the atomic publishes them to the other CTAs.
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
          for (int i = 0; i < kBN; ++i) acc[i] = 0.0f;
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
      for (int e = 0; e < np; ++e) {
        const Pending pe = sh.pending[e];
        if (!pe.last) continue;
        __threadfence();
        const int n = pe.rb * kRows + row;
        const float* base = partials + static_cast<int64_t>(pe.rb) * sp.s_max * (kBN * kRows);
        for (int m = 0; m < M; ++m) {
          float v = __ldcg(base + m * kRows + row);
          for (int c = 1; c < pe.ncover; ++c) v += __ldcg(base + c * (kBN * kRows) + m * kRows + row);
          if (n < N) {
            const int64_t o = static_cast<int64_t>(m) * N + n;
            if (y_f32)
              static_cast<float*>(Y)[o] = v;
            else
              static_cast<__nv_bfloat16*>(Y)[o] = __float2bfloat16_rn(v);
          }
        }
        if (leader) counters[pe.rb] = 0;  // ready for the next call
      }
    }
  }

  tc_fence_before_sync();
  __syncthreads();
  if (warp == kWarpMma) {
    tc_fence_after_sync();
    tmem_dealloc(tmem, kCols);
  }
}

// ---------------------------------------------------------------------------
// Host side
// ---------------------------------------------------------------------------

// Stream-K geometry for a layer on a GPU with `sms` SMs (one CTA per SM).
Split make_split(int64_t N, int64_t K, int sms) {
  Split sp;
  sp.G = static_cast<int>(K / kGroup);
  const int64_t rbs = (N + kRows - 1) / kRows;
  const int64_t total = rbs * sp.G;
  const int64_t ctas = total < sms ? total : sms;
  sp.per = static_cast<int>((total + ctas - 1) / ctas);
  sp.nctas = static_cast<int>((total + sp.per - 1) / sp.per);
  // A row tile of G groups meets at most ceil((G - 1) / per) + 1 CTA ranges.
  int s = (sp.G - 1 + sp.per - 1) / sp.per + 1;
  sp.s_max = s < sp.nctas ? s : sp.nctas;
  return sp;
}

int device_sms() {
  int dev = 0, sms = 148;
  if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  return sms;
}

size_t align256(size_t x) { return (x + 255) & ~static_cast<size_t>(255); }

template <int B>
cudaError_t launch_b(const uint16_t* X, int M, int N, int K, const uint32_t* packed,
                     const uint16_t* scales, const uint8_t* zeros, void* Y, bool y_f32,
                     void* workspace, uint32_t* flags, cudaStream_t stream) {
  using C = Cfg<B>;
  CUtensorMap tw, tx;
  const CUtensorMapSwizzle swz = B == 8   ? CU_TENSOR_MAP_SWIZZLE_128B
                                 : B == 4 ? CU_TENSOR_MAP_SWIZZLE_64B
                                 : B == 2 ? CU_TENSOR_MAP_SWIZZLE_32B
                                          : CU_TENSOR_MAP_SWIZZLE_NONE;
  const int mr = M < kBN ? M : kBN;
  if (!encode_tensor_map_2d(&tw, CU_TENSOR_MAP_DATA_TYPE_UINT32, packed,
                            static_cast<uint64_t>(K) * B / 32, static_cast<uint64_t>(N),
                            static_cast<uint64_t>(K) * B / 8, 4 * B, kRows, swz) ||
      !encode_tensor_map_2d(&tx, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, X, static_cast<uint64_t>(K),
                            static_cast<uint64_t>(M), static_cast<uint64_t>(K) * 2, 64,
                            static_cast<uint32_t>(mr), CU_TENSOR_MAP_SWIZZLE_128B))
    return cudaErrorInvalidValue;
  static bool attr_set = false;  // per template instance
  if (!attr_set) {
    cudaError_t e = cudaFuncSetAttribute(gemm_decode_kernel<B>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, C::kSmem);
    if (e != cudaSuccess) return e;
    attr_set = true;
  }
  const Split sp = make_split(N, K, device_sms());
  const int64_t rbs = (N + kRows - 1) / kRows;
  int* counters = static_cast<int*>(workspace);
  float* partials = reinterpret_cast<float*>(static_cast<uint8_t*>(workspace) +
                                             align256(static_cast<size_t>(rbs) * sizeof(int)));
  gemm_decode_kernel<B><<<sp.nctas, kThreads, C::kSmem, stream>>>(
      tw, tx, M, N, K, scales, zeros, Y, y_f32 ? 1 : 0, sp, counters, partials, flags);
  return cudaGetLastError();
}

}  // namespace

size_t gemm_decode_workspace_bytes(int64_t N, int64_t K) {
  const Split sp = make_split(N, K, device_sms());
  const int64_t rbs = (N + kRows - 1) / kRows;
  if (sp.s_max <= 1) return 0;
  return align256(static_cast<size_t>(rbs) * sizeof(int)) +
         static_cast<size_t>(rbs) * sp.s_max * kBN * kRows * sizeof(float);
}

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

}  // namespace slq
