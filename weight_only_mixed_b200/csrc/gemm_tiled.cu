// gemm_tiled.cu -- tiled dequantize-GEMM on the 5th-generation tensor cores.
//
// Y = X W^T with w = s * (q - z) (the weight-only linear layer of the pages'
// serving path; gist.science summary, Key Results "Inference Speedup").  This
// kernel serves M > 16 (prefill and large batches), where the contraction is
// dense enough for the tensor cores to be the bound.
//
// Orientation: the weight tile is the A operand (M_mma = 128 rows of W), the
// activation tile is the B operand (N_mma = BN rows of X, 64..256), so one
// dequantized weight tile feeds BN activation rows and the product sits in
// TMEM as 128 lanes (rows n of W) x BN fp32 columns (rows m of X).
//
// Exact scaling.  The A operand is (q - z), an integer of at most 8 bits and so
// an exact bf16 value.  Each 128-wide group g is multiplied into its own TMEM
// product buffer, and fold warps -- each thread owns one TMEM lane, i.e. one
// row n of W -- add s[n, g] * P_g into fp32 registers.  The only rounding is
// fp32 accumulation, as in the decode kernels.  (Multiplying the bf16-rounded
// weights bf16_rn(s (q - z)) instead, with one accumulator over K and no
// fold, was measured ~17 % faster but moves y by up to 1.7e-2 of its rms,
// outside the GEMM tolerance of max |y - y_ref| <= 1e-2 rms.)
//
// The kernel, its warp roles and barriers are described below, above
// gemm_tiled_tm_kernel.  Every wait gives up after about 2 s, raises
// SLQ_FLAG_TIMEOUT and lets the CTA drain its copies and free TMEM.
#include <cooperative_groups.h>
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include <mutex>

#include "dequant.cuh"
#include "internal.h"
#include "ptx.cuh"

namespace cg = cooperative_groups;

namespace slq {
namespace {

using dq::load_half;
using dq::sw128_desc;
using dq::unit_pairs;

constexpr int kBM = 128;     // W rows per tile (MMA M)
constexpr int kBK = 64;      // k per A / X stage: one 128-byte swizzle atom of bf16
constexpr int kSRing = 16;   // scale / zero ring (groups); must exceed packed stages + 2
constexpr int kMaxCluster = 8;
constexpr int kWarpX = 0, kWarpMma = 1, kWarpW = 2;

template <int B>
constexpr int p_stage_bytes() {
  return kBM * 16 * B;
}

// Instruction descriptor, kind::f16: bf16 A and B (K-major), fp32 D, M = 128, N = BN.
template <int BN>
__host__ __device__ constexpr uint32_t instr_desc() {
  return (1u << 4) | (1u << 7) | (1u << 10) | (static_cast<uint32_t>(BN >> 3) << 17) |
         (static_cast<uint32_t>(kBM >> 4) << 24);
}

struct Bars {
  uint64_t* x_full;
  uint64_t* x_empty;
  uint64_t* a_full;
  uint64_t* a_empty;
  uint64_t* p_full;
  uint64_t* p_empty;
  uint64_t* pf;  // P buffer filled (tcgen05.commit)
  uint64_t* pe;  // P buffer drained by the workers
  uint64_t* mma_done;
  uint32_t* tmem_base;
  volatile int* abort_flag;
};

// Bounded wait; on timeout raises the flag word and the CTA-wide abort flag.
// The cycle counter and the abort flag are read only every few polls.
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

// ---------------------------------------------------------------------------
// Dequantize-GEMM with the weight operand in tensor memory.
//
// Two limits shape this kernel.  (1) Shared-memory bandwidth, 128 bytes per
// clock per SM: with A in shared memory, one 128-wide group of a 128 x 256
// tile moves ~208 KB through it (MMA reads of A and B, TMA writes of X and
// packed W, the dequant's A writes) -- ~1600 clocks against 1024 clocks of
// tensor-core time.  Here the dequantized (q - z) tile goes from registers
// into TMEM (tcgen05.st) and tcgen05.mma reads A from TMEM, which leaves
// ~144 KB per group.  (2) Issue rate: one thread issues a tcgen05.mma about
// every 60 clocks, the time of one M = 128, N = 128, K = 16 product, so the
// barrier waits and commits between products stall the tensor core unless
// each issuing thread carries no more than half of them.  A 256-wide tile is
// therefore two MMA streams of N = 128, one per half of the activation rows,
// issued by two threads.
//
// TMEM (512 columns): three product buffers P of NW = min(BN, 128) columns at
// columns 0, NW, 2 NW (product h = group * NH + half goes to buffer h % 3),
// and two A buffers of 64 columns (128 codes per row, two bf16 per column)
// at 384 and 448.
//
// Each issuing thread waits on two barriers and commits once per group
// (a second commit per group was measured to cost ~15 % of the tensor
// core's time): ready[s] completes when group g's activations have landed
// (slot s = g % kXG of the activation ring, both 64-k stages) and its A tile
// is in TMEM; pe[b] when product buffer b is free.  Its commit goes to
// gdone[s], which completes once every stream's products of group g are
// done: the fold warps wait on it, and it frees activation slot s and A
// buffer g % 2.
//
// Warp roles (768 threads, one CTA per SM):
//   warp 0        TMA producer of X (two 64 k x BN tiles per group).
//   warp 1        TMEM allocator; one lane issues the MMAs of half 0.
//   warp 2        TMA producer of packed W and the scale / zero staging.
//   warp 3        one lane issues the MMAs of half 1 (BN = 256).
//   warps 4-7     unpack: warp w owns TMEM lanes 32 (w % 4) .. + 31 (rows of
//                 W) and writes all 128 codes of the group for its row.
//   warps 8-23    fold: acc += s[n, g] * P in registers; warp w owns TMEM
//                 lanes 32 (w % 4) .. + 31 and BN / 4 columns of the tile.
// Registers are rebalanced per warpgroup with setmaxnreg: the launch gives
// 768 x 80 = 61440; after the split 128 x 48 + 128 x 48 + 512 x 96 = 61440.
// Narrow tiles (BN <= 128) may split K over a cluster; the partial tiles are
// added in rank order through distributed shared memory.
// The arithmetic: exact bf16 (q - z) tiles, each group's fp32 product in its
// own TMEM buffer, scaled by the fp16 scale and added in fp32, group by group.
// ---------------------------------------------------------------------------
constexpr int kUnpackWarpsTm = 4;
constexpr int kFoldWarpsTm = 16;
constexpr int kWarpMma1 = 3;  // second MMA stream (BN = 256)
constexpr int kWarpUnpackTm = 4, kWarpFoldTm = kWarpUnpackTm + kUnpackWarpsTm;
constexpr int kThreadsTm = (kWarpFoldTm + kFoldWarpsTm) * 32;
constexpr int kRegsTm = 80;
constexpr int kRegsTmWg0 = 48, kRegsTmUnpack = 48, kRegsTmFold = 96;
constexpr int kPBufs = 3;           // product buffers in TMEM
constexpr int kACol = 384;          // first column of the two A buffers
static_assert(kThreadsTm == 768, "six warpgroups");
static_assert(128 * kRegsTmWg0 + 128 * kRegsTmUnpack + 512 * kRegsTmFold <= kThreadsTm * kRegsTm,
              "the register split must fit the launch's registers");

template <int B, int BN>
struct CfgTm {
  static constexpr int kNW = BN > 128 ? 128 : BN;  // MMA N
  static constexpr int kNH = BN / kNW;             // MMA streams (halves of the tile)
  static constexpr int kAcc = BN / 4;              // accumulators per fold thread
  static constexpr int kXG = BN == 256 ? 2 : 4;    // activation ring, in groups
  static constexpr int kXStage = BN * 128;         // one 64-k stage
  static constexpr int kFixed = 1024 /* alignment slack */ + kXG * 2 * kXStage +
                                kSRing * kBM * 3 + 512 /* barriers, TMEM address, flag */;
  static constexpr int kBudget = 227 * 1024;
  static constexpr int kSPRaw = (kBudget - kFixed) / p_stage_bytes<B>();
  static constexpr int kSP = kSPRaw > 8 ? 8 : (kSPRaw < 2 ? 2 : kSPRaw);
  // More than half of the SM's shared memory, so one CTA per SM (TMEM holds
  // one 512-column allocation).
  static constexpr int kSmem = (kFixed + kSP * p_stage_bytes<B>()) > 120 * 1024
                                   ? kFixed + kSP * p_stage_bytes<B>()
                                   : 120 * 1024;
  static_assert(kSmem <= 232448, "shared memory budget");
  static_assert(kPBufs * kNW <= kACol, "product buffers below the A buffers");
  static_assert(kXG >= 2 && kXG % 2 == 0, "A buffer g % 2 is freed with slot g % kXG");
  // Staging the scales of group g needs the unpack of g - kSP done, hence the
  // MMAs of g - kSP - 2 and the folds of every group up to g - kSP - 5.
  static_assert(kSRing >= kSP + 5, "scale ring shorter than the pipeline");
  static_assert(kXG * 2 * kXStage >= kBM * BN * 4, "X ring doubles as the split-K partial buffer");
  static_assert(kNH == 1 || kNH == 2, "one or two MMA streams");
};

template <int B, int BN>
__global__ void __maxnreg__(kRegsTm)
    gemm_tiled_tm_kernel(const __grid_constant__ CUtensorMap tmap_x,
                         const __grid_constant__ CUtensorMap tmap_w, int M, int N, int K,
                         const uint16_t* __restrict__ scales, const uint8_t* __restrict__ zeros,
                         void* __restrict__ Y, int y_f32, int groups_per_slice,
                         uint32_t* __restrict__ flags) {
  using C = CfgTm<B, BN>;
  constexpr int kSP = C::kSP, kXG = C::kXG, kNW = C::kNW, kNH = C::kNH, kAcc = C::kAcc;
  constexpr int kSlot = 2 * C::kXStage;  // one group of X
  constexpr int kCols = 512;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw_addr = smem_u32(smem_raw);
  uint8_t* smem = smem_raw + (((raw_addr + 1023u) & ~1023u) - raw_addr);
  uint8_t* xbuf = smem;
  uint8_t* pbuf = xbuf + kXG * kSlot;
  uint16_t* sring = reinterpret_cast<uint16_t*>(pbuf + kSP * p_stage_bytes<B>());  // [kSRing][128]
  uint8_t* zring = reinterpret_cast<uint8_t*>(sring + kSRing * kBM);                // [kSRing][128]
  uint64_t* bars = reinterpret_cast<uint64_t*>(zring + kSRing * kBM);
  // ready[kXG], gdone[kXG], p_full[kSP], p_empty[kSP], pf[3], pe[3], mma_done
  Bars sh;
  sh.x_full = bars;              // ready: group's X landed and its A tile written
  sh.x_empty = sh.x_full + kXG;  // gdone: the group's products complete
  sh.a_full = nullptr;
  sh.a_empty = nullptr;
  sh.p_full = sh.x_empty + kXG;
  sh.p_empty = sh.p_full + kSP;
  sh.pf = sh.p_empty + kSP;
  sh.pe = sh.pf + kPBufs;
  sh.mma_done = sh.pe + kPBufs;
  sh.tmem_base = reinterpret_cast<uint32_t*>(sh.mma_done + 1);
  sh.abort_flag = reinterpret_cast<volatile int*>(sh.tmem_base + 1);
  uint64_t* ready = sh.x_full;
  uint64_t* gdone = sh.x_empty;

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int n0 = blockIdx.x * kBM;
  const int m0 = blockIdx.y * BN;
  const int G = K / kGroup;
  // K slice of this CTA (blockIdx.z; the CTAs of one slice set form a cluster).
  const int g_begin = blockIdx.z * groups_per_slice;
  const int g_end = min(G, g_begin + groups_per_slice);
  const int ng = g_end - g_begin;

  if (threadIdx.x == 0) {
    for (int i = 0; i < kXG; ++i) {
      mbar_init(&ready[i], 1 + kUnpackWarpsTm);  // X producer (expect_tx) + unpack warps
      mbar_init(&gdone[i], kNH);  // one commit per MMA stream
    }
    for (int i = 0; i < kSP; ++i) {
      mbar_init(&sh.p_full[i], 1 + 32);  // TMA arrival + the producer warp's lanes
      mbar_init(&sh.p_empty[i], kUnpackWarpsTm);
    }
    for (int i = 0; i < kPBufs; ++i) {
      mbar_init(&sh.pf[i], 1);
      mbar_init(&sh.pe[i], kFoldWarpsTm / kNH);  // the fold warps of that buffer's half
    }
    mbar_init(sh.mma_done, kNH);
    *sh.abort_flag = 0;
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

  // Split K: every thread meets the cluster barrier twice -- once when all
  // partial tiles are in shared memory, once after rank 0 has read them.
  auto cluster_arrive_wait = [&]() {
    if (kNH == 1 && gridDim.z > 1) {
      asm volatile("barrier.cluster.arrive.release.aligned;\n" ::: "memory");
      asm volatile("barrier.cluster.wait.acquire.aligned;\n" ::: "memory");
    }
  };

  if (warp < kWarpUnpackTm) {
    // ---------------- producers and MMA issuers (warpgroup 0) ----------------
    asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;\n" ::"n"(kRegsTmWg0) : "memory");
    if (warp == kWarpX) {
      if (lane == 0) {
        prefetch_tmap(&tmap_x);
        int issued = 0;
        for (int g = 0; g < ng; ++g) {
          const int s = g % kXG;
          if (g >= kXG && !wait_or_abort(&gdone[s], ((g / kXG) - 1) & 1, sh, flags)) break;
          mbar_arrive_expect_tx(&ready[s], kSlot);
          tma_load_2d(xbuf + s * kSlot, &tmap_x, &ready[s], (2 * (g_begin + g)) * kBK, m0);
          tma_load_2d(xbuf + s * kSlot + C::kXStage, &tmap_x, &ready[s],
                      (2 * (g_begin + g) + 1) * kBK, m0);
          ++issued;
        }
        // Drain: every issued copy must land before the CTA may exit.
        for (int i = issued - kXG; i < issued; ++i)
          if (i >= 0) mbar_wait_bounded(&ready[i % kXG], (i / kXG) & 1);
      }
      __syncwarp();
    } else if (warp == kWarpW) {
      if (lane == 0) prefetch_tmap(&tmap_w);
      constexpr int kLookahead = 2;
      auto fetch = [&](int g, int q) -> uint32_t {
        const int n = n0 + 4 * lane + q;
        if (g >= ng || n >= N) return 0u;
        const int64_t gi = static_cast<int64_t>(n) * G + g_begin + g;
        return static_cast<uint32_t>(scales[gi]) | (static_cast<uint32_t>(zeros[gi]) << 16);
      };
      uint32_t ring[kLookahead][4];
#pragma unroll
      for (int j = 0; j < kLookahead; ++j)
#pragma unroll
        for (int q = 0; q < 4; ++q) ring[j][q] = fetch(j, q);
      int issued = 0;
      bool run = true;
      for (int g0 = 0; g0 < ng && run; g0 += kLookahead) {
#pragma unroll
        for (int j = 0; j < kLookahead; ++j) {
          const int g = g0 + j;
          if (g >= ng || !run) break;
          const int s = g % kSP;
          const bool ok = wait_or_abort(&sh.p_empty[s], ((g / kSP) & 1) ^ 1, sh, flags);
          if (!__all_sync(0xffffffffu, ok)) {
            run = false;
            break;
          }
          if (lane == 0) {
            mbar_arrive_expect_tx(&sh.p_full[s], p_stage_bytes<B>());
            tma_load_2d(pbuf + s * p_stage_bytes<B>(), &tmap_w, &sh.p_full[s],
                        (g_begin + g) * 4 * B, n0);
          }
          uint16_t* sr = sring + (g % kSRing) * kBM;
          uint8_t* zr = zring + (g % kSRing) * kBM;
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            sr[4 * lane + q] = static_cast<uint16_t>(ring[j][q] & 0xFFFFu);
            zr[4 * lane + q] = static_cast<uint8_t>(ring[j][q] >> 16);
          }
          mbar_arrive(&sh.p_full[s]);
          ++issued;
#pragma unroll
          for (int q = 0; q < 4; ++q) ring[j][q] = fetch(g + kLookahead, q);
        }
      }
      if (lane == 0)
        for (int i = issued - kSP; i < issued; ++i)
          if (i >= 0) mbar_wait_bounded(&sh.p_full[i % kSP], (i / kSP) & 1);
      __syncwarp();
    } else if (warp == kWarpMma || (kNH == 2 && warp == kWarpMma1)) {
      // MMA stream j: products h = NH g + j, each 8 x (M 128, N NW, K 16).
      if (lane == 0) {
        const int j = warp == kWarpMma ? 0 : 1;
        constexpr uint32_t idesc = instr_desc<kNW>();
        bool ok = true;
        for (int g = 0; g < ng && ok; ++g) {
          const int a = g & 1, s = g % kXG;
          const int h = kNH * g + j;
          const int pb = h % kPBufs;
          ok = wait_or_abort(&ready[s], (g / kXG) & 1, sh, flags) &&
               wait_or_abort(&sh.pe[pb], ((h / kPBufs) & 1) ^ 1, sh, flags);
          if (!ok) break;
          tc_fence_after_sync();
          const uint32_t at = tmem + static_cast<uint32_t>(kACol + 64 * a);
          const uint32_t d = tmem + static_cast<uint32_t>(pb * kNW);
          const uint64_t db0 = sw128_desc(smem_u32(xbuf + s * kSlot + j * kNW * 128));
          const uint64_t db1 = db0 + static_cast<uint64_t>(C::kXStage >> 4);
#pragma unroll
          for (int kk = 0; kk < kGroup / 16; ++kk) {
            // K = 16 per MMA: 8 TMEM columns of A, 32 bytes along a 128-byte X row.
            const uint64_t db = (kk < 4 ? db0 : db1) + 2 * (kk & 3);
            umma_bf16_ts(d, at + static_cast<uint32_t>(8 * kk), db, idesc, kk > 0 ? 1u : 0u);
          }
          umma_commit(&gdone[s]);
        }
        umma_commit(sh.mma_done);
        mbar_wait_bounded(sh.mma_done, 0);  // no MMA in flight past this point
      }
      __syncwarp();
    }
    cluster_arrive_wait();
    cluster_arrive_wait();
  } else if (warp < kWarpFoldTm) {
    // ---------------- unpack: row 32 (w % 4) + lane of every group into TMEM ----------------
    asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;\n" ::"n"(kRegsTmUnpack) : "memory");
    const int q = warp & 3;
    const int row = 32 * q + lane;
    const uint32_t lane_base = tmem + (static_cast<uint32_t>(32 * q) << 16) + kACol;
    for (int g = 0; g < ng; ++g) {
      const int a = g & 1;
      const int sp = g % kSP;
      // A buffer a was last read by the MMAs of group g - 2.
      const int gp = g - 2;
      const bool ok = (gp < 0 || wait_or_abort(&gdone[gp % kXG], (gp / kXG) & 1, sh, flags)) &&
                      wait_or_abort(&sh.p_full[sp], (g / kSP) & 1, sh, flags);
      if (!__all_sync(0xffffffffu, ok)) break;
      tc_fence_after_sync();  // the MMAs that read this A buffer have completed
      const uint8_t* pst = pbuf + sp * p_stage_bytes<B>();
      const uint32_t z = zring[(g % kSRing) * kBM + row];
#pragma unroll
      for (int hh = 0; hh < 2; ++hh) {
        uint32_t w[2][B];
        load_half<B>(pst, row, hh, w);
#pragma unroll
        for (int uu = 0; uu < 2; ++uu) {
          uint32_t pr[16];
          unit_pairs<B>(w[uu], z, pr);
          tmem_st_32x32b_x16(lane_base + static_cast<uint32_t>(64 * a + 16 * (2 * hh + uu)), pr);
        }
      }
      tmem_wait_st();
      tc_fence_before_sync();
      __syncwarp();
      if (lane == 0) {
        mbar_arrive(&ready[g % kXG]);
        mbar_arrive(&sh.p_empty[sp]);
      }
    }
    cluster_arrive_wait();
    cluster_arrive_wait();
  } else {
    // ---------------- fold: acc += s[n, g] * P ----------------
    asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;\n" ::"n"(kRegsTmFold) : "memory");
    const int q = warp & 3;                // TMEM lane quarter this warp may access
    const int part = (warp - kWarpFoldTm) >> 2;  // column block of the tile: [part * kAcc, + kAcc)
    const int row = 32 * q + lane;
    // Buffer of group g for this warp, and its columns inside the buffer.
    const int jh = kNH == 2 ? (part >> 1) : 0;
    const int col0 = kNH == 2 ? (part & 1) * kAcc : part * kAcc;
    float acc[kAcc];
#pragma unroll
    for (int j = 0; j < kAcc; ++j) acc[j] = 0.0f;
    bool ok = true;
    for (int g = 0; g < ng && ok; ++g) {
      const int h = kNH * g + jh;
      const int pb = h % kPBufs;
      ok = __all_sync(0xffffffffu, wait_or_abort(&gdone[g % kXG], (g / kXG) & 1, sh, flags));
      if (!ok) break;
      tc_fence_after_sync();
      const float s = __half2float(__ushort_as_half(sring[(g % kSRing) * kBM + row]));
      const uint32_t base = tmem + (static_cast<uint32_t>(32 * q) << 16) +
                            static_cast<uint32_t>(pb * kNW + col0);
#pragma unroll
      for (int c = 0; c < kAcc / 16; ++c) {
        uint32_t r[16];
        tmem_ld_32x32b_x16(base + 16 * c, r);
        tmem_wait_ld();
#pragma unroll
        for (int i = 0; i < 16; ++i) acc[16 * c + i] = fmaf(s, __uint_as_float(r[i]), acc[16 * c + i]);
      }
      tc_fence_before_sync();
      __syncwarp();
      if (lane == 0) mbar_arrive(&sh.pe[pb]);
    }
    const int n = n0 + row;
    if (kNH == 1 && gridDim.z > 1) {
      // Split K: partial sums to shared memory (the X stages are idle: every
      // MMA has completed), then rank 0 adds the cluster's tiles in rank order.
      float* part_buf = reinterpret_cast<float*>(xbuf);
#pragma unroll
      for (int j = 0; j < kAcc; ++j) part_buf[(part * kAcc + j) * kBM + row] = acc[j];
      cluster_arrive_wait();
      cg::cluster_group cluster = cg::this_cluster();
      if (cluster.block_rank() == 0 && !*sh.abort_flag) {
        const int nz = static_cast<int>(gridDim.z);
        const int t = threadIdx.x - kWarpFoldTm * 32;
        for (int e = t; e < kBM * BN; e += kFoldWarpsTm * 32) {
          float v = part_buf[e];
          for (int c = 1; c < nz; ++c) v += cluster.map_shared_rank(part_buf, c)[e];
          const int nn = n0 + e % kBM, m = m0 + e / kBM;
          if (nn < N && m < M) {
            const int64_t o = static_cast<int64_t>(m) * N + nn;
            if (y_f32)
              static_cast<float*>(Y)[o] = v;
            else
              static_cast<__nv_bfloat16*>(Y)[o] = __float2bfloat16_rn(v);
          }
        }
      }
      cluster_arrive_wait();
    } else if (ok && n < N) {
#pragma unroll
      for (int j = 0; j < kAcc; ++j) {
        const int m = m0 + part * kAcc + j;
        if (m < M) {
          const int64_t o = static_cast<int64_t>(m) * N + n;
          if (y_f32)
            static_cast<float*>(Y)[o] = acc[j];
          else
            static_cast<__nv_bfloat16*>(Y)[o] = __float2bfloat16_rn(acc[j]);
        }
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
template <int B, int BN>
cudaError_t launch_tm(const uint16_t* X, int M, int N, int K, const uint32_t* packed,
                      const uint16_t* scales, const uint8_t* zeros, void* Y, bool y_f32,
                      uint32_t* flags, cudaStream_t stream) {
  using C = CfgTm<B, BN>;
  CUtensorMap tx, tw;
  const CUtensorMapSwizzle swz = B == 8   ? CU_TENSOR_MAP_SWIZZLE_128B
                                 : B == 4 ? CU_TENSOR_MAP_SWIZZLE_64B
                                 : B == 2 ? CU_TENSOR_MAP_SWIZZLE_32B
                                          : CU_TENSOR_MAP_SWIZZLE_NONE;
  if (!encode_tensor_map_2d(&tx, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, X, static_cast<uint64_t>(K),
                            static_cast<uint64_t>(M), static_cast<uint64_t>(K) * 2, kBK, BN,
                            CU_TENSOR_MAP_SWIZZLE_128B) ||
      !encode_tensor_map_2d(&tw, CU_TENSOR_MAP_DATA_TYPE_UINT32, packed,
                            static_cast<uint64_t>(K) * B / 32, static_cast<uint64_t>(N),
                            static_cast<uint64_t>(K) * B / 8, 4 * B, kBM, swz))
    return cudaErrorInvalidValue;
  static SmemAttr smem_attr;  // per template instance
  const cudaError_t e = smem_attr.ensure(gemm_tiled_tm_kernel<B, BN>, C::kSmem);
  if (e != cudaSuccess) return e;
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess) dev = -1;
  const int G = K / kGroup;
  const int row_blocks = (N + kBM - 1) / kBM;
  const int col_blocks = (M + BN - 1) / BN;
  cudaLaunchConfig_t cfg = {};
  cfg.blockDim = dim3(kThreadsTm, 1, 1);
  cfg.dynamicSmemBytes = C::kSmem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 1;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;

  // Narrow tiles (one MMA per group): split K over a cluster of C CTAs, with
  // the largest C (at most 8, each slice keeping at least four groups) for
  // which every cluster of the launch is resident at once -- the occupancy
  // API decides, since cluster placement, not only shared memory, limits
  // residency.
  int C_split = 1;
  if (C::kNH == 1) {
    // Resident clusters per cluster size, per device; filled on first use
    // under a lock, since calls may come from several host threads.
    constexpr int kDevs = 64;
    static std::mutex mu;
    static int max_active[kDevs][kMaxCluster + 1];
    static bool known[kDevs][kMaxCluster + 1];
    const int tiles = row_blocks * col_blocks;
    for (int c = kMaxCluster; c >= 2; --c) {
      if (c > G / 4) continue;
      int active = 0;
      {
        std::lock_guard<std::mutex> lock(mu);
        if (dev < 0 || dev >= kDevs || !known[dev][c]) {
          attr[0].val.clusterDim.z = static_cast<unsigned>(c);
          cfg.gridDim = dim3(1, 1, static_cast<unsigned>(c));
          int n = 0;
          if (cudaOccupancyMaxActiveClusters(&n, gemm_tiled_tm_kernel<B, BN>, &cfg) != cudaSuccess) n = 0;
          cudaGetLastError();
          if (dev >= 0 && dev < kDevs) {
            max_active[dev][c] = n;
            known[dev][c] = true;
          }
          active = n;
        } else {
          active = max_active[dev][c];
        }
      }
      if (tiles <= active) {
        C_split = c;
        break;
      }
    }
  }
  const int per_slice = (G + C_split - 1) / C_split;
  C_split = (G + per_slice - 1) / per_slice;  // no empty slices

  cfg.gridDim = dim3(static_cast<unsigned>(row_blocks), static_cast<unsigned>(col_blocks),
                     static_cast<unsigned>(C_split));
  attr[0].val.clusterDim.z = static_cast<unsigned>(C_split);
  return cudaLaunchKernelEx(&cfg, gemm_tiled_tm_kernel<B, BN>, tx, tw, M, N, K, scales, zeros, Y,
                            y_f32 ? 1 : 0, per_slice, flags);
}

// Tile width: the smallest of 64 / 128 / 256 that covers M, so padding rows
// cost no more than needed.
template <int B>
cudaError_t launch_b(const uint16_t* X, int M, int N, int K, const uint32_t* packed,
                     const uint16_t* scales, const uint8_t* zeros, void* Y, bool y_f32,
                     uint32_t* flags, cudaStream_t stream) {
  if (M <= 64) return launch_tm<B, 64>(X, M, N, K, packed, scales, zeros, Y, y_f32, flags, stream);
  if (M <= 128) return launch_tm<B, 128>(X, M, N, K, packed, scales, zeros, Y, y_f32, flags, stream);
  return launch_tm<B, 256>(X, M, N, K, packed, scales, zeros, Y, y_f32, flags, stream);
}

}  // namespace

cudaError_t launch_gemm_tiled(const uint16_t* X, int64_t M, int64_t N, int64_t K, int bits,
                              const uint32_t* packed, const uint16_t* scales, const uint8_t* zeros,
                              void* Y, bool y_f32, uint32_t* flags, cudaStream_t stream) {
  const int m = static_cast<int>(M), n = static_cast<int>(N), k = static_cast<int>(K);
  switch (bits) {
    case 2: return launch_b<2>(X, m, n, k, packed, scales, zeros, Y, y_f32, flags, stream);
    case 3: return launch_b<3>(X, m, n, k, packed, scales, zeros, Y, y_f32, flags, stream);
    case 4: return launch_b<4>(X, m, n, k, packed, scales, zeros, Y, y_f32, flags, stream);
    case 5: return launch_b<5>(X, m, n, k, packed, scales, zeros, Y, y_f32, flags, stream);
    case 6: return launch_b<6>(X, m, n, k, packed, scales, zeros, Y, y_f32, flags, stream);
    case 7: return launch_b<7>(X, m, n, k, packed, scales, zeros, Y, y_f32, flags, stream);
    case 8: return launch_b<8>(X, m, n, k, packed, scales, zeros, Y, y_f32, flags, stream);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace slq
