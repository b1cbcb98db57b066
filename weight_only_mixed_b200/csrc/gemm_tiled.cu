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
// Weights.  Each code is dequantized to bf16_rn(s * (q - z)): the exact
// binary32 product rounded once to bf16, i.e. the weight of the layer's bf16
// fake-quantized copy (the form in which the pages' checkpoints store a
// quantized layer; GitHub README, "4. Build and serve a checkpoint").  With
// the scale inside the weight, one TMEM accumulator runs over the whole K
// range and no per-group rescaling is needed.
//
// Where the time goes, per 128-wide group of a 128 x 256 tile (1024 clocks
// of tensor-core work):
//  - Shared memory (128 bytes per clock per SM).  The dequantized tile goes
//    from registers into TMEM (tcgen05.st) and tcgen05.mma reads A from TMEM,
//    so only the activation tile (written by TMA, read by the MMAs) and the
//    packed codes cross shared memory: ~144 KB per group.
//  - Issue.  One thread issues an MMA every ~60 clocks at best, and a second
//    tcgen05.commit per group costs ~15 % of the tensor core's time; the
//    issuing thread waits once and commits once per group, and each MMA is
//    N = BN wide (128 clocks at N = 256).
//
// Warp roles (384 threads, one CTA per SM):
//   warp 0        TMA producer of X (two 64 k x BN tiles per group).
//   warp 1        TMEM allocator; one lane issues every tcgen05.mma.
//   warp 2        TMA producer of packed W and the scale / zero staging.
//   warp 3        idle.
//   warps 4-11    dequantize: warp w owns TMEM lanes 32 (w % 4) .. + 31 (rows
//                 of W) and half of the group's 128 codes; afterwards they
//                 read the accumulator and store Y.
// Barriers: ready[s] completes when group g's activations have landed (slot
// s = g % kXG of the activation ring, both 64-k stages) and its A tile is in
// TMEM (A buffer s); the MMA thread commits group g to gdone[s], which frees
// the activation slot and the A buffer.  Every wait gives up after 2 s of
// wall time, raises SLQ_FLAG_TIMEOUT and lets the CTA drain its copies and
// free TMEM.  Narrow tiles (BN <= 128) may split K over a thread-block
// cluster; the partial tiles are added in rank order through distributed
// shared memory.
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
using dq::unit_scaled;

constexpr int kBM = 128;      // W rows per tile (MMA M)
constexpr int kBK = 64;       // k per X stage: one 128-byte swizzle atom of bf16
constexpr int kSRing = 16;    // scale / zero ring (groups)
constexpr int kMaxCluster = 8;
constexpr int kWarpX = 0, kWarpMma = 1, kWarpW = 2;
constexpr int kUnpackWarps = 8;
constexpr int kWarpUnpack0 = 4;
constexpr int kThreads = (kWarpUnpack0 + kUnpackWarps) * 32;
constexpr int kACol = 256;    // first TMEM column of the A buffers (the accumulator is below)
constexpr int kTmemCols = 512;

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

// Stage counts and the shared-memory budget: one CTA per SM, up to 227 KB;
// what the activation ring leaves goes to packed-W stages.
template <int B, int BN>
struct Cfg {
  static constexpr int kXG = BN == 256 ? 2 : 4;  // activation ring / A buffers, in groups
  static constexpr int kXStage = BN * 128;       // one 64-k stage
  static constexpr int kSlot = 2 * kXStage;      // one group
  static constexpr int kFixed = 1024 /* alignment slack */ + kXG * kSlot + kSRing * kBM * 3 +
                                512 /* barriers, TMEM address, flag */;
  static constexpr int kBudget = 227 * 1024;
  static constexpr int kSPRaw = (kBudget - kFixed) / p_stage_bytes<B>();
  static constexpr int kSP = kSPRaw > 8 ? 8 : (kSPRaw < 2 ? 2 : kSPRaw);
  // More than half of the SM's shared memory, so one CTA per SM (TMEM holds
  // one 512-column allocation).
  static constexpr int kSmem = (kFixed + kSP * p_stage_bytes<B>()) > 120 * 1024
                                   ? kFixed + kSP * p_stage_bytes<B>()
                                   : 120 * 1024;
  static_assert(kSmem <= 232448, "shared memory budget");
  static_assert(BN <= kACol, "accumulator below the A buffers");
  static_assert(kACol + 64 * kXG <= kTmemCols, "A buffers fit in TMEM");
  // The producer refills scale slot g % kSRing once the dequant of group
  // g - kSP is done; the dequant warps are the only readers.
  static_assert(kSRing >= kSP + 1, "scale ring shorter than the packed-W pipeline");
  static_assert(kXG * kSlot >= kBM * BN * 4, "the activation ring doubles as the split-K buffer");
};

struct Bars {
  uint64_t* ready;    // [kXG] X landed + A written
  uint64_t* gdone;    // [kXG] the group's MMAs completed
  uint64_t* p_full;   // [kSP]
  uint64_t* p_empty;  // [kSP]
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

template <int B, int BN>
__global__ void __launch_bounds__(kThreads, 1)
    gemm_tiled_kernel(const __grid_constant__ CUtensorMap tmap_x,
                      const __grid_constant__ CUtensorMap tmap_w, int M, int N, int K,
                      const uint16_t* __restrict__ scales, const uint8_t* __restrict__ zeros,
                      void* __restrict__ Y, int y_f32, int groups_per_slice,
                      uint32_t* __restrict__ flags) {
  using C = Cfg<B, BN>;
  constexpr int kSP = C::kSP, kXG = C::kXG, kSlot = C::kSlot;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw_addr = smem_u32(smem_raw);
  uint8_t* smem = smem_raw + (((raw_addr + 1023u) & ~1023u) - raw_addr);
  uint8_t* xbuf = smem;
  uint8_t* pbuf = xbuf + kXG * kSlot;
  uint16_t* sring = reinterpret_cast<uint16_t*>(pbuf + kSP * p_stage_bytes<B>());  // [kSRing][128]
  uint8_t* zring = reinterpret_cast<uint8_t*>(sring + kSRing * kBM);                // [kSRing][128]
  uint64_t* bars = reinterpret_cast<uint64_t*>(zring + kSRing * kBM);
  Bars sh;
  sh.ready = bars;
  sh.gdone = sh.ready + kXG;
  sh.p_full = sh.gdone + kXG;
  sh.p_empty = sh.p_full + kSP;
  sh.mma_done = sh.p_empty + kSP;
  sh.tmem_base = reinterpret_cast<uint32_t*>(sh.mma_done + 1);
  sh.abort_flag = reinterpret_cast<volatile int*>(sh.tmem_base + 1);

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
      mbar_init(&sh.ready[i], 1 + kUnpackWarps);  // X producer (expect_tx) + dequant warps
      mbar_init(&sh.gdone[i], 1);                 // tcgen05.commit
    }
    for (int i = 0; i < kSP; ++i) {
      mbar_init(&sh.p_full[i], 1 + 32);  // TMA arrival + the producer warp's lanes
      mbar_init(&sh.p_empty[i], kUnpackWarps);
    }
    mbar_init(sh.mma_done, 1);
    *sh.abort_flag = 0;
    fence_mbarrier_init();
  }
  __syncwarp();
  if (warp == kWarpMma) {
    tmem_alloc(sh.tmem_base, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before_sync();
  __syncthreads();
  tc_fence_after_sync();
  const uint32_t tmem = *sh.tmem_base;

  if (warp == kWarpX) {
    // ---------------- X producer (TMA): group g into slot g % kXG ----------------
    if (lane == 0) {
      prefetch_tmap(&tmap_x);
      int issued = 0;
      for (int g = 0; g < ng; ++g) {
        const int s = g % kXG;
        // The slot was last read by the MMAs of group g - kXG.
        if (g >= kXG && !wait_or_abort(&sh.gdone[s], ((g / kXG) - 1) & 1, sh, flags)) break;
        mbar_arrive_expect_tx(&sh.ready[s], kSlot);
        tma_load_2d(xbuf + s * kSlot, &tmap_x, &sh.ready[s], (2 * (g_begin + g)) * kBK, m0);
        tma_load_2d(xbuf + s * kSlot + C::kXStage, &tmap_x, &sh.ready[s],
                    (2 * (g_begin + g) + 1) * kBK, m0);
        ++issued;
      }
      // Drain: every issued copy must land before the CTA may exit.
      for (int i = issued - kXG; i < issued; ++i)
        if (i >= 0) mbar_wait_bounded(&sh.ready[i % kXG], (i / kXG) & 1);
    }
    __syncwarp();
  } else if (warp == kWarpW) {
    // ---------------- packed-W producer + scale / zero staging ----------------
    // Lane l stages rows 4l..4l+3.  Scale / zero loads are issued kLookahead
    // groups before they are stored, so their latency overlaps the ring.
    if (lane == 0) prefetch_tmap(&tmap_w);
    constexpr int kLookahead = 4;
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
          tma_load_2d(pbuf + s * p_stage_bytes<B>(), &tmap_w, &sh.p_full[s], (g_begin + g) * 4 * B, n0);
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
  } else if (warp == kWarpMma) {
    // ---------------- MMA issuer: group g, 8 x (M 128, N BN, K 16) into D ----------------
    if (lane == 0) {
      constexpr uint32_t idesc = instr_desc<BN>();
      bool ok = true;
      for (int g = 0; g < ng && ok; ++g) {
        const int s = g % kXG;
        ok = wait_or_abort(&sh.ready[s], (g / kXG) & 1, sh, flags);
        if (!ok) break;
        tc_fence_after_sync();
        const uint32_t at = tmem + static_cast<uint32_t>(kACol + 64 * s);
        const uint64_t db0 = sw128_desc(smem_u32(xbuf + s * kSlot));
        const uint64_t db1 = db0 + static_cast<uint64_t>(C::kXStage >> 4);
#pragma unroll
        for (int kk = 0; kk < kGroup / 16; ++kk) {
          // K = 16 per MMA: 8 TMEM columns of A, 32 bytes along a 128-byte X row.
          const uint64_t db = (kk < 4 ? db0 : db1) + 2 * (kk & 3);
          umma_bf16_ts(tmem, at + static_cast<uint32_t>(8 * kk), db, idesc, (g | kk) ? 1u : 0u);
        }
        umma_commit(&sh.gdone[s]);
      }
      umma_commit(sh.mma_done);
      mbar_wait_bounded(sh.mma_done, 0);  // no MMA in flight past this point
    }
    __syncwarp();
  } else if (warp >= kWarpUnpack0) {
    // ---------------- dequantize: row 32 (w % 4) + lane, codes [64 hk, 64 hk + 64) ----------------
    const int q = warp & 3;
    const int hk = (warp - kWarpUnpack0) >> 2;
    const int row = 32 * q + lane;
    const uint32_t lane_base = tmem + (static_cast<uint32_t>(32 * q) << 16);
    bool ok = true;
    for (int g = 0; g < ng; ++g) {
      const int s = g % kXG;
      const int sp = g % kSP;
      // A buffer s was last read by the MMAs of group g - kXG.
      ok = (g < kXG || wait_or_abort(&sh.gdone[s], ((g / kXG) - 1) & 1, sh, flags)) &&
           wait_or_abort(&sh.p_full[sp], (g / kSP) & 1, sh, flags);
      if (!__all_sync(0xffffffffu, ok)) {
        ok = false;
        break;
      }
      tc_fence_after_sync();  // the MMAs that read this A buffer have completed
      const uint8_t* pst = pbuf + sp * p_stage_bytes<B>();
      const uint32_t z = zring[(g % kSRing) * kBM + row];
      const float sc = __half2float(__ushort_as_half(sring[(g % kSRing) * kBM + row]));
      uint32_t w[2][B];
      load_half<B>(pst, row, hk, w);
#pragma unroll
      for (int uu = 0; uu < 2; ++uu) {
        uint32_t pr[16];
        unit_scaled<B>(w[uu], z, sc, pr);
        tmem_st_32x32b_x16(lane_base + static_cast<uint32_t>(kACol + 64 * s + 32 * hk + 16 * uu), pr);
      }
      tmem_wait_st();
      tc_fence_before_sync();
      __syncwarp();
      if (lane == 0) {
        mbar_arrive(&sh.ready[s]);
        mbar_arrive(&sh.p_empty[sp]);
      }
    }

    // ---- epilogue: thread owns row n, columns [hk * BN/2, + BN/2) of the tile ----
    ok = __all_sync(0xffffffffu, ok && wait_or_abort(sh.mma_done, 0, sh, flags));
    tc_fence_after_sync();
    constexpr int kHalf = BN / 2;
    const int n = n0 + row;
    const uint32_t dbase = lane_base + static_cast<uint32_t>(hk * kHalf);
    if (gridDim.z > 1) {
      // Split K: partial sums to shared memory (the activation ring is idle:
      // every MMA has completed), then rank 0 adds the cluster's tiles in
      // rank order.
      float* part = reinterpret_cast<float*>(xbuf);
#pragma unroll 1
      for (int c = 0; c < kHalf / 16; ++c) {
        uint32_t r[16];
        tmem_ld_32x32b_x16(dbase + 16 * c, r);
        tmem_wait_ld();
#pragma unroll
        for (int i = 0; i < 16; ++i) part[(hk * kHalf + 16 * c + i) * kBM + row] = __uint_as_float(r[i]);
      }
    } else if (ok) {  // warp-uniform: tcgen05.ld is a whole-warp instruction
#pragma unroll 1
      for (int c = 0; c < kHalf / 16; ++c) {
        uint32_t r[16];
        tmem_ld_32x32b_x16(dbase + 16 * c, r);
        tmem_wait_ld();
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          const int m = m0 + hk * kHalf + 16 * c + i;
          if (m < M && n < N) {
            const int64_t o = static_cast<int64_t>(m) * N + n;
            if (y_f32)
              static_cast<float*>(Y)[o] = __uint_as_float(r[i]);
            else
              static_cast<__nv_bfloat16*>(Y)[o] = __float2bfloat16_rn(__uint_as_float(r[i]));
          }
        }
      }
    }
  }

  if (gridDim.z > 1) {
    cg::cluster_group cluster = cg::this_cluster();
    cluster.sync();  // every CTA's partial sums are complete and visible
    if (cluster.block_rank() == 0 && !*sh.abort_flag) {
      const float* part = reinterpret_cast<const float*>(xbuf);
      const int nz = static_cast<int>(gridDim.z);
      for (int e = threadIdx.x; e < kBM * BN; e += kThreads) {
        float v = part[e];
        for (int c = 1; c < nz; ++c) v += cluster.map_shared_rank(part, c)[e];
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
    cluster.sync();  // keep every CTA's shared memory alive until rank 0 has read it
  }
  tc_fence_before_sync();
  __syncthreads();
  if (warp == kWarpMma) {
    tc_fence_after_sync();
    tmem_dealloc(tmem, kTmemCols);
  }
}

// ---------------------------------------------------------------------------
// Host side
// ---------------------------------------------------------------------------
template <int B, int BN>
cudaError_t launch_cfg(const uint16_t* X, int M, int N, int K, const uint32_t* packed,
                       const uint16_t* scales, const uint8_t* zeros, void* Y, bool y_f32,
                       uint32_t* flags, cudaStream_t stream) {
  using C = Cfg<B, BN>;
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
  const cudaError_t e = smem_attr.ensure(gemm_tiled_kernel<B, BN>, C::kSmem);
  if (e != cudaSuccess) return e;
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess) dev = -1;
  const int G = K / kGroup;
  const int row_blocks = (N + kBM - 1) / kBM;
  const int col_blocks = (M + BN - 1) / BN;
  cudaLaunchConfig_t cfg = {};
  cfg.blockDim = dim3(kThreads, 1, 1);
  cfg.dynamicSmemBytes = C::kSmem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 1;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;

  // Narrow tiles: split K over a cluster of C CTAs, with
  // the largest C (at most 8, each slice keeping at least four groups) for
  // which every cluster of the launch is resident at once -- the occupancy
  // API decides, since cluster placement, not only shared memory, limits
  // residency.
  int C_split = 1;
  if (BN <= 128) {
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
          if (cudaOccupancyMaxActiveClusters(&n, gemm_tiled_kernel<B, BN>, &cfg) != cudaSuccess) n = 0;
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
  return cudaLaunchKernelEx(&cfg, gemm_tiled_kernel<B, BN>, tx, tw, M, N, K, scales, zeros, Y,
                            y_f32 ? 1 : 0, per_slice, flags);
}

// Tile width: the smallest of 64 / 128 / 256 that covers M, so padding rows
// cost no more than needed.
template <int B>
cudaError_t launch_b(const uint16_t* X, int M, int N, int K, const uint32_t* packed,
                     const uint16_t* scales, const uint8_t* zeros, void* Y, bool y_f32,
                     uint32_t* flags, cudaStream_t stream) {
  if (M <= 64) return launch_cfg<B, 64>(X, M, N, K, packed, scales, zeros, Y, y_f32, flags, stream);
  if (M <= 128) return launch_cfg<B, 128>(X, M, N, K, packed, scales, zeros, Y, y_f32, flags, stream);
  return launch_cfg<B, 256>(X, M, N, K, packed, scales, zeros, Y, y_f32, flags, stream);
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
