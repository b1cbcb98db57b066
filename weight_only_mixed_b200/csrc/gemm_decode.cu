// gemm_decode.cu -- dequantize-GEMM for decode batches (M <= 16) on tcgen05
// with the weight operand in tensor memory.
//
// Y = X W^T, w = s * (q - z) (the weight-only linear layer of the pages'
// serving path; gist.science summary, Key Results "Inference Speedup").  At
// decode sizes the layer must stream the packed weights at HBM speed, and the
// dequantized weights must not go through shared memory: bf16 (q - z) costs
// 4 bytes of shared-memory traffic per weight (write + tensor-core read)
// against b/8 bytes of HBM, which would cap the layer far below HBM rate.  So
// each worker thread owns one weight row -- one TMEM lane -- turns its codes
// into exact bf16 (q - z) in registers and stores them straight into TMEM
// (tcgen05.st); tcgen05.mma reads the A operand from TMEM and the activation
// tile (16 rows, zero-padded) from shared memory.
//
// CTA (256 threads) = 128 weight rows x one K slice:
//   warp 0    TMA producer of packed W (one 128-code group x 128 rows per
//             stage, swizzled); its lanes stage the fp16 scales / uint8 zeros
//             eight groups ahead.
//   warps 1,3 MMA issuers (warp 1 also allocates TMEM): one lane of each
//             issues the four K=16 tcgen05.mma of one k-block of every group
//             into its own two accumulators -- a single issuing thread cannot
//             keep up with decode-sized MMAs, two can.
//   warp 2    X producer: 16-byte cp.async of the 16 x 64 activation tiles
//             (rows >= M zero-filled), four k-blocks ahead.
//   warps 4-7 worker for TMEM lane quarter (warp % 4): dequantize group g into
//             TMEM, then fold group g-1's product, s[n, g-1] * P, into 16 fp32
//             registers (one per activation row).
// The C CTAs of a cluster (1 x 1 x C) take contiguous K slices; their partial
// sums meet through distributed shared memory in rank order.  One
// tcgen05.commit per group (done[g % 4]) releases the A buffer, the X stages
// and the product of group g at once.  Every wait is bounded (SLQ_FLAG_TIMEOUT).
#include <cooperative_groups.h>
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include "dequant.cuh"
#include "internal.h"
#include "ptx.cuh"

namespace cg = cooperative_groups;

namespace slq {
namespace {

using dq::load_unit;
using dq::sw128_desc;
using dq::unit_pairs;

constexpr int kRows = 128;   // weight rows per CTA (MMA M, TMEM lanes)
constexpr int kBN = 16;      // activation rows per MMA (MMA N), M <= 16
constexpr int kBK = 64;      // k per X stage: one 128-byte swizzle atom of bf16
constexpr int kSX = 8;       // X stages
constexpr int kXAhead = 4;   // X k-blocks in flight ahead of consumption
constexpr int kSRing = 16;   // scale / zero ring (groups)
constexpr int kChains = 4;   // independent accumulators per group
constexpr int kThreads = 256;
constexpr int kWarpW = 0, kWarpMma = 1, kWarpX = 2, kWarpMma2 = 3, kWarp0 = 4;
constexpr int kMaxCluster = 8;
// TMEM columns: A buffers (2 x 64: 128 bf16 codes per row, two per column)
// then product buffers (2 x kChains x 16).
constexpr int kColA = 0;
constexpr int kColP = 128;
constexpr int kCols = 256;

template <int B>
constexpr int p_stage_bytes() {
  return kRows * 16 * B;
}

template <int B>
struct Cfg {
  static constexpr int kXStage = kBN * 128;
  static constexpr int kFixed = 1024 /* alignment slack */ + kSX * kXStage +
                                kSRing * kRows * 3 + kRows * kBN * 4 /* split-K partials */ +
                                512 /* barriers, TMEM address, flag */;
  // Two CTAs per SM (the TMEM budget allows two): ~112 KB each.
  static constexpr int kSPRaw = (112 * 1024 - kFixed) / p_stage_bytes<B>();
  static constexpr int kSP = kSPRaw > 8 ? 8 : (kSPRaw < 2 ? 2 : kSPRaw);
  static constexpr int kSmem = kFixed + kSP * p_stage_bytes<B>();
  static_assert(kSmem <= 232448, "shared memory budget");
  static_assert(kSRing >= kSP + 2, "scale ring shorter than the packed-W pipeline");
};

// Instruction descriptor, kind::f16: bf16 A and B (K-major), fp32 D, M = 128, N = 16.
constexpr uint32_t kIdesc = (1u << 4) | (1u << 7) | (1u << 10) |
                            (static_cast<uint32_t>(kBN >> 3) << 17) |
                            (static_cast<uint32_t>(kRows >> 4) << 24);

struct Bars {
  uint64_t* p_full;   // packed stage landed + scales staged
  uint64_t* p_empty;  // packed stage read by the workers
  uint64_t* x_full;   // X stage landed (32 producer lanes)
  uint64_t* a_full;   // A buffer written (4 workers)
  uint64_t* pe;       // product buffer drained (4 workers)
  uint64_t* done;     // MMAs of group g complete (ring of 4)
  uint64_t* mma_done;
  uint32_t* tmem_base;
  volatile int* abort_flag;
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

template <int B>
__global__ void __launch_bounds__(kThreads, 2)
    gemm_decode_kernel(const __grid_constant__ CUtensorMap tmap_w, const uint16_t* __restrict__ X,
                       int M, int N, int K, const uint16_t* __restrict__ scales,
                       const uint8_t* __restrict__ zeros, void* __restrict__ Y, int y_f32,
                       int groups_per_slice, uint32_t* __restrict__ flags) {
  using C = Cfg<B>;
  constexpr int kSP = C::kSP;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw_addr = smem_u32(smem_raw);
  uint8_t* smem = smem_raw + (((raw_addr + 1023u) & ~1023u) - raw_addr);
  uint8_t* xbuf = smem;                                    // [kSX][16 rows][128 B], swizzled
  uint8_t* pbuf = xbuf + kSX * C::kXStage;                 // [kSP][128 rows][16B B]
  uint16_t* sring = reinterpret_cast<uint16_t*>(pbuf + kSP * p_stage_bytes<B>());  // [kSRing][128]
  uint8_t* zring = reinterpret_cast<uint8_t*>(sring + kSRing * kRows);             // [kSRing][128]
  float* part = reinterpret_cast<float*>(zring + kSRing * kRows);                  // [16][128]
  uint64_t* bars = reinterpret_cast<uint64_t*>(part + kRows * kBN);
  Bars sh;
  sh.p_full = bars;
  sh.p_empty = sh.p_full + kSP;
  sh.x_full = sh.p_empty + kSP;
  sh.a_full = sh.x_full + kSX;
  sh.pe = sh.a_full + 2;
  sh.done = sh.pe + 2;
  sh.mma_done = sh.done + 4;
  sh.tmem_base = reinterpret_cast<uint32_t*>(sh.mma_done + 1);
  sh.abort_flag = reinterpret_cast<volatile int*>(sh.tmem_base + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int n0 = blockIdx.x * kRows;
  const int G = K / kGroup;
  const int g_begin = blockIdx.z * groups_per_slice;
  const int g_end = min(G, g_begin + groups_per_slice);
  const int ng = g_end - g_begin;
  const int KB = 2 * ng;

  if (threadIdx.x == 0) {
    for (int i = 0; i < kSP; ++i) {
      mbar_init(&sh.p_full[i], 1 + 32);  // TMA arrival + the producer warp's lanes
      mbar_init(&sh.p_empty[i], 4);
    }
    for (int i = 0; i < kSX; ++i) mbar_init(&sh.x_full[i], 32);
    for (int i = 0; i < 2; ++i) {
      mbar_init(&sh.a_full[i], 4);
      mbar_init(&sh.pe[i], 4);
    }
    for (int i = 0; i < 4; ++i) mbar_init(&sh.done[i], 2);  // one commit per issuer
    mbar_init(sh.mma_done, 2);
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

  float acc[kBN];
#pragma unroll
  for (int j = 0; j < kBN; ++j) acc[j] = 0.0f;
  bool ok = true;

  if (warp == kWarpW) {
    // ---------------- packed-W producer + scale / zero staging ----------------
    // Scale / zero loads run kLookahead groups ahead of their stores; the loop
    // is unrolled by kLookahead so ring slot j is only read once its load,
    // issued kLookahead iterations earlier, has had time to land.
    if (lane == 0) prefetch_tmap(&tmap_w);
    constexpr int kLookahead = 8;
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
        const bool w = wait_or_abort(&sh.p_empty[s], ((g / kSP) & 1) ^ 1, sh, flags);
        if (!__all_sync(0xffffffffu, w)) {
          run = false;
          break;
        }
        if (lane == 0) {
          mbar_arrive_expect_tx(&sh.p_full[s], p_stage_bytes<B>());
          tma_load_2d(pbuf + s * p_stage_bytes<B>(), &tmap_w, &sh.p_full[s], (g_begin + g) * 4 * B, n0);
        }
        uint16_t* sr = sring + (g % kSRing) * kRows;
        uint8_t* zr = zring + (g % kSRing) * kRows;
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
  } else if (warp == kWarpX) {
    // ---------------- X producer: cp.async, rows >= M zero-filled ----------------
    auto copy_kblock = [&](int kb) {
      uint8_t* dst = xbuf + (kb % kSX) * C::kXStage;
      const int64_t k0 = static_cast<int64_t>(2 * g_begin + kb) * kBK;
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const int v = lane + 32 * j;  // 16 rows x 8 chunks of 16 bytes
        const int r = v >> 3, c = v & 7;
        const bool in = r < M;
        const uint16_t* src = in ? X + static_cast<int64_t>(r) * K + k0 + 8 * c : X;
        cp_async_16(dst + r * 128 + ((c ^ (r & 7)) << 4), src, in ? 16u : 0u);
      }
    };
    for (int kb = 0; kb < kXAhead && kb < KB; ++kb) {
      copy_kblock(kb);  // the first stages are free
      cp_async_commit();
    }
    for (int kb = 0; kb < KB && ok; ++kb) {
      const int kn = kb + kXAhead;
      if (kn < KB) {
        bool w = true;
        if (kn >= kSX) {  // the stage held k-block kn - kSX: its group's MMAs must be done
          const int gx = (kn - kSX) >> 1;
          w = wait_or_abort(&sh.done[gx & 3], (gx >> 2) & 1, sh, flags);
        }
        ok = __all_sync(0xffffffffu, w);
        if (ok) copy_kblock(kn);
      }
      cp_async_commit();         // possibly empty: keeps one group per k-block
      cp_async_wait<kXAhead>();  // the group of k-block kb has landed
      fence_proxy_async_smem();
      mbar_arrive(&sh.x_full[kb % kSX]);
    }
    cp_async_wait<0>();
    __syncwarp();
  } else if (warp == kWarpMma || warp == kWarpMma2) {
    // ---------------- MMA issuers: issuer h takes k-block 2g + h ----------------
    // Issuer h writes accumulators 2h and 2h + 1 (two K=16 MMAs each); the
    // four sum to the group's product.
    if (lane == 0) {
      const int h = warp == kWarpMma ? 0 : 1;
      for (int g = 0; g < ng && ok; ++g) {
        const int buf = g & 1;
        const int kb = 2 * g + h;
        ok = wait_or_abort(&sh.pe[buf], ((g >> 1) & 1) ^ 1, sh, flags) &&
             wait_or_abort(&sh.a_full[buf], (g >> 1) & 1, sh, flags) &&
             wait_or_abort(&sh.x_full[kb % kSX], (kb / kSX) & 1, sh, flags);
        if (!ok) break;
        tc_fence_after_sync();
        const uint32_t a = tmem + static_cast<uint32_t>(kColA + buf * 64 + 32 * h);
        const uint32_t d = tmem + static_cast<uint32_t>(kColP + buf * kChains * kBN + 2 * h * kBN);
        const uint64_t bd = sw128_desc(smem_u32(xbuf + (kb % kSX) * C::kXStage));
#pragma unroll
        for (int k = 0; k < 4; ++k)  // K = 16 per MMA: 8 TMEM columns of A, 32 bytes of X
          umma_bf16_ts(d + static_cast<uint32_t>((k & 1) * kBN), a + static_cast<uint32_t>(8 * k),
                       bd + 2 * k, kIdesc, k >= 2 ? 1u : 0u);
        umma_commit(&sh.done[g & 3]);
      }
      umma_commit(sh.mma_done);
      mbar_wait_bounded(sh.mma_done, 0);  // no MMA in flight past this point
    }
    __syncwarp();
  } else if (warp >= kWarp0) {
    // ---------------- workers: TMEM lanes [32q, 32q + 32) ----------------
    const int q = warp & 3;
    const int row = 32 * q + lane;  // weight row n0 + row == TMEM lane
    const uint32_t lane_addr = static_cast<uint32_t>(32 * q) << 16;
    for (int g = 0; g <= ng && ok; ++g) {
      if (g < ng) {
        // ---- dequantize group g into A buffer g % 2 ----
        const int sp = g % kSP;
        ok = (g < 2 || wait_or_abort(&sh.done[(g - 2) & 3], ((g - 2) >> 2) & 1, sh, flags)) &&
             wait_or_abort(&sh.p_full[sp], (g / kSP) & 1, sh, flags);
        ok = __all_sync(0xffffffffu, ok);
        if (!ok) break;
        tc_fence_after_sync();
        const uint8_t* pst = pbuf + sp * p_stage_bytes<B>();
        const uint32_t z = zring[(g % kSRing) * kRows + row];
        const uint32_t a = tmem + lane_addr + static_cast<uint32_t>(kColA + (g & 1) * 64);
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
          mbar_arrive(&sh.a_full[g & 1]);
          mbar_arrive(&sh.p_empty[sp]);
        }
      }
      if (g >= 1) {
        // ---- fold group g-1: acc += s[n, g-1] * (sum of the kChains products) ----
        const int j = g - 1;
        ok = __all_sync(0xffffffffu, wait_or_abort(&sh.done[j & 3], (j >> 2) & 1, sh, flags));
        if (!ok) break;
        tc_fence_after_sync();
        const float s = __half2float(__ushort_as_half(sring[(j % kSRing) * kRows + row]));
        const uint32_t p = tmem + lane_addr + static_cast<uint32_t>(kColP + (j & 1) * kChains * kBN);
        uint32_t r[kChains][16];
#pragma unroll
        for (int c = 0; c < kChains; ++c) tmem_ld_32x32b_x16(p + static_cast<uint32_t>(c * kBN), r[c]);
        tmem_wait_ld();
#pragma unroll
        for (int i = 0; i < kBN; ++i) {
          float v = __uint_as_float(r[0][i]);
#pragma unroll
          for (int c = 1; c < kChains; ++c) v += __uint_as_float(r[c][i]);
          acc[i] = fmaf(s, v, acc[i]);
        }
        tc_fence_before_sync();
        __syncwarp();
        if (lane == 0) mbar_arrive(&sh.pe[j & 1]);
      }
    }
  }

  // ---------------- output ----------------
  auto store = [&](int m, int n, float v) {
    if (n < N && m < M) {
      const int64_t o = static_cast<int64_t>(m) * N + n;
      if (y_f32)
        static_cast<float*>(Y)[o] = v;
      else
        static_cast<__nv_bfloat16*>(Y)[o] = __float2bfloat16_rn(v);
    }
  };
  if (warp >= kWarp0) {
    const int row = 32 * (warp & 3) + lane;
    if (gridDim.z == 1) {
      if (ok)
#pragma unroll
        for (int m = 0; m < kBN; ++m) store(m, n0 + row, acc[m]);
    } else {
#pragma unroll
      for (int m = 0; m < kBN; ++m) part[m * kRows + row] = acc[m];
    }
  }
  __syncwarp();
  if (gridDim.z > 1) {
    cg::cluster_group cluster = cg::this_cluster();
    cluster.sync();  // every CTA's partial sums are complete and visible
    if (cluster.block_rank() == 0) {
      const int nz = static_cast<int>(gridDim.z);
      for (int e = threadIdx.x; e < kRows * kBN; e += kThreads) {
        float v = part[e];
        for (int c = 1; c < nz; ++c) v += cluster.map_shared_rank(part, c)[e];
        store(e / kRows, n0 + e % kRows, v);
      }
    }
    cluster.sync();  // keep every CTA's shared memory alive until rank 0 has read it
  }
  tc_fence_before_sync();
  __syncthreads();
  if (warp == kWarpMma) {
    tc_fence_after_sync();
    tmem_dealloc(tmem, kCols);
  }
}

template <int B>
cudaError_t launch_b(const uint16_t* X, int M, int N, int K, const uint32_t* packed,
                     const uint16_t* scales, const uint8_t* zeros, void* Y, bool y_f32,
                     uint32_t* flags, cudaStream_t stream) {
  using C = Cfg<B>;
  CUtensorMap tw;
  const CUtensorMapSwizzle swz = B == 8   ? CU_TENSOR_MAP_SWIZZLE_128B
                                 : B == 4 ? CU_TENSOR_MAP_SWIZZLE_64B
                                 : B == 2 ? CU_TENSOR_MAP_SWIZZLE_32B
                                          : CU_TENSOR_MAP_SWIZZLE_NONE;
  if (!encode_tensor_map_2d(&tw, CU_TENSOR_MAP_DATA_TYPE_UINT32, packed,
                            static_cast<uint64_t>(K) * B / 32, static_cast<uint64_t>(N),
                            static_cast<uint64_t>(K) * B / 8, 4 * B, kRows, swz))
    return cudaErrorInvalidValue;
  cudaError_t e = cudaFuncSetAttribute(gemm_decode_kernel<B>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, C::kSmem);
  if (e != cudaSuccess) return e;
  e = cudaFuncSetAttribute(gemm_decode_kernel<B>, cudaFuncAttributePreferredSharedMemoryCarveout,
                           static_cast<int>(cudaSharedmemCarveoutMaxShared));
  if (e != cudaSuccess) return e;

  const int G = K / kGroup;
  const int row_blocks = (N + kRows - 1) / kRows;
  cudaLaunchConfig_t cfg = {};
  cfg.blockDim = dim3(kThreads, 1, 1);
  cfg.dynamicSmemBytes = C::kSmem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 1;
  attr[0].val.clusterDim.y = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  // Split K over a cluster of C CTAs so that the launch fills the GPU: the
  // largest C (at most 8, at least four groups per slice) for which all
  // row_blocks * C CTAs are resident at once -- by the per-SM occupancy and by
  // the occupancy API's count of co-resident clusters (cached per device).
  static int cached_dev = -1, slots = 0;
  static int max_active[kMaxCluster + 1];
  int dev = 0;
  e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev != cached_dev) {
    int sms = 0, per_sm = 0;
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, gemm_decode_kernel<B>, kThreads,
                                                      C::kSmem) != cudaSuccess)
      per_sm = 1;
    slots = sms * per_sm;
    for (int c = 2; c <= kMaxCluster; ++c) {
      attr[0].val.clusterDim.z = static_cast<unsigned>(c);
      cfg.gridDim = dim3(1, 1, static_cast<unsigned>(c));
      int n = 0;
      if (cudaOccupancyMaxActiveClusters(&n, gemm_decode_kernel<B>, &cfg) != cudaSuccess) n = 0;
      max_active[c] = n;
    }
    cudaGetLastError();
    cached_dev = dev;
  }
  int C_split = 1;
  for (int c = kMaxCluster; c >= 2; --c) {
    if (c > G / 4) continue;
    if (row_blocks * c <= slots && row_blocks <= max_active[c]) {
      C_split = c;
      break;
    }
  }
  const int per_slice = (G + C_split - 1) / C_split;
  C_split = (G + per_slice - 1) / per_slice;  // no empty slices
  cfg.gridDim = dim3(static_cast<unsigned>(row_blocks), 1, static_cast<unsigned>(C_split));
  attr[0].val.clusterDim.z = static_cast<unsigned>(C_split);
  return cudaLaunchKernelEx(&cfg, gemm_decode_kernel<B>, tw, X, M, N, K, scales, zeros, Y,
                            y_f32 ? 1 : 0, per_slice, flags);
}

}  // namespace

cudaError_t launch_gemm_decode(const uint16_t* X, int64_t M, int64_t N, int64_t K, int bits,
                               const uint32_t* packed, const uint16_t* scales,
                               const uint8_t* zeros, void* Y, bool y_f32, uint32_t* flags,
                               cudaStream_t stream) {
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
