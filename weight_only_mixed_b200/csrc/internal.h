// internal.h -- launchers shared between the C-ABI front end (slq_api.cu) and
// the kernel translation units.  Not part of the public ABI (see include/slq.h).
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <mutex>

namespace slq {

constexpr int kGroup = 128;  // group size along K fixed by the format

// The dynamic shared-memory limit set on one kernel, per device (a function
// attribute belongs to the device's context).  One static instance per
// kernel; safe when launches come from several host threads.
struct SmemAttr {
  std::mutex mu;
  int bytes[64] = {};
  template <typename F>
  cudaError_t ensure(F kernel, int n) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return cudaErrorInvalidDevice;
    std::lock_guard<std::mutex> lock(mu);
    if (dev >= 0 && dev < 64 && bytes[dev] >= n) return cudaSuccess;
    cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, n);
    if (e == cudaSuccess)
      e = cudaFuncSetAttribute(kernel, cudaFuncAttributePreferredSharedMemoryCarveout,
                               static_cast<int>(cudaSharedmemCarveoutMaxShared));
    if (e == cudaSuccess && dev >= 0 && dev < 64) bytes[dev] = n;
    return e;
  }
};

// Flag bits (same values as SLQ_FLAG_* in slq.h).
constexpr uint32_t kFlagNonfinite = 1u;
constexpr uint32_t kFlagScaleOverflow = 2u;
constexpr uint32_t kFlagTimeout = 4u;
constexpr uint32_t kFlagNotPositiveDefinite = 8u;

cudaError_t launch_quantize(const uint16_t* W, int64_t N, int64_t K, int bits,
                            uint32_t* packed, uint16_t* scales, uint8_t* zeros,
                            uint32_t* flags, cudaStream_t stream);

// Encode a 2-D tiled TMA map (inner dimension contiguous); false on failure.
bool encode_tensor_map_2d(CUtensorMap* map, CUtensorMapDataType dtype, const void* base,
                          uint64_t inner, uint64_t outer, uint64_t row_bytes, uint32_t box_inner,
                          uint32_t box_outer, CUtensorMapSwizzle swizzle);

// Decode dequantize-GEMM (M <= 16), the SLQ_GEMM_DECODE path: packed W
// streamed by TMA, dequantized in registers into mma.sync A fragments,
// persistent stream-K over two CTAs per SM with a deterministic fixup.
// `workspace` holds the split tiles' counters and partial sums
// (gemm_decode_workspace_bytes; zero-filled counters on entry and exit).
cudaError_t launch_gemm_decode(const uint16_t* X, int64_t M, int64_t N, int64_t K, int bits,
                               const uint32_t* packed, const uint16_t* scales,
                               const uint8_t* zeros, void* Y, bool y_f32, void* workspace,
                               uint32_t* flags, cudaStream_t stream);

// Workspace bytes of launch_gemm_decode for an [N, K] layer on the current
// device (0 when no row tile is split).
size_t gemm_decode_workspace_bytes(int64_t N, int64_t K, int bits);

// Split-K GEMV for M <= 16 with no workspace: a CTA per 16- or 32-row tile,
// its warps split K, partial tiles added in shared memory.
cudaError_t launch_gemm_gemv(const uint16_t* X, int64_t M, int64_t N, int64_t K, int bits,
                             const uint32_t* packed, const uint16_t* scales, const uint8_t* zeros,
                             void* Y, bool y_f32, uint32_t* flags, cudaStream_t stream);

// One layer of a grouped GEMV launch.
struct GemvCall {
  const uint16_t* X;
  const uint32_t* packed;
  const uint16_t* scales;
  const uint8_t* zeros;
  void* Y;
  int64_t N, K;
  int bits;
};

// Up to gemm_gemv_group_max() layers (any b, N, K; one M <= 16) in one
// launch of the split-K GEMV kernel.
int gemm_gemv_group_max();
cudaError_t launch_gemm_gemv_group(const GemvCall* calls, int count, int64_t M, bool y_f32,
                                   uint32_t* flags, cudaStream_t stream);

// Largest N the decode kernel accepts (the fixed tile-counter region).
int64_t gemm_decode_max_n();

// launch_gemm_decode with its workspace in the library's fixed per-device
// scratch array (gemm_decode_static_scratch_bytes bytes); cudaErrorInvalidValue
// when the layer needs more.
size_t gemm_decode_static_scratch_bytes();
cudaError_t launch_gemm_decode_static(const uint16_t* X, int64_t M, int64_t N, int64_t K, int bits,
                                      const uint32_t* packed, const uint16_t* scales,
                                      const uint8_t* zeros, void* Y, bool y_f32, uint32_t* flags,
                                      cudaStream_t stream);

// Dequantize-GEMM on tcgen05 (TMA + dequant to shared memory + tcgen05.mma
// with TMEM accumulators); the tile width follows M, and K is split over a
// thread-block cluster for narrow tiles.
cudaError_t launch_gemm_tiled(const uint16_t* X, int64_t M, int64_t N, int64_t K, int bits,
                              const uint32_t* packed, const uint16_t* scales,
                              const uint8_t* zeros, void* Y, bool y_f32, uint32_t* flags,
                              cudaStream_t stream);

cudaError_t launch_ear_kl(const uint16_t* a, const uint16_t* b, int64_t T, int64_t V,
                          float temperature, float* ear_tok, float* kl_tok,
                          double* ear_mean, double* kl_mean, uint32_t* flags,
                          cudaStream_t stream);

// Top-K EAR / KL(p_T || q_T) over the K largest reference logits, K <= ear_kl_topk_max().
int ear_kl_topk_max();
cudaError_t launch_ear_kl_topk(const uint16_t* a, const uint16_t* b, int64_t T, int64_t V, int K,
                               float temperature, float* ear_tok, float* kl_tok, double* ear_mean,
                               double* kl_mean, cudaStream_t stream);

// Per-group gamma and the rounding SSE of the asymmetric and symmetric
// continuous b-bit grids; outputs [N, K / 128] fp32.
cudaError_t launch_grid_noise(const uint16_t* W, int64_t N, int64_t K, int bits, float* gamma,
                              float* sse_asym, float* sse_sym, uint32_t* flags, cudaStream_t stream);

// GPTQ encode (binary64, the definition's operation order); workspace of
// gptq_workspace_bytes(N, K) bytes, 16-byte aligned.
size_t gptq_workspace_bytes(int64_t N, int64_t K);
cudaError_t launch_gptq(const uint16_t* W, int64_t N, int64_t K, int bits, const uint16_t* X, int64_t T,
                        double damp, uint32_t* packed, uint16_t* scales, uint8_t* zeros, void* workspace,
                        uint32_t* flags, cudaStream_t stream);

}  // namespace slq
