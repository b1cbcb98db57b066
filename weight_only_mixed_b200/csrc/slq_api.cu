// slq_api.cu -- the C ABI (include/slq.h): argument validation, device check,
// kernel selection.  Every argument error is caught here, on the host, before
// any CUDA call; the kernels themselves assume valid arguments.
#include <cuda_runtime.h>

#include <cmath>
#include <cstdint>
#include <mutex>

#include "../../include/slq.h"
#include "internal.h"

namespace {

constexpr int64_t kMaxDim = (int64_t{1} << 31) - 1;
constexpr int64_t kMaxElems = int64_t{1} << 40;

bool aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

struct Range {
  uintptr_t lo, hi;  // [lo, hi)
};

Range range_of(const void* p, int64_t bytes) {
  const uintptr_t b = reinterpret_cast<uintptr_t>(p);
  return Range{b, b + static_cast<uintptr_t>(bytes)};
}

bool overlap(Range x, Range y) { return x.lo < y.hi && y.lo < x.hi && x.hi > x.lo && y.hi > y.lo; }

// Every output range must be disjoint from every other range.
bool disjoint(const Range* outs, int n_out, const Range* ins, int n_in) {
  for (int i = 0; i < n_out; ++i) {
    for (int j = 0; j < n_in; ++j)
      if (overlap(outs[i], ins[j])) return false;
    for (int j = i + 1; j < n_out; ++j)
      if (overlap(outs[i], outs[j])) return false;
  }
  return true;
}

// CC 10.0 only.  The answer is cached per device ordinal.
slq_status check_device() {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0) {
    cudaGetLastError();
    return SLQ_ERR_UNSUPPORTED_DEVICE;
  }
  static std::mutex mu;
  static int cached[64];
  static bool init = false;
  std::lock_guard<std::mutex> lock(mu);
  if (!init) {
    for (int& c : cached) c = -1;
    init = true;
  }
  if (dev < 64 && cached[dev] >= 0) return cached[dev] ? SLQ_OK : SLQ_ERR_UNSUPPORTED_DEVICE;
  int major = 0, minor = 0;
  if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess) {
    cudaGetLastError();
    return SLQ_ERR_UNSUPPORTED_DEVICE;
  }
  const bool ok = (major == 10 && minor == 0);
  if (dev < 64) cached[dev] = ok ? 1 : 0;
  return ok ? SLQ_OK : SLQ_ERR_UNSUPPORTED_DEVICE;
}

slq_status from_cuda(cudaError_t e) { return e == cudaSuccess ? SLQ_OK : SLQ_ERR_CUDA; }

bool valid_bits(int bits) { return bits >= 2 && bits <= 8; }

bool valid_k(int64_t K) { return K >= slq::kGroup && K % slq::kGroup == 0 && K <= kMaxDim; }

bool product_ok(int64_t a, int64_t b) { return a == 0 || b <= kMaxElems / a; }

// Workspace of the kernel `path` selects (only the stream-K decode kernel
// uses one; AUTO never selects it).
size_t workspace_needed(int64_t M, int64_t N, int64_t K, int bits, slq_gemm_path path) {
  return (path == SLQ_GEMM_DECODE && M >= 1 && M <= 16 && N >= 1)
             ? slq::gemm_decode_workspace_bytes(N, K, bits)
             : 0;
}

slq_status validate_gemm(const void* X, int64_t M, int64_t N, int64_t K, int bits,
                         const uint32_t* packed, const void* scales, const uint8_t* zeros,
                         void* Y, slq_dtype y_dtype, slq_gemm_path path, void* workspace,
                         size_t workspace_bytes, uint32_t* flags) {
  if (M < 0 || N < 0 || M > kMaxDim || N > kMaxDim || !valid_k(K) || !valid_bits(bits))
    return SLQ_ERR_INVALID_ARGUMENT;
  if (!product_ok(M, K) || !product_ok(N, K) || !product_ok(M, N)) return SLQ_ERR_INVALID_ARGUMENT;
  if (y_dtype != SLQ_DTYPE_BF16 && y_dtype != SLQ_DTYPE_F32) return SLQ_ERR_INVALID_ARGUMENT;
  if (M == 0 || N == 0) return SLQ_OK;
  if (!X || !packed || !scales || !zeros || !Y) return SLQ_ERR_INVALID_ARGUMENT;
  if (!aligned(X, 16) || !aligned(packed, 16) || !aligned(Y, 16) || !aligned(scales, 2) ||
      (flags && !aligned(flags, 4)))
    return SLQ_ERR_INVALID_ARGUMENT;
  if (path == SLQ_GEMM_DECODE && N > slq::gemm_decode_max_n())
    return SLQ_ERR_INVALID_ARGUMENT;
  const size_t need = workspace_needed(M, N, K, bits, path);
  if (need > 0 && (!workspace || workspace_bytes < need || !aligned(workspace, 256)))
    return SLQ_ERR_INVALID_ARGUMENT;
  const int64_t G = K / slq::kGroup;
  const Range ins[4] = {range_of(X, M * K * 2), range_of(packed, N * K * bits / 8),
                        range_of(scales, N * G * 2), range_of(zeros, N * G)};
  const Range outs[3] = {range_of(Y, M * N * (y_dtype == SLQ_DTYPE_F32 ? 4 : 2)),
                         range_of(flags, flags ? 4 : 0),
                         range_of(workspace, static_cast<int64_t>(need))};
  if (!disjoint(outs, 3, ins, 4)) return SLQ_ERR_INVALID_ARGUMENT;
  return SLQ_OK;
}

}  // namespace

extern "C" {

int slq_version(void) { return 100; }

const char* slq_status_string(slq_status status) {
  switch (status) {
    case SLQ_OK: return "SLQ_OK";
    case SLQ_ERR_INVALID_ARGUMENT: return "SLQ_ERR_INVALID_ARGUMENT";
    case SLQ_ERR_UNSUPPORTED_DEVICE: return "SLQ_ERR_UNSUPPORTED_DEVICE (needs CC 10.0 / sm_100a)";
    case SLQ_ERR_CUDA: return "SLQ_ERR_CUDA";
    case SLQ_ERR_TIMEOUT: return "SLQ_ERR_TIMEOUT";
  }
  return "unknown slq_status";
}

size_t slq_packed_words(int64_t N, int64_t K, int bits) {
  if (N < 0 || N > kMaxDim || !valid_k(K) || !valid_bits(bits) || !product_ok(N, K)) return 0;
  return static_cast<size_t>(N * K / 32 * bits);
}

slq_gemm_path slq_gemm_select(int64_t M, int64_t N, int64_t K, int bits) {
  (void)N;
  (void)K;
  (void)bits;
  return M <= 16 ? SLQ_GEMM_GEMV : SLQ_GEMM_TILED;
}

slq_status slq_quantize(const void* W_bf16, int64_t N, int64_t K, int bits, uint32_t* packed,
                        void* scales_f16, uint8_t* zeros, uint32_t* flags, void* stream) {
  if (N < 0 || N > kMaxDim || !valid_k(K) || !valid_bits(bits) || !product_ok(N, K))
    return SLQ_ERR_INVALID_ARGUMENT;
  if (N == 0) return SLQ_OK;
  if (!W_bf16 || !packed || !scales_f16 || !zeros) return SLQ_ERR_INVALID_ARGUMENT;
  if (!aligned(W_bf16, 16) || !aligned(packed, 16) || !aligned(scales_f16, 2) ||
      (flags && !aligned(flags, 4)))
    return SLQ_ERR_INVALID_ARGUMENT;
  const int64_t G = K / slq::kGroup;
  const Range ins[1] = {range_of(W_bf16, N * K * 2)};
  const Range outs[4] = {range_of(packed, N * K * bits / 8), range_of(scales_f16, N * G * 2),
                         range_of(zeros, N * G), range_of(flags, flags ? 4 : 0)};
  if (!disjoint(outs, 4, ins, 1)) return SLQ_ERR_INVALID_ARGUMENT;
  const slq_status dev = check_device();
  if (dev != SLQ_OK) return dev;
  return from_cuda(slq::launch_quantize(static_cast<const uint16_t*>(W_bf16), N, K, bits, packed,
                                        static_cast<uint16_t*>(scales_f16), zeros, flags,
                                        static_cast<cudaStream_t>(stream)));
}

size_t slq_gemm_workspace_bytes(int64_t M, int64_t N, int64_t K, int bits) {
  if (M < 0 || N < 0 || M > kMaxDim || N > kMaxDim || !valid_k(K) || !valid_bits(bits) ||
      !product_ok(N, K))
    return 0;
  return M <= 16 ? workspace_needed(M, N, K, bits, SLQ_GEMM_DECODE) : 0;
}

slq_status slq_gemm_ex(const void* X_bf16, int64_t M, int64_t N, int64_t K, int bits,
                       const uint32_t* packed, const void* scales_f16, const uint8_t* zeros,
                       void* Y, slq_dtype y_dtype, slq_gemm_path path, void* workspace,
                       size_t workspace_bytes, uint32_t* flags, void* stream) {
  if (path != SLQ_GEMM_AUTO && path != SLQ_GEMM_DECODE && path != SLQ_GEMM_TILED &&
      path != SLQ_GEMM_GEMV)
    return SLQ_ERR_INVALID_ARGUMENT;
  if ((path == SLQ_GEMM_DECODE || path == SLQ_GEMM_GEMV) && M > 16) return SLQ_ERR_INVALID_ARGUMENT;
  const slq_status v = validate_gemm(X_bf16, M, N, K, bits, packed, scales_f16, zeros, Y, y_dtype,
                                     path, workspace, workspace_bytes, flags);
  if (v != SLQ_OK) return v;
  if (M == 0 || N == 0) return SLQ_OK;
  const slq_status dev = check_device();
  if (dev != SLQ_OK) return dev;
  if (path == SLQ_GEMM_AUTO) path = slq_gemm_select(M, N, K, bits);
  const bool f32 = (y_dtype == SLQ_DTYPE_F32);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const uint16_t* X = static_cast<const uint16_t*>(X_bf16);
  const uint16_t* sc = static_cast<const uint16_t*>(scales_f16);
  if (path == SLQ_GEMM_GEMV)
    return from_cuda(slq::launch_gemm_gemv(X, M, N, K, bits, packed, sc, zeros, Y, f32, flags, s));
  if (path == SLQ_GEMM_DECODE)
    return from_cuda(
        slq::launch_gemm_decode(X, M, N, K, bits, packed, sc, zeros, Y, f32, workspace, flags, s));
  return from_cuda(slq::launch_gemm_tiled(X, M, N, K, bits, packed, sc, zeros, Y, f32, flags, s));
}

slq_status slq_gemm(const void* X_bf16, int64_t M, int64_t N, int64_t K, int bits,
                    const uint32_t* packed, const void* scales_f16, const uint8_t* zeros, void* Y,
                    slq_dtype y_dtype, uint32_t* flags, void* stream) {
  return slq_gemm_ex(X_bf16, M, N, K, bits, packed, scales_f16, zeros, Y, y_dtype, SLQ_GEMM_AUTO,
                     nullptr, 0, flags, stream);
}

int slq_gemm_group_max(void) { return slq::gemm_gemv_group_max(); }

slq_status slq_gemm_group(const slq_gemm_layer* layers, int count, int64_t M, slq_dtype y_dtype,
                          uint32_t* flags, void* stream) {
  if (!layers || count < 1 || count > slq::gemm_gemv_group_max() || M < 0 || M > 16)
    return SLQ_ERR_INVALID_ARGUMENT;
  slq::GemvCall calls[16];
  Range ins[16 * 4], outs[16];
  int n = 0;
  for (int i = 0; i < count; ++i) {
    const slq_gemm_layer& L = layers[i];
    const slq_status v = validate_gemm(L.X_bf16, M, L.N, L.K, L.bits, L.packed, L.scales_f16,
                                       L.zeros, L.Y, y_dtype, SLQ_GEMM_GEMV, nullptr, 0, flags);
    if (v != SLQ_OK) return v;
    if (M == 0 || L.N == 0) continue;
    const int64_t G = L.K / slq::kGroup;
    ins[4 * n + 0] = range_of(L.X_bf16, M * L.K * 2);
    ins[4 * n + 1] = range_of(L.packed, L.N * L.K * L.bits / 8);
    ins[4 * n + 2] = range_of(L.scales_f16, L.N * G * 2);
    ins[4 * n + 3] = range_of(L.zeros, L.N * G);
    outs[n] = range_of(L.Y, M * L.N * (y_dtype == SLQ_DTYPE_F32 ? 4 : 2));
    calls[n] = slq::GemvCall{static_cast<const uint16_t*>(L.X_bf16), L.packed,
                             static_cast<const uint16_t*>(L.scales_f16), L.zeros, L.Y, L.N, L.K,
                             L.bits};
    ++n;
  }
  if (n == 0) return SLQ_OK;
  if (!disjoint(outs, n, ins, 4 * n)) return SLQ_ERR_INVALID_ARGUMENT;
  if (flags) {
    const Range f = range_of(flags, 4);
    if (!disjoint(&f, 1, ins, 4 * n) || !disjoint(&f, 1, outs, n)) return SLQ_ERR_INVALID_ARGUMENT;
  }
  const slq_status dev = check_device();
  if (dev != SLQ_OK) return dev;
  return from_cuda(slq::launch_gemm_gemv_group(calls, n, M, y_dtype == SLQ_DTYPE_F32, flags,
                                               static_cast<cudaStream_t>(stream)));
}

slq_status slq_gemm_decode_static(const void* X_bf16, int64_t M, int64_t N, int64_t K, int bits,
                                  const uint32_t* packed, const void* scales_f16,
                                  const uint8_t* zeros, void* Y, slq_dtype y_dtype,
                                  uint32_t* flags, void* stream) {
  if (M > 16 || N > slq::gemm_decode_max_n()) return SLQ_ERR_INVALID_ARGUMENT;
  // Validated as a call without a workspace; the size limit is checked below.
  const slq_status v = validate_gemm(X_bf16, M, N, K, bits, packed, scales_f16, zeros, Y, y_dtype,
                                     SLQ_GEMM_TILED, nullptr, 0, flags);
  if (v != SLQ_OK) return v;
  if (M == 0 || N == 0) return SLQ_OK;
  if (slq::gemm_decode_workspace_bytes(N, K, bits) > slq::gemm_decode_static_scratch_bytes())
    return SLQ_ERR_INVALID_ARGUMENT;
  const slq_status dev = check_device();
  if (dev != SLQ_OK) return dev;
  return from_cuda(slq::launch_gemm_decode_static(
      static_cast<const uint16_t*>(X_bf16), M, N, K, bits, packed,
      static_cast<const uint16_t*>(scales_f16), zeros, Y, y_dtype == SLQ_DTYPE_F32, flags,
      static_cast<cudaStream_t>(stream)));
}

namespace {
// Shared argument checks of slq_ear_kl and slq_ear_kl_topk.
slq_status validate_ear(const void* logits_p_bf16, const void* logits_q_bf16, int64_t T, int64_t V,
                        float temperature, float* ear_tok, float* kl_tok, double* ear_mean,
                        double* kl_mean, uint32_t* flags) {
  if (T < 0 || T > kMaxDim || V < 1 || V > kMaxDim || !product_ok(T, V))
    return SLQ_ERR_INVALID_ARGUMENT;
  if (!std::isfinite(temperature) || !(temperature > 0.0f)) return SLQ_ERR_INVALID_ARGUMENT;
  if (T == 0) return SLQ_OK;
  if (!logits_p_bf16 || !logits_q_bf16 || !ear_tok || !kl_tok) return SLQ_ERR_INVALID_ARGUMENT;
  if (!aligned(logits_p_bf16, 16) || !aligned(logits_q_bf16, 16) || !aligned(ear_tok, 4) ||
      !aligned(kl_tok, 4) || (ear_mean && !aligned(ear_mean, 8)) ||
      (kl_mean && !aligned(kl_mean, 8)) || (flags && !aligned(flags, 4)))
    return SLQ_ERR_INVALID_ARGUMENT;
  const Range ins[2] = {range_of(logits_p_bf16, T * V * 2), range_of(logits_q_bf16, T * V * 2)};
  const Range outs[5] = {range_of(ear_tok, T * 4), range_of(kl_tok, T * 4),
                         range_of(ear_mean, ear_mean ? 8 : 0), range_of(kl_mean, kl_mean ? 8 : 0),
                         range_of(flags, flags ? 4 : 0)};
  if (!disjoint(outs, 5, ins, 2)) return SLQ_ERR_INVALID_ARGUMENT;
  return SLQ_OK;
}
}  // namespace

int slq_ear_kl_topk_max(void) { return slq::ear_kl_topk_max(); }

slq_status slq_ear_kl_topk(const void* logits_p_bf16, const void* logits_q_bf16, int64_t T,
                           int64_t V, int top_k, float temperature, float* ear_tok, float* kl_tok,
                           double* ear_mean, double* kl_mean, uint32_t* flags, void* stream) {
  if (top_k < 1 || top_k > slq::ear_kl_topk_max() || top_k > V || V > 0x7fffffff)
    return SLQ_ERR_INVALID_ARGUMENT;
  const slq_status v = validate_ear(logits_p_bf16, logits_q_bf16, T, V, temperature, ear_tok,
                                    kl_tok, ear_mean, kl_mean, flags);
  if (v != SLQ_OK || T == 0) return v;
  const slq_status dev = check_device();
  if (dev != SLQ_OK) return dev;
  return from_cuda(slq::launch_ear_kl_topk(
      static_cast<const uint16_t*>(logits_p_bf16), static_cast<const uint16_t*>(logits_q_bf16), T,
      V, top_k, temperature, ear_tok, kl_tok, ear_mean, kl_mean, static_cast<cudaStream_t>(stream)));
}

slq_status slq_ear_kl(const void* logits_p_bf16, const void* logits_q_bf16, int64_t T, int64_t V,
                      float temperature, float* ear_tok, float* kl_tok, double* ear_mean,
                      double* kl_mean, uint32_t* flags, void* stream) {
  if (T < 0 || T > kMaxDim || V < 1 || V > kMaxDim || !product_ok(T, V))
    return SLQ_ERR_INVALID_ARGUMENT;
  if (!std::isfinite(temperature) || !(temperature > 0.0f)) return SLQ_ERR_INVALID_ARGUMENT;
  if (T == 0) return SLQ_OK;
  if (!logits_p_bf16 || !logits_q_bf16 || !ear_tok || !kl_tok) return SLQ_ERR_INVALID_ARGUMENT;
  if (!aligned(logits_p_bf16, 16) || !aligned(logits_q_bf16, 16) || !aligned(ear_tok, 4) ||
      !aligned(kl_tok, 4) || (ear_mean && !aligned(ear_mean, 8)) ||
      (kl_mean && !aligned(kl_mean, 8)) || (flags && !aligned(flags, 4)))
    return SLQ_ERR_INVALID_ARGUMENT;
  const Range ins[2] = {range_of(logits_p_bf16, T * V * 2), range_of(logits_q_bf16, T * V * 2)};
  const Range outs[5] = {range_of(ear_tok, T * 4), range_of(kl_tok, T * 4),
                         range_of(ear_mean, ear_mean ? 8 : 0), range_of(kl_mean, kl_mean ? 8 : 0),
                         range_of(flags, flags ? 4 : 0)};
  if (!disjoint(outs, 5, ins, 2)) return SLQ_ERR_INVALID_ARGUMENT;
  const slq_status dev = check_device();
  if (dev != SLQ_OK) return dev;
  return from_cuda(slq::launch_ear_kl(
      static_cast<const uint16_t*>(logits_p_bf16), static_cast<const uint16_t*>(logits_q_bf16), T,
      V, temperature, ear_tok, kl_tok, ear_mean, kl_mean, flags, static_cast<cudaStream_t>(stream)));
}

slq_status slq_grid_noise(const void* W_bf16, int64_t N, int64_t K, int bits, float* gamma,
                          float* sse_asym, float* sse_sym, uint32_t* flags, void* stream) {
  if (N < 0 || N > kMaxDim || !valid_k(K) || !valid_bits(bits) || !product_ok(N, K))
    return SLQ_ERR_INVALID_ARGUMENT;
  if (N == 0) return SLQ_OK;
  if (!W_bf16 || !gamma || !sse_asym || !sse_sym) return SLQ_ERR_INVALID_ARGUMENT;
  if (!aligned(W_bf16, 16) || !aligned(gamma, 4) || !aligned(sse_asym, 4) || !aligned(sse_sym, 4) ||
      (flags && !aligned(flags, 4)))
    return SLQ_ERR_INVALID_ARGUMENT;
  const int64_t G = N * (K / slq::kGroup);
  const Range ins[1] = {range_of(W_bf16, N * K * 2)};
  const Range outs[4] = {range_of(gamma, G * 4), range_of(sse_asym, G * 4), range_of(sse_sym, G * 4),
                         range_of(flags, flags ? 4 : 0)};
  if (!disjoint(outs, 4, ins, 1)) return SLQ_ERR_INVALID_ARGUMENT;
  const slq_status dev = check_device();
  if (dev != SLQ_OK) return dev;
  return from_cuda(slq::launch_grid_noise(static_cast<const uint16_t*>(W_bf16), N, K, bits, gamma,
                                          sse_asym, sse_sym, flags,
                                          static_cast<cudaStream_t>(stream)));
}

size_t slq_gptq_workspace_bytes(int64_t N, int64_t K) {
  if (N < 0 || N > kMaxDim || !valid_k(K) || K > 16384 || !product_ok(N, K)) return 0;
  return slq::gptq_workspace_bytes(N, K);
}

slq_status slq_gptq(const void* W_bf16, int64_t N, int64_t K, int bits, const void* X_bf16, int64_t T,
                    double damp, uint32_t* packed, void* scales_f16, uint8_t* zeros, void* workspace,
                    size_t workspace_bytes, uint32_t* flags, void* stream) {
  if (N < 0 || N > kMaxDim || !valid_k(K) || K > 16384 || !valid_bits(bits) || !product_ok(N, K))
    return SLQ_ERR_INVALID_ARGUMENT;
  if (T < 1 || T > kMaxDim || !product_ok(T, K) || !std::isfinite(damp) || !(damp >= 0.0))
    return SLQ_ERR_INVALID_ARGUMENT;
  if (N == 0) return SLQ_OK;
  if (!W_bf16 || !X_bf16 || !packed || !scales_f16 || !zeros || !workspace)
    return SLQ_ERR_INVALID_ARGUMENT;
  const size_t need = slq::gptq_workspace_bytes(N, K);
  if (workspace_bytes < need) return SLQ_ERR_INVALID_ARGUMENT;
  if (!aligned(W_bf16, 2) || !aligned(X_bf16, 2) || !aligned(packed, 4) || !aligned(scales_f16, 2) ||
      !aligned(workspace, 16) || (flags && !aligned(flags, 4)))
    return SLQ_ERR_INVALID_ARGUMENT;
  const int64_t G = K / slq::kGroup;
  const Range ins[2] = {range_of(W_bf16, N * K * 2), range_of(X_bf16, T * K * 2)};
  const Range outs[5] = {range_of(packed, N * K * bits / 8), range_of(scales_f16, N * G * 2),
                         range_of(zeros, N * G), range_of(flags, flags ? 4 : 0),
                         range_of(workspace, static_cast<int64_t>(need))};
  if (!disjoint(outs, 5, ins, 2)) return SLQ_ERR_INVALID_ARGUMENT;
  const slq_status dev = check_device();
  if (dev != SLQ_OK) return dev;
  return from_cuda(slq::launch_gptq(static_cast<const uint16_t*>(W_bf16), N, K, bits,
                                    static_cast<const uint16_t*>(X_bf16), T, damp, packed,
                                    static_cast<uint16_t*>(scales_f16), zeros, workspace, flags,
                                    static_cast<cudaStream_t>(stream)));
}

}  // extern "C"
