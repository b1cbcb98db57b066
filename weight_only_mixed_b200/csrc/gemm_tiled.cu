// gemm_tiled.cu -- placeholder until the tcgen05 tiled kernel lands.
#include "internal.h"

namespace slq {
cudaError_t launch_gemm_tiled(const uint16_t*, int64_t, int64_t, int64_t, int, const uint32_t*,
                              const uint16_t*, const uint8_t*, void*, bool, uint32_t*,
                              cudaStream_t) {
  return cudaErrorNotSupported;
}
}  // namespace slq
