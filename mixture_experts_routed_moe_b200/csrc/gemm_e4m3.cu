// FP8 (e4m3) expert GEMMs: not built yet.
#include "moe_internal.h"

namespace moe {

bool e4m3_path_available() { return false; }

cudaError_t launch_gemm_e4m3(const moe_shape*, const Plan&, const void*, const void*, const void*, const uint8_t*,
                             const uint8_t*, uint8_t*, int, int, cudaStream_t) {
  return cudaErrorNotSupported;
}

}  // namespace moe
