// Prefill GEMM on tcgen05 tensor cores (placeholder until the kernel lands).
#include "tern_internal.cuh"

namespace tern {
cudaError_t launch_gemm(const tern_matrix&, const uint16_t*, int64_t, uint16_t*, uint32_t*, cudaStream_t) {
  return cudaErrorNotSupported;
}
}  // namespace tern
