// Compute-regime tcgen05 kernel (M >= 64): not built yet.
#include "tri_internal.cuh"
namespace tri {
bool gemm_tc_supported(int, int64_t, int64_t, int64_t) { return false; }
size_t gemm_tc_ws_bytes(int, int64_t, int64_t, int64_t, int) { return 0; }
cudaError_t launch_gemm_tc(int, const __half*, const uint8_t*, const __half*, __half*, int, int,
                           int, void*, int, cudaStream_t) {
  return cudaErrorNotSupported;
}
}  // namespace tri
