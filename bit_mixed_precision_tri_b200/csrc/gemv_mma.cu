// Decode-regime tensor-core kernel (M <= 16): not built yet.
#include "tri_internal.cuh"
namespace tri {
bool gemv_mma_supported(int, int64_t, int64_t, int64_t) { return false; }
size_t gemv_mma_ws_bytes(int, int64_t, int64_t, int64_t, int) { return 0; }
cudaError_t launch_gemv_mma(int, const __half*, const uint8_t*, const __half*, __half*, int, int,
                            int, void*, int, cudaStream_t) {
  return cudaErrorNotSupported;
}
}  // namespace tri
