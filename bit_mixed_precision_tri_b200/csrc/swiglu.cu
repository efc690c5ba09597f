// SwiGLU combine for the fused gate/up projection when the GEMM kernel that
// served the call has no fused epilogue: Y[m][f] = silu(G[m][f]) * U[m][f]
// from the [M][2F] product whose columns hold gate and up features
// interleaved in groups of eight (column 16j + i: gate feature 8j + i,
// column 16j + 8 + i: up feature 8j + i).  silu(g) = g / (1 + e^-g), the
// gated feed-forward unit of "Scaling Laws and Efficient Inference for
// Ternary Language Models", section "The model".
#include "tri_internal.cuh"

namespace tri {
namespace {

__global__ void __launch_bounds__(256)
swiglu_combine_kernel(const __half* __restrict__ G2, __half* __restrict__ Y, int64_t M, int64_t F) {
  const int64_t total = M * F;
  const int64_t stride = (int64_t)gridDim.x * blockDim.x;
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < total; i += stride) {
    const int64_t m = i / F, f = i % F;
    const int64_t c = 16 * (f >> 3) + (f & 7);
    const float g = __half2float(G2[m * 2 * F + c]);
    const float u = __half2float(G2[m * 2 * F + c + 8]);
    Y[i] = __float2half_rn(g / (1.f + expf(-g)) * u);
  }
}

}  // namespace

cudaError_t launch_swiglu_combine(const __half* G2, __half* Y, int64_t M, int64_t F, cudaStream_t s) {
  const int64_t total = M * F;
  int64_t g = ceil_div(total, 256);
  if (g > 148 * 16) g = 148 * 16;
  if (g < 1) g = 1;
  swiglu_combine_kernel<<<(unsigned)g, 256, 0, s>>>(G2, Y, M, F);
  return cudaGetLastError();
}

}  // namespace tri
