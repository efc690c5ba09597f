// CUDA-core ternary GEMM for any M: the correctness baseline path.
//
// Computes Y[m][n] = fp16( sum_b d[n][b] * sum_{k in b} X[m][k] * t[n][k] )
// ("Scaling Laws and Efficient Inference for Ternary Language Models",
// section "The model", step 3, with the 256-weight fp16-scaled blocks of
// section "Fast inference on CPUs"), accumulating in fp32.
//
// One warp owns one output row n and up to eight batch rows m.  Lanes stride
// over the row's 32-bit TQ2 words (16 weights, weight j at bits 2j) or TQ1
// bytes (5 weights, multiply-by-3 digit extraction); each lane forms the
// exact fp32 sum of x*t over its word, scales it by the block's d, and the
// lane partials are combined by a shuffle tree.  X is re-read per output row
// (from L1/L2), so this path is only meant for shapes the tensor-core paths
// do not serve, and as a second opinion in tests.
#include "tri_internal.cuh"

namespace tri {
namespace {

constexpr int kWarps = 8;
constexpr int kMC = 8;   // batch rows per warp

__global__ void __launch_bounds__(kWarps * 32)
gemm_simt_tq2_kernel(const __half* __restrict__ X, const uint32_t* __restrict__ qs,
                     const __half* __restrict__ d, __half* __restrict__ Y, int M, int N, int K) {
  const int lane = threadIdx.x & 31;
  const int n = blockIdx.x * kWarps + (threadIdx.x >> 5);
  const int m0 = blockIdx.y * kMC;
  if (n >= N) return;
  const int mc = min(kMC, M - m0);
  const int words = K / 16;
  const int nb = K / kBlock;
  float acc[kMC];
#pragma unroll
  for (int i = 0; i < kMC; ++i) acc[i] = 0.f;
  const uint32_t* row = qs + (int64_t)n * words;
  for (int w = lane; w < words; w += 32) {
    const unsigned q = row[w];
    const float sc = __half2float(d[(int64_t)n * nb + (w >> 4)]);
    float t[16];
#pragma unroll
    for (int j = 0; j < 16; ++j) t[j] = (float)((int)((q >> (2 * j)) & 3u) - 1);
#pragma unroll
    for (int i = 0; i < kMC; ++i) {
      if (i < mc) {
        const uint4* xp = reinterpret_cast<const uint4*>(X + (int64_t)(m0 + i) * K + 16 * w);
        const uint4 a = xp[0], b = xp[1];
        const unsigned xs[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
        float p = 0.f;
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          const float2 f = __half22float2(*reinterpret_cast<const __half2*>(&xs[j]));
          p = fmaf(f.x, t[2 * j], p);
          p = fmaf(f.y, t[2 * j + 1], p);
        }
        acc[i] = fmaf(sc, p, acc[i]);
      }
    }
  }
#pragma unroll
  for (int i = 0; i < kMC; ++i) {
    float v = acc[i];
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xFFFFFFFFu, v, o);
    if (lane == 0 && i < mc) Y[(int64_t)(m0 + i) * N + n] = __float2half_rn(v);
  }
}

__global__ void __launch_bounds__(kWarps * 32)
gemm_simt_tq1_kernel(const __half* __restrict__ X, const uint8_t* __restrict__ qs,
                     const __half* __restrict__ d, __half* __restrict__ Y, int M, int N, int K) {
  const int lane = threadIdx.x & 31;
  const int n = blockIdx.x * kWarps + (threadIdx.x >> 5);
  const int m0 = blockIdx.y * kMC;
  if (n >= N) return;
  const int mc = min(kMC, M - m0);
  const int nb = K / kBlock;
  const int rowbytes = nb * kTq1BlockBytes;
  float acc[kMC];
#pragma unroll
  for (int i = 0; i < kMC; ++i) acc[i] = 0.f;
  const uint8_t* row = qs + (int64_t)n * rowbytes;
  for (int j = lane; j < rowbytes; j += 32) {
    const int b = j / kTq1BlockBytes;
    const int jb = j - b * kTq1BlockBytes;
    const int cnt = jb < kTq1Groups ? 5 : 1;
    const int k0 = b * kBlock + 5 * jb;
    const float sc = __half2float(d[(int64_t)n * nb + b]);
    unsigned v = row[j];
    float t[5];
#pragma unroll
    for (int q = 0; q < 5; ++q) {
      v *= 3u;
      t[q] = (float)((int)(v >> 8) - 1);
      v &= 0xFFu;
    }
#pragma unroll
    for (int i = 0; i < kMC; ++i) {
      if (i < mc) {
        const __half* xp = X + (int64_t)(m0 + i) * K + k0;
        float p = 0.f;
#pragma unroll
        for (int q = 0; q < 5; ++q)
          if (q < cnt) p = fmaf(__half2float(xp[q]), t[q], p);
        acc[i] = fmaf(sc, p, acc[i]);
      }
    }
  }
#pragma unroll
  for (int i = 0; i < kMC; ++i) {
    float v = acc[i];
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xFFFFFFFFu, v, o);
    if (lane == 0 && i < mc) Y[(int64_t)(m0 + i) * N + n] = __float2half_rn(v);
  }
}

}  // namespace

cudaError_t launch_gemm_simt(int fmt, const __half* X, const uint8_t* qs, const __half* d,
                             __half* Y, int M, int N, int K, cudaStream_t s) {
  dim3 grid((unsigned)ceil_div(N, kWarps), (unsigned)ceil_div(M, kMC));
  if (grid.y > 65535u) return cudaErrorInvalidValue;
  if (fmt == TRI_TQ2)
    gemm_simt_tq2_kernel<<<grid, kWarps * 32, 0, s>>>(X, reinterpret_cast<const uint32_t*>(qs),
                                                      d, Y, M, N, K);
  else
    gemm_simt_tq1_kernel<<<grid, kWarps * 32, 0, s>>>(X, qs, d, Y, M, N, K);
  return cudaGetLastError();
}

}  // namespace tri
