// TQ2 / TQ1 packing and unpacking on sm_100a.
//
// "Scaling Laws and Efficient Inference for Ternary Language Models",
// section "Packing ternary weights":
//   * every weight d in {-1,0,1} is shifted to d' = d + 1 in {0,1,2};
//   * "2 bits per weight": four digits per byte, decoded by a shift and a mask
//     d' = (b >> 2j) & 3; with the "TriRun" storage line (sixteen 2-bit weights
//     per 32-bit word) this library puts weight j of a 16-weight word at bits 2j;
//   * "1.6 bits per weight": five digits read as a base-3 number N5 (first
//     weight most significant) become the byte floor((256*N5 + 242)/243);
//     decoding multiplies by 3 and splits off the high byte as the next digit.
// Section "Fast inference on CPUs": 256-weight blocks with one 16-bit scale.
//
// TQ1 block layout (52 bytes per 256 weights): bytes 0..50 hold weights
// 5g..5g+4 of the block, byte 51 holds weight 255 followed by four zero
// weights (digit 1 each).
//
// All four kernels are byte streams bound by HBM bandwidth; one thread packs
// or unpacks one 32-bit TQ2 word (16 weights) or one TQ1 byte (5 weights).
#include "tri_internal.cuh"

namespace tri {
namespace {

constexpr int kThreads = 256;

int grid_for(int64_t items) {
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  int64_t g = ceil_div(items, kThreads);
  const int64_t cap = (int64_t)sms * 16;
  if (g > cap) g = cap;
  return (int)(g < 1 ? 1 : g);
}

__device__ __forceinline__ void block_count_add(int cnt, int32_t* counter) {
  // warp reduce, then one atomic per warp
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) cnt += __shfl_xor_sync(0xFFFFFFFFu, cnt, o);
  if ((threadIdx.x & 31) == 0 && cnt != 0 && counter != nullptr) atomicAdd(counter, cnt);
}

// digit d' of a trit byte; values outside {-1,0,1} count as invalid, packed as 0
__device__ __forceinline__ unsigned digit_of(int8_t t, int& bad) {
  const int v = (int)t;
  if (v < -1 || v > 1) { ++bad; return 1u; }
  return (unsigned)(v + 1);
}

__global__ void __launch_bounds__(kThreads)
pack_tq2_kernel(const int8_t* __restrict__ trits, int64_t nwords, uint32_t* __restrict__ qs,
                int32_t* invalid) {
  const int64_t stride = (int64_t)gridDim.x * kThreads;
  int64_t i = (int64_t)blockIdx.x * kThreads + threadIdx.x;
  int bad = 0;
  for (int64_t base = (int64_t)blockIdx.x * kThreads; base < nwords; base += stride, i += stride) {
    if (i < nwords) {
      const uint4 v = reinterpret_cast<const uint4*>(trits)[i];
      const unsigned w4[4] = {v.x, v.y, v.z, v.w};
      unsigned word = 0u;
#pragma unroll
      for (int q = 0; q < 4; ++q)
#pragma unroll
        for (int b = 0; b < 4; ++b) {
          const int8_t t = (int8_t)((w4[q] >> (8 * b)) & 0xFFu);
          word |= digit_of(t, bad) << (2 * (4 * q + b));
        }
      qs[i] = word;
    }
  }
  block_count_add(bad, invalid);
}

__global__ void __launch_bounds__(kThreads)
pack_tq1_kernel(const int8_t* __restrict__ trits, int64_t N, int64_t K, uint8_t* __restrict__ qs,
                int32_t* invalid) {
  const int64_t nb = K / kBlock;
  const int64_t nbytes = N * nb * kTq1BlockBytes;
  const int64_t stride = (int64_t)gridDim.x * kThreads;
  int64_t i = (int64_t)blockIdx.x * kThreads + threadIdx.x;
  int bad = 0;
  for (int64_t base = (int64_t)blockIdx.x * kThreads; base < nbytes; base += stride, i += stride) {
    if (i < nbytes) {
      const int64_t rowblk = i / kTq1BlockBytes;          // n * nb + b
      const int j = (int)(i - rowblk * kTq1BlockBytes);
      const int64_t n = rowblk / nb, b = rowblk - n * nb;
      const int8_t* t = trits + n * K + b * kBlock + 5 * j;
      unsigned n5 = 0u;
      if (j < kTq1Groups) {
#pragma unroll
        for (int q = 0; q < 5; ++q) n5 = 3u * n5 + digit_of(t[q], bad);
      } else {
        n5 = digit_of(t[0], bad);
#pragma unroll
        for (int q = 0; q < 4; ++q) n5 = 3u * n5 + 1u;     // four zero weights
      }
      qs[i] = (uint8_t)((n5 * 256u + 242u) / 243u);
    }
  }
  block_count_add(bad, invalid);
}

__global__ void __launch_bounds__(kThreads)
scales_kernel(const float* __restrict__ scales, int64_t n_scales, int64_t count,
              __half* __restrict__ d) {
  const int64_t stride = (int64_t)gridDim.x * kThreads;
  for (int64_t i = (int64_t)blockIdx.x * kThreads + threadIdx.x; i < count; i += stride)
    d[i] = __float2half_rn(scales[n_scales == 1 ? 0 : i]);
}

__global__ void __launch_bounds__(kThreads)
unpack_tq2_kernel(const uint32_t* __restrict__ qs, int64_t nwords, int8_t* __restrict__ trits,
                  int32_t* invalid) {
  const int64_t stride = (int64_t)gridDim.x * kThreads;
  int64_t i = (int64_t)blockIdx.x * kThreads + threadIdx.x;
  int bad = 0;
  for (int64_t base = (int64_t)blockIdx.x * kThreads; base < nwords; base += stride, i += stride) {
    if (i < nwords) {
      const unsigned w = qs[i];
      unsigned out[4];
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        unsigned o = 0u;
#pragma unroll
        for (int b = 0; b < 4; ++b) {
          const unsigned f = (w >> (2 * (4 * q + b))) & 3u;
          bad += (f == 3u);
          o |= ((f - 1u) & 0xFFu) << (8 * b);
        }
        out[q] = o;
      }
      reinterpret_cast<uint4*>(trits)[i] = make_uint4(out[0], out[1], out[2], out[3]);
    }
  }
  block_count_add(bad, invalid);
}

__global__ void __launch_bounds__(kThreads)
unpack_tq1_kernel(const uint8_t* __restrict__ qs, int64_t N, int64_t K, int8_t* __restrict__ trits,
                  int32_t* invalid) {
  const int64_t nb = K / kBlock;
  const int64_t nbytes = N * nb * kTq1BlockBytes;
  const int64_t stride = (int64_t)gridDim.x * kThreads;
  int64_t i = (int64_t)blockIdx.x * kThreads + threadIdx.x;
  int bad = 0;
  for (int64_t base = (int64_t)blockIdx.x * kThreads; base < nbytes; base += stride, i += stride) {
    if (i < nbytes) {
      const int64_t rowblk = i / kTq1BlockBytes;
      const int j = (int)(i - rowblk * kTq1BlockBytes);
      const int64_t n = rowblk / nb, b = rowblk - n * nb;
      const unsigned byte = qs[i];
      // multiply-shift decoder: x*3, high byte is the digit, low byte goes on
      unsigned v = byte, dig[5], n5 = 0u;
#pragma unroll
      for (int q = 0; q < 5; ++q) {
        v *= 3u;
        dig[q] = v >> 8;
        v &= 0xFFu;
        n5 = 3u * n5 + dig[q];
      }
      bad += ((n5 * 256u + 242u) / 243u) != byte;     // not in the encoder's image
      int8_t* t = trits + n * K + b * kBlock + 5 * j;
      if (j < kTq1Groups) {
#pragma unroll
        for (int q = 0; q < 5; ++q) t[q] = (int8_t)((int)dig[q] - 1);
      } else {
        t[0] = (int8_t)((int)dig[0] - 1);
        bad += (dig[1] != 1u || dig[2] != 1u || dig[3] != 1u || dig[4] != 1u) &&
               ((n5 * 256u + 242u) / 243u) == byte;
      }
    }
  }
  block_count_add(bad, invalid);
}

// TQ1 -> TQ2 transcode, so the tensor-core GEMM paths can consume TQ1
// weights.  A warp takes 32 consecutive (row, block) units: it copies their
// 32 x 52 contiguous bytes into shared memory with 16-byte loads, each lane
// turns one unit's 52 bytes into sixteen TQ2 words (a per-CTA table maps
// each byte value to its five digits as 2-bit fields, first weight lowest,
// built with the multiply-by-3 decoder; the fields of consecutive bytes form
// one 512-bit stream, 10 bits per byte and 2 for the last byte's single
// weight, cut into 32-bit words at compile-time offsets), and the warp
// writes the 32 x 64 output bytes back with 16-byte stores.  A lane's 13
// input words sit at a 13-word stride (odd: no bank conflicts) and its 16
// output words at a 17-word stride.
constexpr int kTcWarps = kThreads / 32;
constexpr int kInWords = kTq1BlockBytes / 4;     // 13
constexpr int kOutStride = 17;

__global__ void __launch_bounds__(kThreads)
transcode_tq1_tq2_kernel(const uint8_t* __restrict__ qs1, int64_t rowblocks, uint32_t* __restrict__ qs2) {
  __shared__ uint16_t lut[256];
  __shared__ __align__(16) uint32_t sin[kTcWarps][32 * kInWords];
  __shared__ uint32_t sout[kTcWarps][32 * kOutStride];
  for (int i = threadIdx.x; i < 256; i += kThreads) {
    unsigned v = (unsigned)i, code = 0u;
#pragma unroll
    for (int q = 0; q < 5; ++q) {
      v *= 3u;
      code |= (v >> 8) << (2 * q);
      v &= 0xFFu;
    }
    lut[i] = (uint16_t)code;
  }
  __syncthreads();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  uint32_t* wi = sin[warp];
  uint32_t* wo = sout[warp];
  const int64_t step = (int64_t)gridDim.x * kTcWarps * 32;
  const bool a16 = (reinterpret_cast<uintptr_t>(qs1) & 15u) == 0;   // TQ1 planes need only 4-byte alignment
  for (int64_t rb0 = ((int64_t)blockIdx.x * kTcWarps + warp) * 32; rb0 < rowblocks; rb0 += step) {
    const int nb = rowblocks - rb0 < 32 ? (int)(rowblocks - rb0) : 32;
    const uint32_t* src = reinterpret_cast<const uint32_t*>(qs1 + rb0 * kTq1BlockBytes);
    const int nw = nb * kInWords;
    if (nb == 32 && a16) {             // 416 words = 104 aligned 16-byte pieces (rb0 * 52 % 16 == 0)
      const uint4* s4 = reinterpret_cast<const uint4*>(src);
      for (int i = lane; i < 32 * kInWords / 4; i += 32) reinterpret_cast<uint4*>(wi)[i] = __ldg(s4 + i);
    } else {
      for (int i = lane; i < nw; i += 32) wi[i] = __ldg(src + i);
    }
    __syncwarp();
    if (lane < nb) {
      uint32_t in[kInWords];
#pragma unroll
      for (int j = 0; j < kInWords; ++j) in[j] = wi[lane * kInWords + j];
      uint64_t acc = 0;
      int nbits = 0, o = 0;
#pragma unroll
      for (int i = 0; i < kTq1BlockBytes; ++i) {
        const unsigned byte = (in[i >> 2] >> (8 * (i & 3))) & 0xFFu;
        unsigned code = lut[byte];
        const int nbt = i == kTq1BlockBytes - 1 ? 2 : 10;   // byte 51 holds one weight
        if (nbt == 2) code &= 3u;
        acc |= (uint64_t)code << nbits;
        nbits += nbt;
        if (nbits >= 32) {
          wo[lane * kOutStride + o++] = (uint32_t)acc;
          acc >>= 32;
          nbits -= 32;
        }
      }
    }
    __syncwarp();
    uint4* dst = reinterpret_cast<uint4*>(qs2 + rb0 * 16);
    for (int i = lane; i < nb * 4; i += 32) {            // output word 4i .. 4i+3 of the group
      const int u = i >> 2, o = (i & 3) * 4;
      const uint32_t* w = wo + u * kOutStride + o;
      dst[i] = make_uint4(w[0], w[1], w[2], w[3]);
    }
    __syncwarp();
  }
}

}  // namespace

cudaError_t launch_transcode_tq1_tq2(const uint8_t* qs1, int64_t N, int64_t K, uint8_t* qs2,
                                     cudaStream_t s) {
  const int64_t rowblocks = N * (K / kBlock);
  int64_t g = ceil_div(rowblocks, kThreads);      // one (row, block) unit per thread
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  if (g > (int64_t)sms * 8) g = (int64_t)sms * 8;
  transcode_tq1_tq2_kernel<<<(unsigned)g, kThreads, 0, s>>>(qs1, rowblocks,
                                                            reinterpret_cast<uint32_t*>(qs2));
  return cudaGetLastError();
}

cudaError_t launch_pack_tq2(const int8_t* trits, int64_t N, int64_t K, const float* scales,
                            int64_t n_scales, uint8_t* qs, uint16_t* d, int32_t* invalid,
                            cudaStream_t s) {
  if (invalid) {
    cudaError_t e = cudaMemsetAsync(invalid, 0, sizeof(int32_t), s);
    if (e != cudaSuccess) return e;
  }
  const int64_t nwords = N * K / 16;
  pack_tq2_kernel<<<grid_for(nwords), kThreads, 0, s>>>(trits, nwords,
                                                         reinterpret_cast<uint32_t*>(qs), invalid);
  const int64_t nd = N * (K / kBlock);
  scales_kernel<<<grid_for(nd), kThreads, 0, s>>>(scales, n_scales, nd,
                                                   reinterpret_cast<__half*>(d));
  return cudaGetLastError();
}

cudaError_t launch_pack_tq1(const int8_t* trits, int64_t N, int64_t K, const float* scales,
                            int64_t n_scales, uint8_t* qs, uint16_t* d, int32_t* invalid,
                            cudaStream_t s) {
  if (invalid) {
    cudaError_t e = cudaMemsetAsync(invalid, 0, sizeof(int32_t), s);
    if (e != cudaSuccess) return e;
  }
  const int64_t nbytes = N * (K / kBlock) * kTq1BlockBytes;
  pack_tq1_kernel<<<grid_for(nbytes), kThreads, 0, s>>>(trits, N, K, qs, invalid);
  const int64_t nd = N * (K / kBlock);
  scales_kernel<<<grid_for(nd), kThreads, 0, s>>>(scales, n_scales, nd,
                                                   reinterpret_cast<__half*>(d));
  return cudaGetLastError();
}

cudaError_t launch_unpack_tq2(const uint8_t* qs, int64_t N, int64_t K, int8_t* trits,
                              int32_t* invalid, cudaStream_t s) {
  if (invalid) {
    cudaError_t e = cudaMemsetAsync(invalid, 0, sizeof(int32_t), s);
    if (e != cudaSuccess) return e;
  }
  const int64_t nwords = N * K / 16;
  unpack_tq2_kernel<<<grid_for(nwords), kThreads, 0, s>>>(
      reinterpret_cast<const uint32_t*>(qs), nwords, trits, invalid);
  return cudaGetLastError();
}

cudaError_t launch_unpack_tq1(const uint8_t* qs, int64_t N, int64_t K, int8_t* trits,
                              int32_t* invalid, cudaStream_t s) {
  if (invalid) {
    cudaError_t e = cudaMemsetAsync(invalid, 0, sizeof(int32_t), s);
    if (e != cudaSuccess) return e;
  }
  const int64_t nbytes = N * (K / kBlock) * kTq1BlockBytes;
  unpack_tq1_kernel<<<grid_for(nbytes), kThreads, 0, s>>>(qs, N, K, trits, invalid);
  return cudaGetLastError();
}

}  // namespace tri
