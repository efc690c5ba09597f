// Decode-regime ternary GEMM (M <= 16) for TQ2 weights on the fifth-generation
// tensor cores of sm_100a.
//
// Y = X (d * W_hat)^T ("Scaling Laws and Efficient Inference for Ternary
// Language Models", section "The model", step 3) for decode batches, where the
// layer is bound by streaming the packed weights (section "TriRun: ternary
// inference on GPUs": 2-bit weights move 8x fewer bytes than fp16).
//
// Design:
//  * Units of (128 weight rows) x (one 256-weight block) are split over a
//    persistent grid (one CTA per SM) as contiguous ranges (stream-K).
//  * A producer thread stages each unit: a 2-D TMA load of the packed tile
//    (128 rows x 64 bytes, 64-byte swizzle, L2 evict-first) plus bulk copies of
//    the block's prepared activations (four [16 x 64] fp16 sub-tiles in the
//    128-byte-swizzled K-major layout), decode bias and 128 row scales.
//  * Four decoder warps (one weight row per thread, i.e. one TMEM lane)
//    expand sixteen 2-bit fields per 32-bit word with one LOP3 per pair --
//    (w & (0x00030003 << 2j)) | fp16 exponent of 2^(10-2j) is the pair
//    (2^(10-2j) + d'_j, 2^(10-2j) + d'_{j+8}), the "TriRun" mask-and-exponent
//    idea -- and write them straight into tensor memory with tcgen05.st: the
//    decoded weights never touch shared memory.
//  * One thread issues tcgen05.mma with A = decoded weights (TMEM, 128 x 16),
//    B = activations (shared memory, 16 batch columns), D = fp32 in TMEM, per
//    block into one of two accumulators, so a block's scale can be applied.
//  * The decoder warps read each block's accumulator back (tcgen05.ld),
//    subtract the constant part sum_k (2^(10-2j(k)) + 1) x_k (prepared with the
//    activations) and add d * (D - c) to registers; a row tile split across
//    CTAs is reduced by its last CTA (atomic ticket, no waiting), in CTA order.
#include <cudaTypedefs.h>

#include "sm100_ptx.cuh"
#include "tri_internal.cuh"

namespace tri {
namespace {

constexpr int kRows = 128;                      // weight rows per unit (MMA M, TMEM lanes)
constexpr int kNB = 16;                         // MMA N: batch columns, zero-padded
constexpr int kDecWarps = 4;
constexpr int kThreads = (2 + kDecWarps) * 32;  // producer, MMA issuer, decoders
constexpr int kWBytes = kRows * 64;             // packed bytes per unit
constexpr int kXBytes = 4 * kNB * 128;          // four [16 x 64] fp16 sub-tiles
constexpr int kCBytes = kNB * 4;                // decode bias per batch column
constexpr int kSBytes = kRows * 2;              // fp16 scale per row
constexpr int kACols = 128;                     // TMEM columns per decoded block (256 fp16)
constexpr int kDCol0 = 2 * kACols;              // first accumulator column
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kWaitLimit = 1u << 22;
constexpr int kSmemBudget = 210 * 1024;

struct Params {
  const uint8_t* xt;    // [B][4][16][128 B] swizzled activation sub-tiles
  const float* bias;    // [B][16]
  const __half* dT;     // [B][Npad] scales, block-major
  float* partials;      // [G][2][128][16]
  unsigned* counters;   // [T]
  unsigned* error;
  int M, N, K, B, T, G, stages, Npad;
  long long U;
};

__host__ __device__ inline long long range_start(long long c, long long U, long long G) {
  return c * U / G;
}
__host__ __device__ inline long long cta_of_unit(long long u, long long U, long long G) {
  return ((u + 1) * G + U - 1) / U - 1;
}

// ---------------------------------------------------------------- prep kernel
// CTAs [0, B): activations of block b in the decode's pair order (x_j, x_{j+8})
// inside each 16-group, as four 128-byte-swizzled K-major [16 x 64] tiles, and
// the decode bias of every batch row.  CTAs [B, B + Npad/64): transpose 64
// rows of the scale plane into dT[B][Npad].
__global__ void __launch_bounds__(256)
xprep_tc_kernel(const __half* __restrict__ X, const __half* __restrict__ dsc, int M, int N, int K,
                int B, int Npad, uint8_t* __restrict__ xt, float* __restrict__ bias,
                __half* __restrict__ dT, unsigned* __restrict__ tickets, int T) {
  ptx::griddep_launch_dependents();
  if (blockIdx.x == 0)    // tickets start at zero on every call
    for (int i = threadIdx.x; i < T; i += blockDim.x) tickets[i] = 0u;
  if ((int)blockIdx.x >= B) {
    __shared__ __half tile[64][66];
    const int r0 = ((int)blockIdx.x - B) * 64;
    for (int b0 = 0; b0 < B; b0 += 64) {
      for (int idx = threadIdx.x; idx < 64 * 64; idx += blockDim.x) {
        const int r = idx >> 6, bb = idx & 63;
        tile[r][bb] = (r0 + r < N && b0 + bb < B) ? dsc[(size_t)(r0 + r) * B + b0 + bb]
                                                  : __float2half(0.f);
      }
      __syncthreads();
      for (int idx = threadIdx.x; idx < 64 * 64; idx += blockDim.x) {
        const int bb = idx >> 6, r = idx & 63;
        if (b0 + bb < B) dT[(size_t)(b0 + bb) * Npad + r0 + r] = tile[r][bb];
      }
      __syncthreads();
    }
    return;
  }
  const int b = blockIdx.x;
  const int m = threadIdx.x >> 4, G = threadIdx.x & 15;
  uint4 lo = make_uint4(0, 0, 0, 0), hi = lo;
  if (m < M) {
    const uint4* src = reinterpret_cast<const uint4*>(X + (size_t)m * K + (size_t)b * kBlock + G * 16);
    lo = src[0];
    hi = src[1];
  }
  const uint32_t lw[4] = {lo.x, lo.y, lo.z, lo.w}, hw[4] = {hi.x, hi.y, hi.z, hi.w};
  uint32_t pr[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) pr[i] = __byte_perm(lw[i >> 1], hw[i >> 1], (i & 1) ? 0x7632 : 0x5410);
  const int t = G >> 2, g4 = G & 3;           // sub-tile, 16-group within it
  uint8_t* sub = xt + ((size_t)b * 4 + t) * (kNB * 128) + m * 128;
  const int c0 = 2 * g4, c1 = 2 * g4 + 1;     // logical 16-byte chunks of row m
  *reinterpret_cast<uint4*>(sub + ((c0 ^ (m & 7)) * 16)) = make_uint4(pr[0], pr[1], pr[2], pr[3]);
  *reinterpret_cast<uint4*>(sub + ((c1 ^ (m & 7)) * 16)) = make_uint4(pr[4], pr[5], pr[6], pr[7]);
  const float beta1[4] = {1025.f, 257.f, 65.f, 17.f};
  float s = 0.f;
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const float2 a = __half22float2(*reinterpret_cast<const __half2*>(&lw[i >> 1]));
    const float2 c = __half22float2(*reinterpret_cast<const __half2*>(&hw[i >> 1]));
    s = fmaf(beta1[i & 3], (i & 1) ? a.y : a.x, s);
    s = fmaf(beta1[i & 3], (i & 1) ? c.y : c.x, s);
  }
#pragma unroll
  for (int o = 8; o > 0; o >>= 1) s += __shfl_xor_sync(0xFFFFFFFFu, s, o);
  if (G == 0) bias[(size_t)b * kNB + m] = s;
}

// ---------------------------------------------------------------- main kernel
__device__ __forceinline__ uint32_t decode_pair(uint32_t w, int j) {
  const uint32_t mask = 0x00030003u << (2 * j);
  const uint32_t e = (j == 0) ? 0x6400u : (j == 1) ? 0x5C00u : (j == 2) ? 0x5400u : 0x4C00u;
  return (w & mask) | (e | (e << 16));
}

__global__ void __launch_bounds__(kThreads, 1)
gemv_tc_kernel(const __grid_constant__ CUtensorMap qmap, __half* __restrict__ Y, const Params p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int S = p.stages;
  uint8_t* xs = smem;                                   // S x kXBytes (1024-aligned)
  uint8_t* ws_ = xs + (size_t)S * kXBytes;              // S x kWBytes (1024-aligned)
  uint8_t* cs = ws_ + (size_t)S * kWBytes;              // S x kCBytes
  uint8_t* ss = cs + (size_t)S * kCBytes;               // S x kSBytes
  uint64_t* fullS = reinterpret_cast<uint64_t*>(ss + (size_t)S * kSBytes);
  uint64_t* emptyS = fullS + S;
  uint64_t* aFull = emptyS + S;       // [2]
  uint64_t* aEmpty = aFull + 2;       // [2]
  uint64_t* dFull = aEmpty + 2;       // [2]
  uint64_t* dEmpty = dFull + 2;       // [2]
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(dEmpty + 2);
  volatile int* s_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const long long U = p.U, G = p.G;
  const long long u0 = range_start(blockIdx.x, U, G), u1 = range_start(blockIdx.x + 1, U, G);
  const long long n = u1 - u0;
  const int B = p.B;

  if (threadIdx.x == 0) {
    for (int s = 0; s < S; ++s) {
      ptx::mbar_init(&fullS[s], 1);
      ptx::mbar_init(&emptyS[s], 1 + kDecWarps);
    }
    for (int i = 0; i < 2; ++i) {
      ptx::mbar_init(&aFull[i], kDecWarps);
      ptx::mbar_init(&aEmpty[i], 1);
      ptx::mbar_init(&dFull[i], 1);
      ptx::mbar_init(&dEmpty[i], kDecWarps);
    }
    ptx::fence_mbar_init();
  }
  if (warp == 1) {
    ptx::tmem_alloc(tmem_slot, kTmemCols);
    ptx::tmem_relinquish();
  }
  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      ptx::prefetch_tensormap(&qmap);
      const uint64_t pol = ptx::policy_evict_first();
      const uint32_t tx = kWBytes + kXBytes + kCBytes + kSBytes;
      const long long pre = n < S ? n : S;
      uint32_t limit = kWaitLimit;
      for (long long i = 0; i < pre; ++i) {      // weights do not depend on the prep kernel
        const long long u = u0 + i;
        ptx::mbar_arrive_expect_tx(&fullS[i], tx);
        ptx::tma_load_2d(ws_ + i * kWBytes, &qmap, (int)(u % B) * 64, (int)(u / B) * kRows, &fullS[i], pol);
      }
      ptx::griddep_wait();
      for (long long i = 0; i < pre; ++i) {
        const long long u = u0 + i;
        const int b = (int)(u % B), rt = (int)(u / B);
        ptx::bulk_load(xs + i * kXBytes, p.xt + (size_t)b * kXBytes, kXBytes, &fullS[i]);
        ptx::bulk_load(cs + i * kCBytes, p.bias + (size_t)b * kNB, kCBytes, &fullS[i]);
        ptx::bulk_load(ss + i * kSBytes, p.dT + (size_t)b * p.Npad + (size_t)rt * kRows, kSBytes, &fullS[i]);
      }
      int s = (int)(pre % S);
      uint32_t ph = (uint32_t)((pre / S) & 1);
      int b = (int)((u0 + pre) % B), rt = (int)((u0 + pre) / B);
      for (long long i = pre; i < n; ++i) {
        if (!ptx::mbar_wait(&emptyS[s], ph ^ 1u, limit)) {
          atomicExch(p.error, 21u);
          limit = 1;
        }
        ptx::mbar_arrive_expect_tx(&fullS[s], tx);
        ptx::tma_load_2d(ws_ + (size_t)s * kWBytes, &qmap, b * 64, rt * kRows, &fullS[s], pol);
        ptx::bulk_load(xs + (size_t)s * kXBytes, p.xt + (size_t)b * kXBytes, kXBytes, &fullS[s]);
        ptx::bulk_load(cs + (size_t)s * kCBytes, p.bias + (size_t)b * kNB, kCBytes, &fullS[s]);
        ptx::bulk_load(ss + (size_t)s * kSBytes, p.dT + (size_t)b * p.Npad + (size_t)rt * kRows, kSBytes,
                       &fullS[s]);
        if (++s == S) { s = 0; ph ^= 1u; }
        if (++b == B) { b = 0; ++rt; }
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      const uint32_t idesc = (1u << 4)                            // D: f32
                             | ((uint32_t)(kNB >> 3) << 17)        // N = 16
                             | ((uint32_t)(kRows >> 4) << 24);     // M = 128; A, B: f16, K-major
      uint32_t limit = kWaitLimit;
      const uint32_t xs_u = ptx::smem_u32(xs);
      int s = 0;
      uint32_t ph = 0;
      for (long long i = 0; i < n; ++i) {
        const int ab = (int)(i & 1);
        const uint32_t aph = (uint32_t)((i >> 1) & 1);
        bool ok = ptx::mbar_wait(&fullS[s], ph, limit);
        ok = ptx::mbar_wait(&aFull[ab], aph, limit) && ok;
        if (i >= 2) ok = ptx::mbar_wait(&dEmpty[ab], aph ^ 1u, limit) && ok;
        if (!ok) {
          atomicExch(p.error, 22u);
          limit = 1;
        }
        ptx::tc_fence_after();
        const uint32_t xb = xs_u + (uint32_t)(s * kXBytes);
        const uint32_t a_tm = tmem + (uint32_t)(ab * kACols);
        const uint32_t d_tm = tmem + (uint32_t)(kDCol0 + ab * kNB);
#pragma unroll
        for (int k16 = 0; k16 < 16; ++k16) {
          const uint64_t bd = ptx::sw128_kmajor_desc(xb + (uint32_t)((k16 >> 2) * (kNB * 128))) +
                              (uint64_t)(2 * (k16 & 3));
          ptx::umma_f16_ts(d_tm, a_tm + (uint32_t)(8 * k16), bd, idesc, k16 > 0 ? 1u : 0u);
        }
        ptx::umma_commit(&emptyS[s]);
        ptx::umma_commit(&aEmpty[ab]);
        ptx::umma_commit(&dFull[ab]);
        if (++s == S) { s = 0; ph ^= 1u; }
      }
    }
  } else {
    // ------------------------------------------------------------ decoders + epilogue
    const int q4 = warp & 3;
    const int r = 32 * q4 + lane;                  // row within the unit = TMEM lane
    const uint32_t lane_base = tmem + ((uint32_t)(32 * q4) << 16);
    const uint32_t ws_u = ptx::smem_u32(ws_), cs_u = ptx::smem_u32(cs);
    uint32_t limit = kWaitLimit;
    float acc[kNB];
#pragma unroll
    for (int m = 0; m < kNB; ++m) acc[m] = 0.f;
    float cb[kNB], cb_prev[kNB];
    float dv = 0.f, dv_prev = 0.f;
    int s = 0;
    uint32_t ph = 0;
    int b = (int)(u0 % B), rt = (int)(u0 / B);
    int seg_b0 = b;
    int prev_b = b, prev_rt = rt;

    // epilogue of unit j: fold block partial into registers; finish segments
    auto retire = [&](long long j, int jb, int jrt) {
      const int db = (int)(j & 1);
      const uint32_t dph = (uint32_t)((j >> 1) & 1);
      if (!ptx::mbar_wait(&dFull[db], dph, limit)) {
        atomicExch(p.error, 23u);
        limit = 1;
      }
      ptx::tc_fence_after();
      uint32_t v[kNB];
      ptx::tmem_ld_32x32b_x16(lane_base + (uint32_t)(kDCol0 + db * kNB), v);
      ptx::tmem_ld_wait();
      ptx::tc_fence_before();
      __syncwarp();
      if (lane == 0) ptx::mbar_arrive(&dEmpty[db]);
#pragma unroll
      for (int m = 0; m < kNB; ++m) acc[m] = fmaf(dv_prev, __uint_as_float(v[m]) - cb_prev[m], acc[m]);
      const long long u = u0 + j;
      if (jb != B - 1 && u != u1 - 1) return;
      const int row = jrt * kRows + r;
      const bool whole = (seg_b0 == 0 && jb == B - 1);
      if (whole) {
        if (row < p.N) {
#pragma unroll
          for (int m = 0; m < kNB; ++m)
            if (m < p.M) Y[(size_t)m * p.N + row] = __float2half_rn(acc[m]);
        }
      } else {
        const int slot = (jrt == (int)(u0 / B)) ? 0 : 1;
        float4* mine = reinterpret_cast<float4*>(p.partials + (((size_t)blockIdx.x * 2 + slot) * kRows + r) * kNB);
#pragma unroll
        for (int q = 0; q < kNB / 4; ++q) mine[q] = make_float4(acc[4 * q], acc[4 * q + 1], acc[4 * q + 2], acc[4 * q + 3]);
        __threadfence();
        ptx::named_bar_sync(1, kDecWarps * 32);
        const long long cfirst = cta_of_unit((long long)jrt * B, U, G);
        const long long clast = cta_of_unit((long long)jrt * B + B - 1, U, G);
        if (warp == 2 && lane == 0) {
          const unsigned old = atomicAdd(&p.counters[jrt], 1u);
          *s_flag = (old == (unsigned)(clast - cfirst)) ? 1 : 0;
        }
        ptx::named_bar_sync(1, kDecWarps * 32);
        if (*s_flag) {
          __threadfence();
          float sum[kNB];
#pragma unroll
          for (int m = 0; m < kNB; ++m) sum[m] = 0.f;
          for (long long cc = cfirst; cc <= clast; ++cc) {
            const int sl = (jrt == (int)(range_start(cc, U, G) / B)) ? 0 : 1;
            const float4* src = reinterpret_cast<const float4*>(p.partials + (((size_t)cc * 2 + sl) * kRows + r) * kNB);
#pragma unroll
            for (int q = 0; q < kNB / 4; ++q) {
              const float4 f = __ldcg(src + q);
              sum[4 * q] += f.x; sum[4 * q + 1] += f.y; sum[4 * q + 2] += f.z; sum[4 * q + 3] += f.w;
            }
          }
          if (row < p.N) {
#pragma unroll
            for (int m = 0; m < kNB; ++m)
              if (m < p.M) Y[(size_t)m * p.N + row] = __float2half_rn(sum[m]);
          }
          if (warp == 2 && lane == 0) p.counters[jrt] = 0u;
        }
      }
#pragma unroll
      for (int m = 0; m < kNB; ++m) acc[m] = 0.f;
    };

    for (long long i = 0; i < n; ++i) {
      const int ab = (int)(i & 1);
      const uint32_t aph = (uint32_t)((i >> 1) & 1);
      if (!ptx::mbar_wait(&fullS[s], ph, limit)) {
        atomicExch(p.error, 24u);
        limit = 1;
      }
      // this row's 64 packed bytes (64-byte swizzle: chunk q sits at q ^ ((r >> 1) & 3))
      uint32_t w[16];
      const uint32_t rowp = ws_u + (uint32_t)(s * kWBytes + r * 64);
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const uint4 v = ptx::lds128(rowp + (uint32_t)(((q ^ ((r >> 1) & 3)) * 16)));
        w[4 * q] = v.x; w[4 * q + 1] = v.y; w[4 * q + 2] = v.z; w[4 * q + 3] = v.w;
      }
#pragma unroll
      for (int q = 0; q < kNB / 4; ++q) {
        const uint4 v = ptx::lds128(cs_u + (uint32_t)(s * kCBytes + 16 * q));
        cb[4 * q] = __uint_as_float(v.x); cb[4 * q + 1] = __uint_as_float(v.y);
        cb[4 * q + 2] = __uint_as_float(v.z); cb[4 * q + 3] = __uint_as_float(v.w);
      }
      dv = __half2float(reinterpret_cast<const __half*>(ss + (size_t)s * kSBytes)[r]);
      __syncwarp();
      if (lane == 0) ptx::mbar_arrive(&emptyS[s]);
      if (++s == S) { s = 0; ph ^= 1u; }
      // decoded block -> TMEM (A operand), once the MMAs two units back are done
      if (i >= 2 && !ptx::mbar_wait(&aEmpty[ab], aph ^ 1u, limit)) {
        atomicExch(p.error, 25u);
        limit = 1;
      }
      ptx::tc_fence_after();
#pragma unroll
      for (int c4 = 0; c4 < 4; ++c4) {
        uint32_t a[32];
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const uint32_t wv = w[4 * c4 + q], wh = wv >> 8;
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            a[8 * q + j] = decode_pair(wv, j);
            a[8 * q + 4 + j] = decode_pair(wh, j);
          }
        }
        ptx::tmem_st_32x32b_x32(lane_base + (uint32_t)(ab * kACols + 32 * c4), a);
      }
      ptx::tmem_st_wait();
      ptx::tc_fence_before();
      __syncwarp();
      if (lane == 0) ptx::mbar_arrive(&aFull[ab]);
      if (i > 0) retire(i - 1, prev_b, prev_rt);
      if (i == 0 || b == 0) seg_b0 = b;
#pragma unroll
      for (int m = 0; m < kNB; ++m) cb_prev[m] = cb[m];
      dv_prev = dv;
      prev_b = b;
      prev_rt = rt;
      if (++b == B) { b = 0; ++rt; }
    }
    if (n > 0) retire(n - 1, prev_b, prev_rt);
  }
  ptx::tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    ptx::tc_fence_after();
    ptx::tmem_dealloc(tmem, kTmemCols);
  }
}

// ---------------------------------------------------------------- host side
struct Layout {
  size_t off_err, off_cnt, off_xt, off_bias, off_dt, off_part, total;
  int64_t Npad, T, G, B;
};

size_t up256(size_t x) { return (x + 255) & ~size_t(255); }

Layout layout_for(int64_t N, int64_t K, int num_sms) {
  Layout L;
  L.B = K / kBlock;
  L.T = ceil_div(N, kRows);
  const int64_t U = L.T * L.B;
  L.G = U < num_sms ? U : num_sms;
  L.Npad = L.T * kRows;
  L.off_err = 0;
  L.off_cnt = 256;
  L.off_xt = L.off_cnt + up256((size_t)L.T * 4);
  L.off_bias = L.off_xt + up256((size_t)L.B * kXBytes);
  L.off_dt = L.off_bias + up256((size_t)L.B * kCBytes);
  L.off_part = L.off_dt + up256((size_t)L.B * L.Npad * 2);
  L.total = L.off_part + up256((size_t)L.G * 2 * kRows * kNB * 4);
  return L;
}

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  if (!fn) {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(ptr);
  }
  return fn;
}

int stages_for() {
  const int per = kWBytes + kXBytes + kCBytes + kSBytes;
  int s = (kSmemBudget - 2048) / per;
  return s > 12 ? 12 : s;
}

}  // namespace

size_t gemv_tc_ws_bytes(int64_t N, int64_t K, int num_sms) { return layout_for(N, K, num_sms).total; }

cudaError_t launch_gemv_tc(const __half* X, const uint8_t* qs, const __half* d, __half* Y, int M, int N,
                           int K, void* ws, int num_sms, cudaStream_t s) {
  if (M < 1 || M > kNB) return cudaErrorNotSupported;
  const Layout L = layout_for(N, K, num_sms);
  uint8_t* w = static_cast<uint8_t*>(ws);
  Params p;
  p.B = (int)L.B;
  p.T = (int)L.T;
  p.U = (long long)L.T * L.B;
  p.G = (int)L.G;
  p.M = M; p.N = N; p.K = K;
  p.stages = stages_for();
  p.Npad = (int)L.Npad;
  p.xt = w + L.off_xt;
  p.bias = reinterpret_cast<const float*>(w + L.off_bias);
  p.dT = reinterpret_cast<const __half*>(w + L.off_dt);
  p.partials = reinterpret_cast<float*>(w + L.off_part);
  p.counters = reinterpret_cast<unsigned*>(w + L.off_cnt);
  p.error = reinterpret_cast<unsigned*>(w + L.off_err);

  auto enc = encode_fn();
  if (!enc) return cudaErrorNotSupported;
  CUtensorMap map;
  const cuuint64_t gdim[2] = {(cuuint64_t)(K / 4), (cuuint64_t)N};
  const cuuint64_t gstride[1] = {(cuuint64_t)(K / 4)};
  const cuuint32_t box[2] = {64, (cuuint32_t)kRows};
  const cuuint32_t estr[2] = {1, 1};
  if (enc(&map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<uint8_t*>(qs), gdim, gstride, box, estr,
          CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_64B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
          CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
    return cudaErrorInvalidValue;

  xprep_tc_kernel<<<p.B + p.Npad / 64, 256, 0, s>>>(X, d, M, N, K, p.B, p.Npad, w + L.off_xt,
                                                    reinterpret_cast<float*>(w + L.off_bias),
                                                    reinterpret_cast<__half*>(w + L.off_dt), p.counters, p.T);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  const int S = p.stages;
  const size_t smem = (size_t)S * (kWBytes + kXBytes + kCBytes + kSBytes) + (2 * S + 8) * 8 + 16 + 1024;
  e = cudaFuncSetAttribute(gemv_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)p.G);
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, gemv_tc_kernel, map, Y, p);
}

}  // namespace tri
