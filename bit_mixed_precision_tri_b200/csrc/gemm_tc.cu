// Compute-regime ternary GEMM (M >= 17) for TQ2 weights on sm_100a.
//
// Y = X (d * W_hat)^T ("Scaling Laws and Efficient Inference for Ternary
// Language Models", section "The model", step 3) once the batch is large
// enough that arithmetic, not weight traffic, bounds the layer (section
// "TriRun: ternary inference on GPUs": the speedup falls once the product
// becomes compute-bound).  The pages' kernel used mma.sync; this one uses the
// fifth-generation tensor cores:
//
//  * a producer thread TMA-loads, per 64-wide K step, the activation tile
//    (128 rows x 64 fp16, 128-byte swizzle) and the packed weight tile
//    (BN rows x 16 bytes) into a ring of mbarrier-tracked stages;
//  * BN/32 decoder warps (one weight row per thread) turn sixteen 2-bit
//    fields per 32-bit word into exact fp16 values t * d (mask + OR with an
//    fp16 exponent, subtract the bias, multiply by the block scale) and
//    store them as the K-major, 128-byte-swizzled B operand;
//  * one thread issues tcgen05.mma (M = 128, N = BN, K = 16, fp32 accumulate)
//    with both operands in shared memory and the accumulator in tensor
//    memory, and frees stages with tcgen05.commit;
//  * the decoder warps finally read the accumulator with tcgen05.ld and
//    write fp16 Y (or fp32 partials when K is split across CTAs; the last
//    CTA of a tile sums them in split order, so results are deterministic).
//
// The decode emits the pairs (w_j, w_{j+8}) of each 16-weight word, so the
// activations are consumed in the same within-16 order: a prep kernel writes
// X once per call in that order (pairs (x_j, x_{j+8}) adjacent) and zeroes
// the split-K tickets; it is chained to the main kernel with programmatic
// dependent launch.
#include <cstdlib>

#include <cudaTypedefs.h>

#include "sm100_ptx.cuh"
#include "tri_internal.cuh"

namespace tri {
namespace {

constexpr int BM = 128;   // activation rows per tile (MMA M)
constexpr int BK = 64;    // K per stage: one 128-byte swizzle row of fp16
constexpr uint32_t kWaitLimit = 1u << 22;

template <int BN>
struct Cfg {
  static constexpr int DW = BN / 32;                 // decoder / epilogue warps
  static constexpr int kThreads = (2 + DW) * 32;
  static constexpr int kXBytes = BM * BK * 2;        // 16 KB
  static constexpr int kDBytes = BN * BK * 2;        // decoded fp16 weight tile
  static constexpr int kPBytes = BN * BK / 4;        // packed 2-bit weight tile
  static constexpr int kStages = (BN == 256) ? 4 : 6;
  static constexpr int kSmem = kStages * (kXBytes + kDBytes + kPBytes) + 1024 + 512;
};

struct TcParams {
  float* partials;      // [tiles][splits][BM][BN]
  unsigned* counters;   // [tiles]
  unsigned* error;
  int M, N, K, B, ksteps, splits, tiles_n;
};

// ---------------------------------------------------------------- prep kernel
__global__ void __launch_bounds__(256)
xperm_kernel(const __half* __restrict__ X, int64_t groups, __half* __restrict__ Xp,
             unsigned* __restrict__ tickets, int ntickets) {
  ptx::griddep_launch_dependents();
  if (blockIdx.x == 0)    // split-K tickets start at zero on every call
    for (int i = threadIdx.x; i < ntickets; i += blockDim.x) tickets[i] = 0u;
  const int64_t stride = (int64_t)gridDim.x * blockDim.x;
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < groups; i += stride) {
    const uint4* src = reinterpret_cast<const uint4*>(X) + 2 * i;
    const uint4 lo = src[0], hi = src[1];
    const uint32_t lw[4] = {lo.x, lo.y, lo.z, lo.w}, hw[4] = {hi.x, hi.y, hi.z, hi.w};
    uint32_t pr[8];
#pragma unroll
    for (int j = 0; j < 8; ++j) pr[j] = __byte_perm(lw[j >> 1], hw[j >> 1], (j & 1) ? 0x7632 : 0x5410);
    uint4* dst = reinterpret_cast<uint4*>(Xp) + 2 * i;
    dst[0] = make_uint4(pr[0], pr[1], pr[2], pr[3]);
    dst[1] = make_uint4(pr[4], pr[5], pr[6], pr[7]);
  }
}

// (beta_j + d') pair from field position j of both halves, then exact t * d
__device__ __forceinline__ uint32_t decode_scaled(uint32_t w, int j, __half2 dd) {
  const uint32_t mask = 0x00030003u << (2 * j);
  const uint32_t e = (j == 0) ? 0x6400u : (j == 1) ? 0x5C00u : (j == 2) ? 0x5400u : 0x4C00u;
  const uint32_t b1 = (j == 0) ? 0x6401u : (j == 1) ? 0x5C04u : (j == 2) ? 0x5410u : 0x4C40u;
  const uint32_t h = (w & mask) | (e | (e << 16));
  __half2 hv = *reinterpret_cast<const __half2*>(&h);
  const uint32_t bb = b1 | (b1 << 16);
  const __half2 bias = *reinterpret_cast<const __half2*>(&bb);
  __half2 t = __hsub2(hv, bias);          // exactly d' - 1
  t = __hmul2(t, dd);                     // exactly t * d
  return *reinterpret_cast<uint32_t*>(&t);
}

template <int BN>
__global__ void __launch_bounds__(Cfg<BN>::kThreads, 1)
gemm_tc_kernel(const __grid_constant__ CUtensorMap xmap, const __grid_constant__ CUtensorMap qmap,
               const __half* __restrict__ dsc, __half* __restrict__ Y, const TcParams p) {
  using C = Cfg<BN>;
  constexpr int S = C::kStages;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* xs = smem;                                   // S x kXBytes (1024-aligned)
  uint8_t* ds = xs + S * C::kXBytes;                    // S x kDBytes (1024-aligned)
  uint8_t* ps = ds + S * C::kDBytes;                    // S x kPBytes
  uint64_t* full = reinterpret_cast<uint64_t*>(ps + S * C::kPBytes);
  uint64_t* dec = full + S;
  uint64_t* empty = dec + S;
  uint64_t* accf = empty + S;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(accf + 1);
  volatile int* s_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int n_tile = blockIdx.x, m_tile = blockIdx.y, split = blockIdx.z;
  const int ks0 = (int)((int64_t)p.ksteps * split / p.splits);
  const int ks1 = (int)((int64_t)p.ksteps * (split + 1) / p.splits);
  const int nks = ks1 - ks0;

  if (threadIdx.x == 0) {
    for (int s = 0; s < S; ++s) {
      ptx::mbar_init(&full[s], 1);
      ptx::mbar_init(&dec[s], C::DW);
      ptx::mbar_init(&empty[s], 1);
    }
    ptx::mbar_init(accf, 1);
    ptx::fence_mbar_init();
  }
  if (warp == 1) {
    ptx::tmem_alloc(tmem_slot, BN);
    ptx::tmem_relinquish();
  }
  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      ptx::prefetch_tensormap(&xmap);
      ptx::prefetch_tensormap(&qmap);
      const uint64_t pol_w = ptx::policy_evict_first();
      uint64_t pol_x;
      asm volatile("createpolicy.fractional.L2::evict_last.b64 %0, 1.0;" : "=l"(pol_x));
      uint32_t limit = kWaitLimit;
      ptx::griddep_wait();      // activations are written by the prep kernel
      for (int i = 0; i < nks; ++i) {
        const int s = i % S;
        const uint32_t ph = (uint32_t)((i / S) & 1);
        if (i >= S && !ptx::mbar_wait(&empty[s], ph ^ 1u, limit)) {
          atomicExch(p.error, 11u);
          limit = 1;
        }
        const int ks = ks0 + i;
        ptx::mbar_arrive_expect_tx(&full[s], C::kXBytes + C::kPBytes);
        ptx::tma_load_2d(xs + s * C::kXBytes, &xmap, ks * BK, m_tile * BM, &full[s], pol_x);
        ptx::tma_load_2d(ps + s * C::kPBytes, &qmap, ks * (BK / 4), n_tile * BN, &full[s], pol_w);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      const uint32_t idesc = (1u << 4)                  // D: f32
                             | ((uint32_t)(BN >> 3) << 17)  // N
                             | ((uint32_t)(BM >> 4) << 24); // M ; A, B: f16, K-major
      uint32_t limit = kWaitLimit;
      for (int i = 0; i < nks; ++i) {
        const int s = i % S;
        const uint32_t ph = (uint32_t)((i / S) & 1);
        if (!ptx::mbar_wait(&dec[s], ph, limit) || !ptx::mbar_wait(&full[s], ph, limit)) {
          atomicExch(p.error, 12u);
          limit = 1;
        }
        ptx::tc_fence_after();
        const uint64_t a0 = ptx::sw128_kmajor_desc(ptx::smem_u32(xs + s * C::kXBytes));
        const uint64_t b0 = ptx::sw128_kmajor_desc(ptx::smem_u32(ds + s * C::kDBytes));
#pragma unroll
        for (int k = 0; k < BK / 16; ++k)
          ptx::umma_f16_ss(tmem, a0 + 2 * k, b0 + 2 * k, idesc, (i > 0 || k > 0) ? 1u : 0u);
        ptx::umma_commit(&empty[s]);
      }
      ptx::umma_commit(accf);
    }
  } else {
    // ------------------------------------------------------------ decoders
    const int r = (warp - 2) * 32 + lane;            // weight row within the tile
    const int n = n_tile * BN + r;
    const uint32_t ps_u = ptx::smem_u32(ps), ds_u = ptx::smem_u32(ds);
    uint32_t limit = kWaitLimit;
    __half2 dd = __float2half2_rn(0.f);
    for (int i = 0; i < nks; ++i) {
      const int s = i % S;
      const uint32_t ph = (uint32_t)((i / S) & 1);
      const int ks = ks0 + i;
      if (i == 0 || (ks & 3) == 0) {
        const __half dv = n < p.N ? __ldg(dsc + (size_t)n * p.B + (ks >> 2)) : __float2half(0.f);
        dd = __halves2half2(dv, dv);
      }
      if (!ptx::mbar_wait(&full[s], ph, limit)) {
        atomicExch(p.error, 13u);
        limit = 1;
      }
      const uint4 pw = ptx::lds128(ps_u + (uint32_t)(s * C::kPBytes + r * 16));
      const uint32_t w4[4] = {pw.x, pw.y, pw.z, pw.w};
      const uint32_t row_base = ds_u + (uint32_t)(s * C::kDBytes + r * 128);
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const uint32_t w = w4[q], wsh = w >> 8;
        const int c0 = (2 * q) ^ (r & 7), c1 = (2 * q + 1) ^ (r & 7);
        ptx::sts128(row_base + c0 * 16, decode_scaled(w, 0, dd), decode_scaled(w, 1, dd),
                    decode_scaled(w, 2, dd), decode_scaled(w, 3, dd));
        ptx::sts128(row_base + c1 * 16, decode_scaled(wsh, 0, dd), decode_scaled(wsh, 1, dd),
                    decode_scaled(wsh, 2, dd), decode_scaled(wsh, 3, dd));
      }
      ptx::fence_proxy_async();
      __syncwarp();
      if (lane == 0) ptx::mbar_arrive(&dec[s]);
    }
    // ------------------------------------------------------------ epilogue
    if (!ptx::mbar_wait(accf, 0, limit)) atomicExch(p.error, 14u);
    ptx::tc_fence_after();
    const int quarter = warp & 3;
    constexpr int kColsPerWarp = BN / (C::DW / 4);
    const int col_base = ((warp - 2) / 4) * kColsPerWarp;
    const int m = m_tile * BM + 32 * quarter + lane;
    const int tile = m_tile * p.tiles_n + n_tile;
    for (int j = 0; j < kColsPerWarp / 32; ++j) {
      const int col0 = col_base + 32 * j;
      uint32_t v[32];
      ptx::tmem_ld_32x32b_x32(tmem + ((uint32_t)(32 * quarter) << 16) + (uint32_t)col0, v);
      ptx::tmem_ld_wait();
      const int n0 = n_tile * BN + col0;
      if (p.splits == 1) {
        if (m < p.M) {
          __half* yrow = Y + (size_t)m * p.N + n0;
          if ((p.N & 7) == 0 && n0 + 32 <= p.N) {
#pragma unroll
            for (int q = 0; q < 4; ++q) {
              uint32_t h[4];
#pragma unroll
              for (int e = 0; e < 4; ++e) {
                __half2 t = __floats2half2_rn(__uint_as_float(v[8 * q + 2 * e]),
                                              __uint_as_float(v[8 * q + 2 * e + 1]));
                h[e] = *reinterpret_cast<uint32_t*>(&t);
              }
              reinterpret_cast<uint4*>(yrow)[q] = make_uint4(h[0], h[1], h[2], h[3]);
            }
          } else {
            for (int e = 0; e < 32; ++e)
              if (n0 + e < p.N) yrow[e] = __float2half_rn(__uint_as_float(v[e]));
          }
        }
      } else {
        float* part = p.partials + (((size_t)tile * p.splits + split) * BM + 32 * quarter + lane) * BN + col0;
#pragma unroll
        for (int q = 0; q < 8; ++q)
          reinterpret_cast<float4*>(part)[q] =
              make_float4(__uint_as_float(v[4 * q]), __uint_as_float(v[4 * q + 1]),
                          __uint_as_float(v[4 * q + 2]), __uint_as_float(v[4 * q + 3]));
      }
    }
    if (p.splits > 1) {
      __threadfence();
      ptx::named_bar_sync(1, C::DW * 32);
      if (warp == 2 && lane == 0) {
        const unsigned old = atomicAdd(&p.counters[tile], 1u);
        *s_flag = (old == (unsigned)(p.splits - 1)) ? 1 : 0;
      }
      ptx::named_bar_sync(1, C::DW * 32);
      if (*s_flag) {
        __threadfence();
        for (int j = 0; j < kColsPerWarp / 32; ++j) {
          const int col0 = col_base + 32 * j;
          const int n0 = n_tile * BN + col0;
          float acc[32];
#pragma unroll
          for (int e = 0; e < 32; ++e) acc[e] = 0.f;
          for (int sp = 0; sp < p.splits; ++sp) {
            const float4* src = reinterpret_cast<const float4*>(
                p.partials + (((size_t)tile * p.splits + sp) * BM + 32 * quarter + lane) * BN + col0);
#pragma unroll
            for (int q = 0; q < 8; ++q) {
              const float4 f = __ldcg(src + q);
              acc[4 * q] += f.x; acc[4 * q + 1] += f.y; acc[4 * q + 2] += f.z; acc[4 * q + 3] += f.w;
            }
          }
          if (m < p.M) {
            __half* yrow = Y + (size_t)m * p.N + n0;
            for (int e = 0; e < 32; ++e)
              if (n0 + e < p.N) yrow[e] = __float2half_rn(acc[e]);
          }
        }
        if (warp == 2 && lane == 0) p.counters[tile] = 0u;
      }
    }
  }
  ptx::tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    ptx::tc_fence_after();
    ptx::tmem_dealloc(tmem, BN);
  }
}

// ---------------------------------------------------------------- host side
size_t up256(size_t x) { return (x + 255) & ~size_t(255); }

struct Plan {
  int BN, splits, tiles_n, tiles_m;
  size_t off_err, off_cnt, off_xp, off_part, total;
};

Plan plan_for(int64_t M, int64_t N, int64_t K, int num_sms) {
  Plan pl;
  const int64_t tm = ceil_div(M, BM);
  const int64_t t128 = tm * ceil_div(N, 128), t256 = tm * ceil_div(N, 256);
  const char* env = std::getenv("TRI_TC_BN");
  int bn = env ? std::atoi(env) : 0;
  if (bn != 128 && bn != 256) bn = (t128 <= num_sms) ? 128 : 256;
  pl.BN = bn;
  const int64_t tiles = bn == 128 ? t128 : t256;
  const int64_t ksteps = K / BK;
  int64_t sp = tiles >= num_sms ? 1 : num_sms / tiles;
  const char* envs = std::getenv("TRI_TC_SPLITS");
  if (envs) sp = std::atoi(envs);
  if (sp < 1) sp = 1;
  if (sp > ksteps) sp = ksteps;
  if (sp > 16) sp = 16;
  pl.splits = (int)sp;
  pl.tiles_n = (int)ceil_div(N, bn);
  pl.tiles_m = (int)tm;
  pl.off_err = 0;
  pl.off_cnt = 256;
  pl.off_xp = pl.off_cnt + up256((size_t)tiles * 4);
  pl.off_part = pl.off_xp + up256((size_t)M * K * 2);
  pl.total = pl.off_part + (pl.splits > 1 ? up256((size_t)tiles * pl.splits * BM * bn * 4) : 0);
  return pl;
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

template <int BN>
cudaError_t launch_bn(const Plan& pl, const __half* X, const uint8_t* qs, const __half* d, __half* Y,
                      int M, int N, int K, void* ws, cudaStream_t s) {
  using C = Cfg<BN>;
  uint8_t* w = static_cast<uint8_t*>(ws);
  __half* Xp = reinterpret_cast<__half*>(w + pl.off_xp);
  auto enc = encode_fn();
  if (!enc) return cudaErrorNotSupported;
  CUtensorMap xmap, qmap;
  {
    const cuuint64_t gdim[2] = {(cuuint64_t)K, (cuuint64_t)M};
    const cuuint64_t gstr[1] = {(cuuint64_t)K * 2};
    const cuuint32_t box[2] = {BK, BM};
    const cuuint32_t es[2] = {1, 1};
    if (enc(&xmap, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, Xp, gdim, gstr, box, es,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return cudaErrorInvalidValue;
  }
  {
    const cuuint64_t gdim[2] = {(cuuint64_t)(K / 4), (cuuint64_t)N};
    const cuuint64_t gstr[1] = {(cuuint64_t)(K / 4)};
    const cuuint32_t box[2] = {BK / 4, (cuuint32_t)BN};
    const cuuint32_t es[2] = {1, 1};
    if (enc(&qmap, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<uint8_t*>(qs), gdim, gstr, box, es,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return cudaErrorInvalidValue;
  }
  const int64_t groups = (int64_t)M * K / 16;
  int64_t gx = ceil_div(groups, 256);
  if (gx > 148 * 8) gx = 148 * 8;
  xperm_kernel<<<(unsigned)gx, 256, 0, s>>>(X, groups, Xp, reinterpret_cast<unsigned*>(w + pl.off_cnt),
                                            pl.tiles_n * pl.tiles_m);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;

  TcParams p;
  p.partials = reinterpret_cast<float*>(w + pl.off_part);
  p.counters = reinterpret_cast<unsigned*>(w + pl.off_cnt);
  p.error = reinterpret_cast<unsigned*>(w + pl.off_err);
  p.M = M; p.N = N; p.K = K; p.B = K / kBlock; p.ksteps = K / BK; p.splits = pl.splits;
  p.tiles_n = pl.tiles_n;
  e = cudaFuncSetAttribute(gemm_tc_kernel<BN>, cudaFuncAttributeMaxDynamicSharedMemorySize, C::kSmem);
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)pl.tiles_n, (unsigned)pl.tiles_m, (unsigned)pl.splits);
  cfg.blockDim = dim3(C::kThreads);
  cfg.dynamicSmemBytes = C::kSmem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, gemm_tc_kernel<BN>, xmap, qmap, d, Y, p);
}

}  // namespace

bool gemm_tc_supported(int fmt, int64_t M, int64_t N, int64_t K) {
  return fmt == TRI_TQ2 && M >= 17 && N >= 1 && K >= kBlock && K % kBlock == 0 &&
         ceil_div(M, BM) <= 65535;
}

size_t gemm_tc_ws_bytes(int, int64_t M, int64_t N, int64_t K, int num_sms) {
  return plan_for(M, N, K, num_sms).total;
}

cudaError_t launch_gemm_tc(int fmt, const __half* X, const uint8_t* qs, const __half* d, __half* Y,
                           int M, int N, int K, void* ws, int num_sms, cudaStream_t s) {
  if (!gemm_tc_supported(fmt, M, N, K)) return cudaErrorNotSupported;
  const Plan pl = plan_for(M, N, K, num_sms);
  if (pl.BN == 256) return launch_bn<256>(pl, X, qs, d, Y, M, N, K, ws, s);
  return launch_bn<128>(pl, X, qs, d, Y, M, N, K, ws, s);
}

}  // namespace tri
