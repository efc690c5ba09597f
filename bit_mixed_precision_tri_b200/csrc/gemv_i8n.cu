// Decode-regime ternary GEMM for 3 <= M <= 16 activation rows (TQ2) on the
// integer tensor-core path: exact int8 products of the 2-bit weight fields
// with fixed-point activation digits, as for M <= 2, with more batch columns.
//
// Y = X (d * W_hat)^T ("Scaling Laws and Efficient Inference for Ternary
// Language Models", section "The model", step 3).  Up to batch 16 the layer
// is still bound by the packed weight bytes ("TriRun: ternary inference on
// GPUs": the speedup over fp16 holds up to batch 16), so products must cost
// few instructions per weight:
//
//  * Activations.  A prep kernel writes each 256-element block of X once per
//    call as 24-bit fixed point x = s x^ (|x^| <= 8e6, s per block and batch
//    row) in three balanced base-256 digits, directly in the per-lane order of
//    the B operand of mma.sync m16n8k32 (s8).  NT = 3 (M <= 8) or 6 (M <= 16)
//    tiles of 8 columns: column n of tile t is digit level (2t + n mod 2) mod 3
//    of batch row T (n / 2) + (2t + n mod 2) / 3, T = 2 NT / 3, so the columns
//    a thread holds in C (n = 2 tig, 2 tig + 1 of every tile) are all three
//    levels of T whole batch rows; with s and sum_k x^_k per block and row.
//  * Weights.  TMA loads one 256-wide block of a 128-row tile (8 KB, 64-byte
//    swizzle).  In a 32-bit word of sixteen fields, (w >> 2g) & 0x03030303 is
//    field g of four bytes, d' = t + 1 in {0, 1, 2} as unsigned bytes: the A
//    operand (16 rows x 32 bytes per warp).  The K order inside a block is
//    permuted so that every lane loads its A bytes with two 16-byte reads; the
//    prep kernel writes the activation digits in the same permuted order.
//  * Per block: sum_k t_k x_k = s (sum_k d'_k x^_k - sum_k x^_k); the three
//    digit columns are weighted 65536 / 256 / 1, scaled by s and the block
//    scale d[n][b], and accumulated per column in fp32; the columns of a batch
//    row are added at the end.  The one rounding of the method's arithmetic
//    is the activation quantisation (half a step, 2^-24 of the block's
//    largest |x|), as on the M <= 2 path.
//  * Split K.  A 128-row tile's blocks may be split over the CTAs of a
//    thread-block cluster; partial sums go through an L2-resident scratch and
//    rank 0 adds them in rank order after one cluster barrier: deterministic.
//  * SwiGLU epilogue (optional).  With gate and up rows interleaved in groups
//    of eight, the two rows a thread holds (r and r + 8) are the gate and up
//    projections of one output feature, and it writes silu(g) * u directly
//    (the feed-forward unit of "Scaling Laws and Efficient Inference for
//    Ternary Language Models", section "The model").
#include <cudaTypedefs.h>

#include "sm100_ptx.cuh"
#include "tri_internal.cuh"

namespace tri {
namespace {

constexpr int kRows = 128;                      // rows per tile (8 warps x 16)
constexpr int kConsumers = 8;
constexpr int kThreads = (kConsumers + 2) * 32; // + two producer warps
constexpr int kCtasPerSm = 2;
constexpr int kSmemBudget = 110 * 1024;         // two CTAs per SM
constexpr int kABytes = kRows * (kBlock / 4);   // 8 KB packed weights per block and tile
constexpr float kQMax = 8.0e6f;
constexpr uint32_t kWaitLimit = 1u << 18;   // mbarrier polls: ~4 us each when pending, ~1 s in all
constexpr int kMaxSplit = 8;

// activation record of one block: [ks 2][g 4][t NT][lane 32] uint2, then
// [s 16][sum 16] floats
__host__ __device__ constexpr int frag_bytes(int nt) { return 2 * 4 * nt * 32 * 8; }
__host__ __device__ constexpr int rec_bytes(int nt) { return frag_bytes(nt) + 32 * 4; }

struct NParams {
  const uint8_t* recs;     // [B] records
  float* scratch;          // [tile][rank][128][M]
  unsigned* error;
  int M, N, K, B, splits, stages;
  int swiglu;              // N = 2F fused gate/up rows, Y = silu(gate) * up, [M][F]
};

// ---------------------------------------------------------------- prep kernel
// One CTA of 256 threads per 256-element block.  Thread 16 m + (tig, ks, r)
// holds elements e = 64 tig + 32 ks + 16 r + (4 j + g), j, g < 4, of batch
// row m: exactly the bytes of the twelve record words (3 levels x 4 fields)
// that lane (gid, tig) of tile t reads as register r of step (ks, g), where
// (t, gid) is the column of (row m, level).  The block maximum of a row is a
// reduction over its 16 threads (half a warp).
template <int NT>
__global__ void __launch_bounds__(256)
i8n_prep_kernel(const __half* __restrict__ X, int M, int K, uint8_t* __restrict__ recs) {
  ptx::griddep_launch_dependents();
  ptx::griddep_wait();                         // X may be the previous kernel's output
  constexpr int T = 2 * NT / 3;
  const int b = blockIdx.x, m = threadIdx.x >> 4, sub = threadIdx.x & 15;
  const int tig = sub >> 2, ks = (sub >> 1) & 1, r = sub & 1;
  const int e0 = 64 * tig + 32 * ks + 16 * r;
  uint8_t* rec = recs + (size_t)b * rec_bytes(NT);
  float xv[16];
  if (m < M) {
    const uint4* src = reinterpret_cast<const uint4*>(X + (size_t)m * K + (size_t)b * kBlock + e0);
    const uint4 u0 = __ldg(src), u1 = __ldg(src + 1);
    const uint32_t hw[8] = {u0.x, u0.y, u0.z, u0.w, u1.x, u1.y, u1.z, u1.w};
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const float2 f = __half22float2(*reinterpret_cast<const __half2*>(&hw[i]));
      xv[2 * i] = f.x;
      xv[2 * i + 1] = f.y;
    }
  } else {
#pragma unroll
    for (int i = 0; i < 16; ++i) xv[i] = 0.f;
  }
  float amax = 0.f;
#pragma unroll
  for (int i = 0; i < 16; ++i) amax = fmaxf(amax, fabsf(xv[i]));
#pragma unroll
  for (int o = 8; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xFFFFFFFFu, amax, o));
  const float inv = amax > 0.f ? kQMax / amax : 0.f;
  // Balanced base-256 digits of q as bytes: with u = q + 0x808080 (in
  // [0, 2^24) for |q| <= 8e6), byte i of u ^ 0x808080 is digit i as a signed
  // byte.  Level l (0 = highest digit) of element 4 j + g goes to byte j of
  // wd[l][g].
  uint32_t dg[16];
  int sum = 0;
#pragma unroll
  for (int i = 0; i < 16; ++i) {
    const int q = __float2int_rn(xv[i] * inv);         // |q| <= 8e6 < 2^23
    sum += q;
    dg[i] = ((uint32_t)q + 0x808080u) ^ 0x808080u;
  }
  uint32_t wd[3][4];
#pragma unroll
  for (int l = 0; l < 3; ++l)
#pragma unroll
    for (int g = 0; g < 4; ++g) {
      const uint32_t sel = (uint32_t)(2 - l) | ((uint32_t)(6 - l) << 4);
      const uint32_t lo = __byte_perm(dg[g], dg[4 + g], sel), hi = __byte_perm(dg[8 + g], dg[12 + g], sel);
      wd[l][g] = __byte_perm(lo, hi, 0x5410);
    }
#pragma unroll
  for (int o = 8; o > 0; o >>= 1) sum += __shfl_xor_sync(0xFFFFFFFFu, sum, o);
  if (m < 8 * NT / 3) {                        // rows that have columns (all of them when NT = 6)
    uint32_t* out = reinterpret_cast<uint32_t*>(rec);
    const int mq = m % T, mgrp = m / T;        // row m = T (gid >> 1) + (2t + (gid & 1)) / 3
#pragma unroll
    for (int l = 0; l < 3; ++l) {
      const int cq = 3 * mq + l;               // = 2t + (gid & 1)
      const int t = cq >> 1, gid = 2 * mgrp + (cq & 1);
      const int L = 4 * gid + tig;
#pragma unroll
      for (int g = 0; g < 4; ++g) out[(((ks * 4 + g) * NT + t) * 32 + L) * 2 + r] = wd[l][g];
    }
  }
  if (sub == 0) {
    float* sc = reinterpret_cast<float*>(rec + frag_bytes(NT));
    sc[m] = amax > 0.f ? amax / kQMax : 0.f;   // s
    sc[16 + m] = (float)sum;                   // sum_k x^_k
  }
}

// silu(g) * u in fp32 (silu(g) = g / (1 + e^-g))
__device__ __forceinline__ float silu_mul(float g, float u) { return g / (1.f + expf(-g)) * u; }

// ---------------------------------------------------------------- main kernel
template <int NT>
__global__ void __launch_bounds__(kThreads, kCtasPerSm)
i8n_kernel(const __grid_constant__ CUtensorMap qmap, const __half* __restrict__ d, __half* __restrict__ Y,
           const NParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  constexpr int kRec = rec_bytes(NT);
  constexpr int kStage = kABytes + ((kRec + 1023) & ~1023);
  constexpr int T = 2 * NT / 3;                        // batch rows per thread
  const int S = p.stages;
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + (size_t)S * kStage);
  uint64_t* empty = full + S;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int gid = lane >> 2, tig = lane & 3;
  const int tile = blockIdx.x, split = blockIdx.z;
  const int b0 = (int)((int64_t)p.B * split / p.splits);
  const int nblk = (int)((int64_t)p.B * (split + 1) / p.splits) - b0;

  ptx::griddep_launch_dependents();
  if (threadIdx.x == 0) {
    for (int s = 0; s < S; ++s) {
      ptx::mbar_init(&full[s], 2);        // A bytes and activation record (two arrivals with tx)
      ptx::mbar_init(&empty[s], kConsumers);
    }
    ptx::fence_mbar_init();
  }
  __syncthreads();
  uint32_t limit = kWaitLimit;
  float y[T][2];                                       // [batch row][row half]
#pragma unroll
  for (int k = 0; k < T; ++k) y[k][0] = y[k][1] = 0.f;
  const int r0 = warp * 16 + gid;                      // rows r0 and r0 + 8 of the tile
  const int n0 = tile * kRows + r0, n1 = n0 + 8;

  if (warp >= kConsumers) {
    // ------------------------------------------------ producers: A by warp 8, records by warp 9
    if (lane == 0) {
      const bool is_a = warp == kConsumers;
      if (is_a) {
        ptx::prefetch_tensormap(&qmap);
      } else {
        ptx::griddep_wait();              // records come from the prep kernel
      }
      const uint64_t pol = ptx::policy_evict_first();
      int s = 0, round = 0;
      for (int j = 0; j < nblk; ++j) {
        if (round > 0 && !ptx::mbar_wait(&empty[s], (uint32_t)((round - 1) & 1), limit)) {
          ptx::record_wait_failure(p.error, 41u);
          limit = 1;
        }
        uint8_t* st = smem + (size_t)s * kStage;
        if (is_a) {
          ptx::mbar_arrive_expect_tx(&full[s], kABytes);
          ptx::tma_load_2d(st, &qmap, (b0 + j) * (kBlock / 4), tile * kRows, &full[s], pol);
        } else {
          ptx::mbar_arrive_expect_tx(&full[s], kRec);
          ptx::bulk_load(st + kABytes, p.recs + (size_t)(b0 + j) * kRec, kRec, &full[s]);
        }
        if (++s == S) { s = 0; ++round; }
      }
    }
  } else {
    // ------------------------------------------------ consumers
    const uint32_t sw0 = (uint32_t)((r0 >> 1) & 3), sw1 = (uint32_t)(((r0 + 8) >> 1) & 3);
    const unsigned short* dr0 = reinterpret_cast<const unsigned short*>(d) + (size_t)(n0 < p.N ? n0 : 0) * p.B + b0;
    const unsigned short* dr1 = reinterpret_cast<const unsigned short*>(d) + (size_t)(n1 < p.N ? n1 : 0) * p.B + b0;
    unsigned short dn0 = __ldg(dr0), dn1 = __ldg(dr1);
    unsigned short dm0 = nblk > 1 ? __ldg(dr0 + 1) : (unsigned short)0, dm1 = nblk > 1 ? __ldg(dr1 + 1) : (unsigned short)0;
    int s = 0;
    uint32_t ph = 0;
    for (int j = 0; j < nblk; ++j) {
      const float d0 = n0 < p.N ? __half2float(__ushort_as_half(dn0)) : 0.f;
      const float d1 = n1 < p.N ? __half2float(__ushort_as_half(dn1)) : 0.f;
      dn0 = dm0;
      dn1 = dm1;
      if (j + 2 < nblk) { dm0 = __ldg(dr0 + j + 2); dm1 = __ldg(dr1 + j + 2); }
      if (!ptx::mbar_wait(&full[s], ph, limit)) {
        ptx::record_wait_failure(p.error, 42u);
        limit = 1;
      }
      const uint32_t st = ptx::smem_u32(smem + (size_t)s * kStage);
      const uint4 wa = ptx::lds128(st + (uint32_t)(r0 * 64) + (((uint32_t)tig ^ sw0) << 4));
      const uint4 wb = ptx::lds128(st + (uint32_t)((r0 + 8) * 64) + (((uint32_t)tig ^ sw1) << 4));
      const uint32_t rec = st + kABytes;
      int c[NT][4];
#pragma unroll
      for (int kg = 0; kg < 8; ++kg) {
        const int ks = kg >> 2, g = kg & 3;
        uint2 bf[NT];
#pragma unroll
        for (int t = 0; t < NT; ++t) bf[t] = ptx::lds64(rec + (uint32_t)(((kg * NT + t) * 32 + lane) * 8));
        const uint32_t a0 = ks ? wa.z : wa.x, a2 = ks ? wa.w : wa.y;   // row r0, bytes 8ks + 0..3 / 4..7
        const uint32_t a1 = ks ? wb.z : wb.x, a3 = ks ? wb.w : wb.y;   // row r0 + 8
        const uint32_t m0 = (a0 >> (2 * g)) & 0x03030303u, m1 = (a1 >> (2 * g)) & 0x03030303u;
        const uint32_t m2 = (a2 >> (2 * g)) & 0x03030303u, m3 = (a3 >> (2 * g)) & 0x03030303u;
#pragma unroll
        for (int t = 0; t < NT; ++t) {
          if (kg == 0)
            asm volatile(
                "mma.sync.aligned.m16n8k32.row.col.s32.u8.s8.s32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
                "{%10,%10,%10,%10};"
                : "=r"(c[t][0]), "=r"(c[t][1]), "=r"(c[t][2]), "=r"(c[t][3])
                : "r"(m0), "r"(m1), "r"(m2), "r"(m3), "r"(bf[t].x), "r"(bf[t].y), "r"(0));
          else
            asm volatile(
                "mma.sync.aligned.m16n8k32.row.col.s32.u8.s8.s32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
                "{%0,%1,%2,%3};"
                : "+r"(c[t][0]), "+r"(c[t][1]), "+r"(c[t][2]), "+r"(c[t][3])
                : "r"(m0), "r"(m1), "r"(m2), "r"(m3), "r"(bf[t].x), "r"(bf[t].y));
        }
      }
      // batch row T tig + k: levels at (t, e) with 2t + e = 3k, 3k+1, 3k+2
      const float* sc = reinterpret_cast<const float*>(smem + (size_t)s * kStage + kABytes + frag_bytes(NT)) + T * tig;
#pragma unroll
      for (int k = 0; k < T; ++k) {
        const float sx = sc[k], sq = sc[16 + k];
        const int q0 = 3 * k, q1 = 3 * k + 1, q2 = 3 * k + 2;
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          const float v = fmaf((float)c[q0 >> 1][2 * h + (q0 & 1)], 65536.f,
                               fmaf((float)c[q1 >> 1][2 * h + (q1 & 1)], 256.f,
                                    (float)c[q2 >> 1][2 * h + (q2 & 1)] - sq));
          y[k][h] = fmaf(v, sx * (h ? d1 : d0), y[k][h]);
        }
      }
      __syncwarp();
      if (lane == 0) ptx::mbar_arrive(&empty[s]);
      if (++s == S) { s = 0; ph ^= 1u; }
    }
  }

  // ---------------------------------------------------------------- epilogue
  const int M = p.M;
  const int F = p.N / 2;
  if (p.splits == 1) {
    if (warp < kConsumers) {
#pragma unroll
      for (int k = 0; k < T; ++k) {
        const int m = T * tig + k;
        if (m >= M) continue;
        if (p.swiglu) {
          const int f = tile * (kRows / 2) + warp * 8 + gid;    // rows n0 (gate), n1 = n0 + 8 (up)
          if (n0 < p.N) Y[(size_t)m * F + f] = __float2half_rn(silu_mul(y[k][0], y[k][1]));
        } else {
          if (n0 < p.N) Y[(size_t)m * p.N + n0] = __float2half_rn(y[k][0]);
          if (n1 < p.N) Y[(size_t)m * p.N + n1] = __float2half_rn(y[k][1]);
        }
      }
    }
  } else {
    if (warp < kConsumers) {
      float* mine = p.scratch + ((size_t)tile * p.splits + split) * kRows * M;
#pragma unroll
      for (int k = 0; k < T; ++k) {
        const int m = T * tig + k;
        if (m < M) {
          mine[r0 * M + m] = y[k][0];
          mine[(r0 + 8) * M + m] = y[k][1];
        }
      }
    }
    ptx::cluster_sync();
    if (split == 0) {
      const float* base = p.scratch + (size_t)tile * p.splits * kRows * M;
      if (p.swiglu) {
        for (int i = threadIdx.x; i < (kRows / 2) * M; i += kThreads) {
          const int q = i / M, m = i % M, rg = 16 * (q >> 3) + (q & 7), f = tile * (kRows / 2) + q;
          float g = 0.f, u = 0.f;
          for (int sp = 0; sp < p.splits; ++sp) {
            g += __ldcg(base + (size_t)sp * kRows * M + rg * M + m);
            u += __ldcg(base + (size_t)sp * kRows * M + (rg + 8) * M + m);
          }
          if (tile * kRows + rg < p.N) Y[(size_t)m * F + f] = __float2half_rn(silu_mul(g, u));
        }
      } else {
        for (int i = threadIdx.x; i < kRows * M; i += kThreads) {
          const int r = i / M, m = i % M, n = tile * kRows + r;
          float v = 0.f;
          for (int sp = 0; sp < p.splits; ++sp) v += __ldcg(base + (size_t)sp * kRows * M + i);
          if (n < p.N) Y[(size_t)m * p.N + n] = __float2half_rn(v);
        }
      }
    }
  }
}

// ---------------------------------------------------------------- host side
int nt_for(int64_t M) { return M <= 8 ? 3 : 6; }

template <int NT>
int stages_for() {
  constexpr int kRec = rec_bytes(NT);
  constexpr int kStage = kABytes + ((kRec + 1023) & ~1023);
  int s = (kSmemBudget - 2048) / kStage;
  return s > 16 ? 16 : s;
}

template <int NT>
size_t smem_for(int S) {
  constexpr int kRec = rec_bytes(NT);
  constexpr int kStage = kABytes + ((kRec + 1023) & ~1023);
  return 1024 + (size_t)S * kStage + 2 * (size_t)S * 8;
}

struct NPlan {
  int NT, S, tiles, splits;
  size_t smem, off_rec, off_scr, total;
};

NPlan nplan(int64_t M, int64_t N, int64_t K, int num_sms) {
  NPlan pl;
  pl.NT = nt_for(M);
  if (pl.NT == 3) {
    pl.S = stages_for<3>(); pl.smem = smem_for<3>(pl.S);
  } else {
    pl.S = stages_for<6>(); pl.smem = smem_for<6>(pl.S);
  }
  pl.tiles = (int)ceil_div(N, kRows);
  const int64_t B = K / kBlock;
  // smallest split that fills the SMs in one wave (clusters of at most 8)
  int sp = 1;
  while (sp < kMaxSplit && sp < B && (int64_t)pl.tiles * (sp * 2) <= (int64_t)num_sms * kCtasPerSm) sp *= 2;
  pl.splits = sp;
  pl.off_rec = 0;
  pl.off_scr = pl.off_rec + (((size_t)B * rec_bytes(pl.NT) + 255) & ~size_t(255));
  pl.total = pl.off_scr + (sp > 1 ? (size_t)pl.tiles * sp * kRows * M * 4 : 0);
  return pl;
}

PFN_cuTensorMapEncodeTiled_v12000 encode_fn_n() {
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

template <int NT>
cudaError_t launch_nt(const NPlan& pl, const __half* X, const uint8_t* qs, const __half* d, __half* Y, int M,
                      int N, int K, void* ws, bool swiglu, cudaStream_t s) {
  uint8_t* w = static_cast<uint8_t*>(ws);
  auto enc = encode_fn_n();
  if (!enc) return cudaErrorNotSupported;
  CUtensorMap qmap;
  {
    const cuuint64_t gdim[2] = {(cuuint64_t)(K / 4), (cuuint64_t)N};
    const cuuint64_t gstr[1] = {(cuuint64_t)(K / 4)};
    const cuuint32_t box[2] = {kBlock / 4, kRows};
    const cuuint32_t es[2] = {1, 1};
    if (enc(&qmap, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<uint8_t*>(qs), gdim, gstr, box, es,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_64B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return cudaErrorInvalidValue;
  }
  const int B = K / kBlock;
  uint8_t* recs = w + pl.off_rec;
  {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)B);
    cfg.blockDim = dim3(256);
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    const cudaError_t e = cudaLaunchKernelEx(&cfg, i8n_prep_kernel<NT>, X, M, K, recs);
    if (e != cudaSuccess) return e;
  }
  static bool attr_done[16] = {};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 0 || dev >= 16 || !attr_done[dev]) {
    const cudaError_t e = cudaFuncSetAttribute(i8n_kernel<NT>, cudaFuncAttributeMaxDynamicSharedMemorySize, 232448);
    if (e != cudaSuccess) return e;
    if (dev >= 0 && dev < 16) attr_done[dev] = true;
  }
  NParams p;
  p.recs = recs;
  p.scratch = reinterpret_cast<float*>(w + pl.off_scr);
  const cudaError_t ew = wait_status_word(&p.error);
  if (ew != cudaSuccess) return ew;
  p.M = M; p.N = N; p.K = K; p.B = B; p.splits = pl.splits; p.stages = pl.S;
  p.swiglu = swiglu ? 1 : 0;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)pl.tiles, 1, (unsigned)pl.splits);
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = pl.smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  attr[1].id = cudaLaunchAttributeClusterDimension;
  attr[1].val.clusterDim.x = 1;
  attr[1].val.clusterDim.y = 1;
  attr[1].val.clusterDim.z = (unsigned)pl.splits;
  cfg.attrs = attr;
  cfg.numAttrs = pl.splits > 1 ? 2 : 1;
  return cudaLaunchKernelEx(&cfg, i8n_kernel<NT>, qmap, d, Y, p);
}

}  // namespace

bool gemv_i8n_supported(int64_t M, int64_t N, int64_t K) {
  return M >= 3 && M <= 16 && N >= 1 && K >= kBlock && K % kBlock == 0 && ceil_div(N, kRows) <= 65535;
}

size_t gemv_i8n_ws_bytes(int64_t M, int64_t N, int64_t K, int num_sms) {
  return nplan(M, N, K, num_sms).total;
}

cudaError_t launch_gemv_i8n(const __half* X, const uint8_t* qs, const __half* d, __half* Y, int M, int N, int K,
                            void* ws, int num_sms, cudaStream_t s, bool swiglu) {
  if (!gemv_i8n_supported(M, N, K)) return cudaErrorNotSupported;
  if (swiglu && N % 16 != 0) return cudaErrorNotSupported;
  const NPlan pl = nplan(M, N, K, num_sms);
  if (pl.NT == 3) return launch_nt<3>(pl, X, qs, d, Y, M, N, K, ws, swiglu, s);
  return launch_nt<6>(pl, X, qs, d, Y, M, N, K, ws, swiglu, s);
}

}  // namespace tri
