// Decode-regime ternary GEMM (M <= 16) for TQ2 weights on sm_100a.
//
// Computes Y = X (d * W_hat)^T ("Scaling Laws and Efficient Inference for
// Ternary Language Models", section "The model", step 3) when the batch is
// small enough that the kernel is bound by streaming the packed weights from
// HBM (section "TriRun: ternary inference on GPUs": 2-bit weights move 8x
// fewer bytes than fp16 while the product stays memory-bound).
//
// Design (B200):
//  * Work = (row tile of 256 rows) x (256-weight block) units, split over a
//    persistent grid of one CTA per SM as contiguous ranges (stream-K), so
//    every SM streams the same number of weight bytes for any N and K.
//  * One producer thread stages each unit with a 2-D TMA load of the packed
//    tile (256 rows x 64 bytes, L2 evict-first: each weight byte is used once)
//    plus a bulk copy of the block's prepared activations, into a ring of
//    mbarrier-tracked shared-memory stages.
//  * Eight consumer warps decode in registers and multiply on the tensor
//    cores with mma.sync m16n8k16 (fp16 x fp16 -> fp32): the weight tile is
//    the 16-row A operand, the batch (<= 8 or <= 16 columns) the B operand.
//  * Decode follows the "TriRun" dequantization idea (mask plus a three-input
//    logical op that sets an fp16 exponent in one step): for a 32-bit word of
//    sixteen 2-bit fields, (w & (0x00030003 << 2j)) | magic_j is the fp16 pair
//    (2^(10-2j) + d'_j, 2^(10-2j) + d'_{j+8}); the same on w >> 8 gives weights
//    j+4 and j+12.  Instead of a per-weight correction, the constant part
//    sum_k (2^(10-2j(k)) + 1) x_k is subtracted once per block and batch
//    column (computed with the activations), leaving sum_k t_k x_k.  Each
//    weight costs half a LOP3 plus 1/16 of a shift.
//  * The pairs (j, j+8) that one fp16x2 register holds fix which columns of
//    X the MMA's k index maps to; a small prep kernel writes X in that pair
//    order (and a bank-conflict-free swizzle) once per call, chained to the
//    main kernel with programmatic dependent launch.
//  * Partial sums of a row tile split across CTAs are combined by the last
//    CTA to finish (an atomic ticket, no waiting), in CTA order, so results
//    are deterministic.
#include <mutex>

#include <cudaTypedefs.h>

#include "sm100_ptx.cuh"
#include "tri_internal.cuh"

namespace tri {
namespace {

constexpr int kConsumerWarps = 8;
constexpr int kThreads = kConsumerWarps * 32;   // lane 0 of warp 0 also issues the copies
constexpr int kBoxRows = 256;                  // TMA box height
// 16-row mma tiles per consumer warp: four for batches up to 8 (one n8
// column block), two for batches up to 16 (two column blocks), which keeps
// both variants inside the register file without spills.
template <int MP> struct Unit {
  static constexpr int kTiles = MP == 8 ? 4 : 2;
  static constexpr int kWarpRows = 16 * kTiles;
  static constexpr int kRT = kWarpRows * kConsumerWarps;   // rows per unit
  static constexpr int kWBytes = kRT * 64;                 // packed bytes per unit
  static constexpr int kBoxes = kRT / kBoxRows;
};
constexpr uint32_t kWaitLimit = 1u << 18;   // mbarrier polls: ~4 us each when pending, ~1 s in all
constexpr int kSmemBudget = 220 * 1024;

struct Params {
  const uint4* xil;     // [B][MP][32] 16-byte units
  const float* bias;    // [B][MP]
  const __half* dT;     // [B][Npad] block scales, block-major (prepared per call)
  float* partials;      // [G][2][kRT][MP]
  unsigned* counters;   // [T]
  unsigned* error;      // [1]
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
// CTAs [0, B) write the activations of block b in the MMA's pair order (and a
// bank-conflict-free swizzle) plus the decode bias of each batch row; CTAs
// [B, B + Npad/64) transpose 64 rows of the scale plane d[N][B] into
// dT[B][Npad] so that a unit's scales are one contiguous bulk copy.
template <int MP>
__global__ void __launch_bounds__(MP * 16)
xprep_kernel(const __half* __restrict__ X, const __half* __restrict__ dsc, int M, int N, int K,
             int B, int Npad, uint4* __restrict__ xil, float* __restrict__ bias,
             __half* __restrict__ dT, unsigned* __restrict__ tickets, int T) {
  ptx::griddep_launch_dependents();
  // the main kernel's per-row-tile tickets start at zero on every call (the
  // workspace may hold another shape's data); it reads them only after data
  // that depends on this grid's completion has arrived
  if (blockIdx.x == 0)
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
  const int sw = (2 * (G >> 2) + (m & 1)) & 7;
  uint4* dst = xil + ((size_t)b * MP + m) * 32;
  dst[(2 * G + 0) ^ sw] = make_uint4(pr[0], pr[1], pr[2], pr[3]);
  dst[(2 * G + 1) ^ sw] = make_uint4(pr[4], pr[5], pr[6], pr[7]);
  // constant part of the magic-exponent decode: sum_i (2^(10-2(i%4)) + 1) x_i
  const float beta1[4] = {1025.f, 257.f, 65.f, 17.f};
  float s = 0.f;
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const float2 a = __half22float2(*reinterpret_cast<const __half2*>(&lw[i >> 1]));
    const float2 c = __half22float2(*reinterpret_cast<const __half2*>(&hw[i >> 1]));
    const float xi = (i & 1) ? a.y : a.x;          // x_i
    const float xj = (i & 1) ? c.y : c.x;          // x_{i+8}
    s = fmaf(beta1[i & 3], xi, s);
    s = fmaf(beta1[i & 3], xj, s);
  }
#pragma unroll
  for (int o = 8; o > 0; o >>= 1) s += __shfl_xor_sync(0xFFFFFFFFu, s, o);
  if (G == 0) bias[(size_t)b * MP + m] = s;
}

// ---------------------------------------------------------------- main kernel
__device__ __forceinline__ uint32_t decode_pair(uint32_t w, int j) {
  const uint32_t mask = 0x00030003u << (2 * j);
  const uint32_t e = (j == 0) ? 0x6400u : (j == 1) ? 0x5C00u : (j == 2) ? 0x5400u : 0x4C00u;
  return (w & mask) | (e | (e << 16));
}

template <int MP>
__global__ void __launch_bounds__(kThreads, 1)
gemv_mma_kernel(const __grid_constant__ CUtensorMap qmap, const __half* __restrict__ dsc,
                __half* __restrict__ Y, const Params p) {
  constexpr int NT = MP / 8;
  constexpr int kTiles = Unit<MP>::kTiles;
  constexpr int kWarpRows = Unit<MP>::kWarpRows;
  constexpr int kRT = Unit<MP>::kRT;
  constexpr int kWBytes = Unit<MP>::kWBytes;
  constexpr int kXBytes = MP * 512;
  constexpr int kCBytes = 64;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int S = p.stages;
  uint8_t* wst = smem;                                   // S x kWBytes
  uint8_t* xst = wst + (size_t)S * kWBytes;              // S x kXBytes
  uint8_t* cst = xst + (size_t)S * kXBytes;              // S x kCBytes
  uint8_t* dst_ = cst + (size_t)S * kCBytes;              // S x kRT fp16 scales
  uint64_t* full = reinterpret_cast<uint64_t*>(dst_ + (size_t)S * kRT * 2);
  uint64_t* empty = full + S;
  volatile int* s_flag = reinterpret_cast<volatile int*>(empty + S);
  volatile int* s_abort = s_flag + 1;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const long long U = p.U, G = p.G;
  const long long u0 = range_start(blockIdx.x, U, G), u1 = range_start(blockIdx.x + 1, U, G);
  const int B = p.B;

  if (threadIdx.x == 0) {
    for (int s = 0; s < S; ++s) {
      ptx::mbar_init(&full[s], 1);
      ptx::mbar_init(&empty[s], kConsumerWarps);
    }
    *s_abort = 0;
    ptx::fence_mbar_init();
  }
  __syncthreads();

  // ---------------------------------------------------------------- copies
  // Lane 0 of warp 0 issues every copy: the first S units up front (weights
  // first: they do not depend on the prep kernel), then one refill per unit,
  // as soon as all eight warps have released the stage it reuses.
  const long long n = u1 - u0;
  const uint32_t tx = kWBytes + kXBytes + MP * 4 + kRT * 2;
  uint64_t pol = 0;
  int pb = 0, prt = 0;          // block / row tile of the next unit to load
  auto issue = [&](int st, int b_, int rt_) {
    ptx::mbar_arrive_expect_tx(&full[st], tx);
    ptx::tma_load_2d(wst + (size_t)st * kWBytes, &qmap, b_ * 64, rt_ * kRT, &full[st], pol);
    if (Unit<MP>::kBoxes == 2)
      ptx::tma_load_2d(wst + (size_t)st * kWBytes + kBoxRows * 64, &qmap, b_ * 64, rt_ * kRT + kBoxRows,
                       &full[st], pol);
    ptx::bulk_load(xst + (size_t)st * kXBytes, p.xil + (size_t)b_ * MP * 32, kXBytes, &full[st]);
    ptx::bulk_load(cst + (size_t)st * kCBytes, p.bias + (size_t)b_ * MP, MP * 4, &full[st]);
    ptx::bulk_load(dst_ + (size_t)st * kRT * 2, p.dT + (size_t)b_ * p.Npad + (size_t)rt_ * kRT, kRT * 2,
                   &full[st]);
  };
  if (warp == 0 && lane == 0) {
    ptx::prefetch_tensormap(&qmap);
    pol = ptx::policy_evict_first();
    const long long pre = n < S ? n : S;
    for (long long i = 0; i < pre; ++i) {
      const long long u = u0 + i;
      ptx::mbar_arrive_expect_tx(&full[i], tx);
      const int bx = (int)(u % B) * 64, ry = (int)(u / B) * kRT;
      ptx::tma_load_2d(wst + i * kWBytes, &qmap, bx, ry, &full[i], pol);
      if (Unit<MP>::kBoxes == 2)
        ptx::tma_load_2d(wst + i * kWBytes + kBoxRows * 64, &qmap, bx, ry + kBoxRows, &full[i], pol);
    }
    ptx::griddep_wait();        // activations, bias and scales come from the prep kernel
    for (long long i = 0; i < pre; ++i) {
      const int b0 = (int)((u0 + i) % B), rt0 = (int)((u0 + i) / B);
      ptx::bulk_load(xst + i * kXBytes, p.xil + (size_t)b0 * MP * 32, kXBytes, &full[i]);
      ptx::bulk_load(cst + i * kCBytes, p.bias + (size_t)b0 * MP, MP * 4, &full[i]);
      ptx::bulk_load(dst_ + i * kRT * 2, p.dT + (size_t)b0 * p.Npad + (size_t)rt0 * kRT, kRT * 2, &full[i]);
    }
    pb = (int)((u0 + pre) % B);
    prt = (int)((u0 + pre) / B);
  }

  // -------------------------------------------------------------- consumers
  const int g = lane >> 2, c = lane & 3;
  const uint32_t wst_u = ptx::smem_u32(wst), xst_u = ptx::smem_u32(xst);
  float acc[kTiles][NT][4];
  uint32_t limit = kWaitLimit;
  int seg_b0 = 0;
  int s = 0;
  uint32_t ph = 0;
  int b = (int)(u0 % B), rt = (int)(u0 / B);
  float dg[kTiles][2];
  for (long long u = u0; u < u1; ++u) {
    if (u == u0 || b == 0) {
      seg_b0 = b;
#pragma unroll
      for (int t = 0; t < kTiles; ++t)
#pragma unroll
        for (int nt = 0; nt < NT; ++nt)
#pragma unroll
          for (int e = 0; e < 4; ++e) acc[t][nt][e] = 0.f;
    }
    if (!ptx::mbar_wait(&full[s], ph, limit)) {
      ptx::record_wait_failure(p.error, 2u);
      limit = 1;
    }
    // B fragments: pairs (x_{16G+j}, x_{16G+j+8}) for the 16-groups G = 4c + q
    uint32_t bf[NT][4][4][2];
    float cb[NT][2];
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
      const int m = g + 8 * nt;
      const uint32_t base = xst_u + (uint32_t)(s * kXBytes + m * 512);
      const int sw = (2 * c + (m & 1)) & 7;
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const int G = 4 * c + q;
        const uint4 v0 = ptx::lds128(base + (uint32_t)(((2 * G) ^ sw) * 16));
        const uint4 v1 = ptx::lds128(base + (uint32_t)(((2 * G + 1) ^ sw) * 16));
        bf[nt][q][0][0] = v0.x; bf[nt][q][1][0] = v0.y; bf[nt][q][2][0] = v0.z; bf[nt][q][3][0] = v0.w;
        bf[nt][q][0][1] = v1.x; bf[nt][q][1][1] = v1.y; bf[nt][q][2][1] = v1.z; bf[nt][q][3][1] = v1.w;
      }
      const float* cs = reinterpret_cast<const float*>(cst + (size_t)s * kCBytes);
      cb[nt][0] = cs[2 * c + 8 * nt];
      cb[nt][1] = cs[2 * c + 1 + 8 * nt];
    }
    // packed words of the warp's rows: rows r and r + 8 of each 16-row tile
    uint32_t wa[kTiles][4], wb[kTiles][4];
    const __half* ds_s = reinterpret_cast<const __half*>(dst_ + (size_t)s * kRT * 2);
#pragma unroll
    for (int t = 0; t < kTiles; ++t) {
      const int r = warp * kWarpRows + t * 16 + g;
      const uint4 va = ptx::lds128(wst_u + (uint32_t)(s * kWBytes + r * 64 + 16 * c));
      const uint4 vb = ptx::lds128(wst_u + (uint32_t)(s * kWBytes + (r + 8) * 64 + 16 * c));
      wa[t][0] = va.x; wa[t][1] = va.y; wa[t][2] = va.z; wa[t][3] = va.w;
      wb[t][0] = vb.x; wb[t][1] = vb.y; wb[t][2] = vb.z; wb[t][3] = vb.w;
      dg[t][0] = __half2float(ds_s[r]);
      dg[t][1] = __half2float(ds_s[r + 8]);
    }
    // everything this warp needs from the stage is in registers: hand it back
    __syncwarp();
    if (lane == 0) ptx::mbar_arrive(&empty[s]);
    if (warp == 0 && lane == 0 && (u - u0) + S < n) {
      // refill this stage with unit u + S once every warp has released it
      if (!ptx::mbar_wait(&empty[s], ph, limit)) {
        ptx::record_wait_failure(p.error, 1u);
        limit = 1;
      }
      issue(s, pb, prt);
      if (++pb == B) { pb = 0; ++prt; }
    }
    __syncwarp();
    // one accumulator chain per (row tile, 16-group q): 4 x kTiles independent
    // chains of depth 4, enough to keep the legacy tensor pipe busy (a single
    // dependent mma.sync chain waits ~140 cycles per step on this part)
    float C[kTiles][4][NT][4];
#pragma unroll
    for (int t = 0; t < kTiles; ++t)
#pragma unroll
      for (int q = 0; q < 4; ++q)
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
          C[t][q][nt][0] = q == 0 ? -cb[nt][0] : 0.f;
          C[t][q][nt][1] = q == 0 ? -cb[nt][1] : 0.f;
          C[t][q][nt][2] = q == 0 ? -cb[nt][0] : 0.f;
          C[t][q][nt][3] = q == 0 ? -cb[nt][1] : 0.f;
        }
#pragma unroll
    for (int jj = 0; jj < 4; ++jj) {
#pragma unroll
      for (int q = 0; q < 4; ++q) {
#pragma unroll
        for (int t = 0; t < kTiles; ++t) {
          const uint32_t A[4] = {decode_pair(wa[t][q], jj), decode_pair(wb[t][q], jj),
                                 decode_pair(wa[t][q] >> 8, jj), decode_pair(wb[t][q] >> 8, jj)};
#pragma unroll
          for (int nt = 0; nt < NT; ++nt)
            ptx::mma_16816(C[t][q][nt], A, bf[nt][q][jj][0], bf[nt][q][jj][1]);
        }
      }
    }
#pragma unroll
    for (int t = 0; t < kTiles; ++t)
#pragma unroll
      for (int nt = 0; nt < NT; ++nt) {
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const float sum = (C[t][0][nt][e] + C[t][1][nt][e]) + (C[t][2][nt][e] + C[t][3][nt][e]);
          acc[t][nt][e] = fmaf(dg[t][e >> 1], sum, acc[t][nt][e]);
        }
      }
    if (++s == S) { s = 0; ph ^= 1u; }
    const int cur_b = b, cur_rt = rt;
    if (++b == B) { b = 0; ++rt; }

    if (cur_b != B - 1 && u != u1 - 1) continue;
    // ------------------------------------------------------------ epilogue
    const bool whole = (seg_b0 == 0 && cur_b == B - 1);
    const int row0e = cur_rt * kRT + warp * kWarpRows;
    if (whole) {
#pragma unroll
      for (int t = 0; t < kTiles; ++t)
#pragma unroll
        for (int nt = 0; nt < NT; ++nt)
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const int n = row0e + t * 16 + g + 8 * (e >> 1);
            const int m = 2 * c + (e & 1) + 8 * nt;
            if (n < p.N && m < p.M) Y[(size_t)m * p.N + n] = __float2half_rn(acc[t][nt][e]);
          }
      continue;
    }
    const int slot = (cur_rt == (int)(u0 / B)) ? 0 : 1;
    float* mine = p.partials + ((size_t)blockIdx.x * 2 + slot) * kRT * MP;
#pragma unroll
    for (int t = 0; t < kTiles; ++t)
#pragma unroll
      for (int nt = 0; nt < NT; ++nt)
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          const int r = warp * kWarpRows + t * 16 + g + 8 * h;
          *reinterpret_cast<float2*>(mine + r * MP + 2 * c + 8 * nt) =
              make_float2(acc[t][nt][2 * h], acc[t][nt][2 * h + 1]);
        }
    __threadfence();
    ptx::named_bar_sync(1, kConsumerWarps * 32);
    const long long cfirst = cta_of_unit((long long)cur_rt * B, U, G);
    const long long clast = cta_of_unit((long long)cur_rt * B + B - 1, U, G);
    if (threadIdx.x == 0) {
      const unsigned old = atomicAdd(&p.counters[cur_rt], 1u);
      *s_flag = (old == (unsigned)(clast - cfirst)) ? 1 : 0;
    }
    ptx::named_bar_sync(1, kConsumerWarps * 32);
    if (*s_flag) {
      __threadfence();
      float sum[kTiles][NT][4];
#pragma unroll
      for (int t = 0; t < kTiles; ++t)
#pragma unroll
        for (int nt = 0; nt < NT; ++nt)
#pragma unroll
          for (int e = 0; e < 4; ++e) sum[t][nt][e] = 0.f;
      for (long long cc = cfirst; cc <= clast; ++cc) {
        const int sl = (cur_rt == (int)(range_start(cc, U, G) / B)) ? 0 : 1;
        const float* src = p.partials + ((size_t)cc * 2 + sl) * kRT * MP;
#pragma unroll
        for (int t = 0; t < kTiles; ++t)
#pragma unroll
          for (int nt = 0; nt < NT; ++nt)
#pragma unroll
            for (int h = 0; h < 2; ++h) {
              const int r = warp * kWarpRows + t * 16 + g + 8 * h;
              const float2 v = __ldcg(reinterpret_cast<const float2*>(src + r * MP + 2 * c + 8 * nt));
              sum[t][nt][2 * h] += v.x;
              sum[t][nt][2 * h + 1] += v.y;
            }
      }
#pragma unroll
      for (int t = 0; t < kTiles; ++t)
#pragma unroll
        for (int nt = 0; nt < NT; ++nt)
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const int n = row0e + t * 16 + g + 8 * (e >> 1);
            const int m = 2 * c + (e & 1) + 8 * nt;
            if (n < p.N && m < p.M) Y[(size_t)m * p.N + n] = __float2half_rn(sum[t][nt][e]);
          }
      if (threadIdx.x == 0) p.counters[cur_rt] = 0u;
    }
  }
}

// ---------------------------------------------------------------- host side
struct Layout {
  size_t off_cnt, off_xil, off_bias, off_dt, off_part, total;
  int64_t Npad;
};

size_t up256(size_t x) { return (x + 255) & ~size_t(255); }

Layout layout_for(int64_t M, int64_t N, int64_t K, int num_sms) {
  const int MP = M <= 8 ? 8 : 16;
  const int kRT = MP == 8 ? Unit<8>::kRT : Unit<16>::kRT;
  const int64_t B = K / kBlock, T = ceil_div(N, kRT);
  const int64_t U = T * B;
  const int64_t G = U < num_sms ? U : num_sms;
  Layout L;
  L.off_cnt = 0;
  L.off_xil = L.off_cnt + up256((size_t)T * 4);
  L.off_bias = L.off_xil + up256((size_t)B * MP * 512);
  L.Npad = T * kRT;
  L.off_dt = L.off_bias + up256((size_t)B * MP * 4);
  L.off_part = L.off_dt + up256((size_t)B * L.Npad * 2);
  L.total = L.off_part + up256((size_t)G * 2 * kRT * MP * 4);
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

int stages_for(int MP) {
  const int rt = MP == 8 ? Unit<8>::kRT : Unit<16>::kRT;
  const int per = (MP == 8 ? Unit<8>::kWBytes : Unit<16>::kWBytes) + MP * 512 + 64 + rt * 2;
  int s = (kSmemBudget - 2048) / per;
  return s > 12 ? 12 : s;
}

template <int MP>
cudaError_t launch_mp(const __half* X, const uint8_t* qs, const __half* d, __half* Y, int M, int N,
                      int K, void* ws, int num_sms, cudaStream_t s) {
  const Layout L = layout_for(M, N, K, num_sms);
  uint8_t* w = static_cast<uint8_t*>(ws);
  Params p;
  constexpr int kRT = Unit<MP>::kRT;
  constexpr int kWBytes = Unit<MP>::kWBytes;
  p.B = K / kBlock;
  p.T = (int)ceil_div(N, kRT);
  p.U = (long long)p.T * p.B;
  p.G = (int)(p.U < num_sms ? p.U : num_sms);
  p.M = M; p.N = N; p.K = K;
  p.stages = stages_for(MP);
  p.xil = reinterpret_cast<const uint4*>(w + L.off_xil);
  p.bias = reinterpret_cast<const float*>(w + L.off_bias);
  p.dT = reinterpret_cast<const __half*>(w + L.off_dt);
  p.Npad = (int)L.Npad;
  p.partials = reinterpret_cast<float*>(w + L.off_part);
  p.counters = reinterpret_cast<unsigned*>(w + L.off_cnt);
  const cudaError_t ew = wait_status_word(&p.error);
  if (ew != cudaSuccess) return ew;

  auto enc = encode_fn();
  if (!enc) return cudaErrorNotSupported;
  CUtensorMap map;
  const cuuint64_t gdim[2] = {(cuuint64_t)(K / 4), (cuuint64_t)N};
  const cuuint64_t gstride[1] = {(cuuint64_t)(K / 4)};
  const cuuint32_t box[2] = {64, (cuuint32_t)kBoxRows};
  const cuuint32_t estr[2] = {1, 1};
  CUresult r = enc(&map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<uint8_t*>(qs), gdim, gstride,
                   box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return cudaErrorInvalidValue;

  xprep_kernel<MP><<<p.B + p.Npad / 64, MP * 16, 0, s>>>(
      X, d, M, N, K, p.B, p.Npad, reinterpret_cast<uint4*>(w + L.off_xil),
      reinterpret_cast<float*>(w + L.off_bias), reinterpret_cast<__half*>(w + L.off_dt), p.counters, p.T);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;

  const size_t smem = (size_t)p.stages * (kWBytes + MP * 512 + 64 + kRT * 2) + 2 * p.stages * 8 + 16 + 1024;
  e = cudaFuncSetAttribute(gemv_mma_kernel<MP>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
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
  return cudaLaunchKernelEx(&cfg, gemv_mma_kernel<MP>, map, d, Y, p);
}

}  // namespace

bool gemv_mma_supported(int fmt, int64_t M, int64_t N, int64_t K) {
  return fmt == TRI_TQ2 && M >= 1 && M <= 16 && N >= 1 && K >= kBlock && K % kBlock == 0;
}

size_t gemv_mma_ws_bytes(int, int64_t M, int64_t N, int64_t K, int num_sms) {
  return layout_for(M, N, K, num_sms).total;
}

cudaError_t launch_gemv_mma(int fmt, const __half* X, const uint8_t* qs, const __half* d, __half* Y,
                            int M, int N, int K, void* ws, int num_sms, cudaStream_t s) {
  if (!gemv_mma_supported(fmt, M, N, K)) return cudaErrorNotSupported;
  if (M <= 8) return launch_mp<8>(X, qs, d, Y, M, N, K, ws, num_sms, s);
  return launch_mp<16>(X, qs, d, Y, M, N, K, ws, num_sms, s);
}

// ---------------------------------------------------------------------------
// Static-scratch variant for callers that cannot allocate device memory.
//
// Some hosts of this library may not call cudaMalloc at all: a plugin inside
// a framework that owns every device allocation and hands out only the
// tensors of the call, or a real-time or embedded loop that has to keep a
// fixed, preallocated memory footprint.  They still pass X, the packed
// weights and Y, but the scratch this kernel needs (prepared activations,
// split-K partials, tickets) lives in the file-scope array below instead of
// a caller-provided workspace.
//
// The array is a module global: every device that loads the library keeps
// kNoAllocScratchBytes reserved until the process exits, and every call on a
// device uses the same bytes, so calls that can overlap on that device (two
// streams, or two host threads) race and must be ordered by the caller.
// Host code only ever sees a host-side stand-in for the symbol; the device
// address is looked up with cudaGetSymbolAddress on the first call on each
// device, with that device current (which may also load the module, so make
// that first call before any stream capture).  A failed lookup is not
// cached: the next call tries again.  What must start at zero (the per-tile
// tickets) is cleared by the prep kernel of every call, inside the launch
// sequence, so bytes left in the array by an earlier call never matter.
constexpr size_t kNoAllocScratchBytes = size_t(8) << 20;   // 8 MiB
static __device__ __align__(256) uint8_t g_noalloc_scratch[kNoAllocScratchBytes];

namespace {
constexpr int kMaxDev = 64;
void* g_scratch_addr[kMaxDev];
std::mutex g_scratch_mu[kMaxDev];

// device address of the static array on the current device (looked up once
// per device; only a successful lookup is kept)
cudaError_t scratch_address(int dev, uint8_t** out) {
  std::lock_guard<std::mutex> lock(g_scratch_mu[dev]);
  if (!g_scratch_addr[dev]) {
    void* ptr = nullptr;
    const cudaError_t e = cudaGetSymbolAddress(&ptr, g_noalloc_scratch);
    if (e != cudaSuccess) return e;
    g_scratch_addr[dev] = ptr;
  }
  *out = static_cast<uint8_t*>(g_scratch_addr[dev]);
  return cudaSuccess;
}
}  // namespace

size_t gemv_noalloc_scratch_limit() { return kNoAllocScratchBytes; }

size_t gemv_noalloc_scratch_need(int64_t M, int64_t N, int64_t K, int num_sms) {
  return gemv_mma_ws_bytes(TRI_TQ2, M, N, K, num_sms);
}

cudaError_t launch_gemv_mma_noalloc(const __half* X, const uint8_t* qs, const __half* d, __half* Y,
                                    int M, int N, int K, int num_sms, cudaStream_t s) {
  int dev = -1;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDev) return cudaErrorInvalidDevice;
  if (gemv_noalloc_scratch_need(M, N, K, num_sms) > kNoAllocScratchBytes) return cudaErrorInvalidValue;
  uint8_t* ws = nullptr;
  e = scratch_address(dev, &ws);
  if (e != cudaSuccess) return e;
  return launch_gemv_mma(TRI_TQ2, X, qs, d, Y, M, N, K, ws, num_sms, s);
}

}  // namespace tri
