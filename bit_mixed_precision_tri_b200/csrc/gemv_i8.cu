// Decode-regime ternary GEMV for one or two activation rows (TQ2) on the
// integer tensor-core path: exact int8 products of the 2-bit weight fields
// with fixed-point activation digits.
//
// Y = X (d * W_hat)^T ("Scaling Laws and Efficient Inference for Ternary
// Language Models", section "The model", step 3).  At M <= 2 the layer is
// bound by streaming the packed weights ("TriRun: ternary inference on
// GPUs": 2-bit weights move 8x fewer bytes than fp16), so the kernel is built
// to spend as few instructions per weight byte as possible:
//
//  * Weights.  A TQ2 byte holds four fields d' = t + 1; in a 32-bit word of
//    sixteen fields, w & (0x03030303 << 2g) keeps field g of each byte, i.e.
//    four weights 4^g * d' as unsigned bytes, one LOP3 for four weights and
//    no shift.  Four such registers (rows r and r+8, two words each) are the
//    A operand of one mma.sync m16n8k32 u8 x s8 -> s32: 512 weights per
//    instruction.  The field g is kept in a chain of its own (accumulator set
//    g), and the chains are combined exactly once per block as
//    64 c0 + 16 c1 + 4 c2 + c3 = 64 * sum_k d'_k x^_k.
//  * Activations.  Each 256-element block of X is written as 24-bit fixed
//    point x = s_b x^ (|x^| <= 8e6) split into three balanced base-256
//    digits (levels); level l of batch row m is column 3m + l of the n8 B
//    operand, so M <= 2 fits one instruction.  Every CTA quantises the blocks
//    its range touches itself, straight into shared memory in the exact
//    per-thread fragment order (with the k permutation that the weight-side
//    masks imply): no separate prep kernel, whose launch would serialise
//    with this one.  The only rounding of the method's arithmetic is this
//    quantisation: at most half a step (2^-24 of the block's largest |x|)
//    per element.
//  * Per block and row:  sum_k t_k x_k ~= s_b (sum_k d'_k x^_k - sum_k x^_k),
//    times the block scale d[n][b], accumulated in fp32.
//  * Streaming.  Work = (128-row tile) x (pair of blocks) units split over a
//    persistent grid as contiguous ranges (stream-K): every CTA streams the
//    same number of weight bytes.  Each warp owns 16 rows of the tile and
//    keeps four units of 16-byte cp.async copies in flight, the first four
//    copied before the wait for the preceding grid.  A row tile split
//    between CTAs is finished by whichever CTA completes its share last:
//    every contributing warp stores its rows' partial sums, stamped with the
//    call (one 64-bit store each: no fence), and takes the warp's ticket of
//    the tile (one atomic add); the warp that draws the last ticket adds the
//    partials in CTA order (deterministic, whoever is last) and writes Y.  A
//    value whose stamp is not yet this call's is one whose store was already
//    issued (its warp took a ticket after it) and is read again until it
//    lands: no CTA ever waits for work another CTA still has to do, so the
//    result does not depend on which CTAs are resident together.  The stamp
//    is a per-workspace call counter on the device (a small library-owned
//    pool), advanced by the last CTA of each call, so bytes left in the
//    workspace by earlier calls never pass for this call's sums; tickets live
//    in the same pool, start at zero and are returned to zero by the warp
//    that draws the last one.
#include <mutex>

#include "sm100_ptx.cuh"
#include "tri_internal.cuh"

namespace tri {

constexpr int kEpochSlots = 32;        // workspaces with an epoch slot per device
constexpr int kMaxG = 512;             // grid size limit
// [slot][0]: epoch of the next call, [slot][1]: CTAs of the current call done,
// [slot][2 + 8 c + w]: ticket of warp w for the row tile whose first CTA is c
constexpr int kSlotWords = 2 + kMaxG * 8;
static __device__ unsigned g_i8_epochs[kEpochSlots][kSlotWords];

namespace {

constexpr int kWarps = 8;
constexpr int kThreads = kWarps * 32;
constexpr int kRT = kWarps * 16;       // rows per unit (row tile)
constexpr float kQMax = 8.0e6f;        // |x^| bound: three balanced base-256 digits

struct Params {
  const __half* X;       // [M][K]
  unsigned long long* partials;  // [G][2][kRT][M]: stamp << 32 | fp32 bits; [c][0]: the CTA's last
                                 // segment (a tile's start), [c][1]: its first (a tile continued)
  unsigned* epoch;       // this workspace's [epoch, done, tickets...] words in the pool
  unsigned slot;         // its index (part of every stamp)
  unsigned* error;       // set when a wait for a partial sum gives up (never expected)
  int N, K, B, P, T, G;
  long long U;
  int k4, k16, k64;      // 4, 16, 64 (runtime values: the combine runs as IMAD, off the ALU pipe)
};

__host__ __device__ inline long long range_start(long long c, long long U, long long G) {
  return c * U / G;
}
__host__ __device__ inline long long cta_of_unit(long long u, long long U, long long G) {
  return ((u + 1) * G + U - 1) / U - 1;
}

// ---------------------------------------------------------------- main kernel
// A unit is (128-row tile, pair of blocks): every warp handles 16 rows x 512
// weights per step, 16 MMAs in eight independent chains.
//
// Shared memory per CTA:
//  * a ring of kStages weight stages per warp, filled with cp.async (16 bytes
//    per copy); every lane reads back exactly the bytes it copied, so a stage
//    needs no synchronisation beyond the lane's own cp.async.wait_group;
//  * the activation fragments and block scalars of every block pair that the
//    CTA's range touches (at most kMaxPairs), computed once at the start.
//    Lanes without a B column read a zero slot.
template <int M> struct Cfg {
  static constexpr int kStages = 4;                       // pairs of weights in flight per warp
  static constexpr int kWStage = 2048;                    // [block h][row half][32 lanes][16 B]
  static constexpr int kRing = kWarps * kStages * kWStage;
  static constexpr int kBL = 12 * M;                      // lanes with a B column (gid < 3M)
  static constexpr int kBSlots = kBL + 1;                 // + a zero slot
  static constexpr int kBlkBytes = 4 * kBSlots * 16;      // [i][slot][16 B]
  static constexpr int kPairBytes = 2 * kBlkBytes + 2 * 2 * M * 4;   // + [h][step M, bias M]
  static constexpr int kMaxPairs = M == 1 ? 27 : 14;      // keeps two CTAs per SM
};

__device__ __forceinline__ void cp_async_cg16(uint32_t dst, const void* src, uint32_t src_bytes) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src), "r"(src_bytes)
               : "memory");
}
constexpr int kSpinLimit = 1 << 22;   // stamp polls: a 64 ns sleep + an L2 read, ~256 ns each, ~1 s in all

__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

__device__ __forceinline__ void mma_u8s8(int (&c)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                         uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k32.row.col.s32.u8.s8.s32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+r"(c[0]), "+r"(c[1]), "+r"(c[2]), "+r"(c[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// first MMA of a chain: C = 0
__device__ __forceinline__ void mma_u8s8_z(int (&c)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                           uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k32.row.col.s32.u8.s8.s32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%10,%10,%10,%10};"
      : "=r"(c[0]), "=r"(c[1]), "=r"(c[2]), "=r"(c[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1), "r"(0));
}

template <int M>
__global__ void __launch_bounds__(kThreads, 2)
gemv_i8_kernel(const uint8_t* __restrict__ qs, const __half* __restrict__ d, __half* __restrict__ Y,
               const Params p) {
  using C = Cfg<M>;
  constexpr int S = C::kStages;
  extern __shared__ __align__(16) uint8_t smem[];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int gid = lane >> 2, tig = lane & 3;
  const long long U = p.U, G = p.G;
  const long long u0 = range_start(blockIdx.x, U, G), u1 = range_start(blockIdx.x + 1, U, G);
  const int n_units = (int)(u1 - u0);
  const int B = p.B, P = p.P;                          // blocks and block pairs per row
  const size_t rs = (size_t)p.K / 4;                  // packed bytes per row
  const uint32_t ring = ptx::smem_u32(smem) + warp * (S * C::kWStage);
  const uint32_t pairs = ptx::smem_u32(smem) + C::kRing;
  const int q0 = (int)(u0 % P);

  // ---- producer state: next unit to copy
  int il = 0;                                          // units issued
  int rt_l = (int)(u0 / P), q_l = q0;
  // rows outside the matrix copy 0 bytes (zero fill) from a valid address
  const uint8_t* pa = qs;                             // row gid, block 2 q_l
  const uint8_t* pb = qs;                             // row gid + 8
  const unsigned short* da_p = nullptr;
  const unsigned short* db_p = nullptr;
  uint32_t szA = 0, szB = 0;
  const bool odd_b = (B & 1) != 0;
  auto set_rows = [&]() {
    const int rowA = rt_l * kRT + warp * 16 + gid;
    szA = rowA < p.N ? 16u : 0u;
    szB = rowA + 8 < p.N ? 16u : 0u;
    const int ra = szA ? rowA : 0, rb = szB ? rowA + 8 : 0;
    pa = qs + (size_t)ra * rs + (size_t)q_l * 128 + tig * 16;
    pb = qs + (size_t)rb * rs + (size_t)q_l * 128 + tig * 16;
    da_p = reinterpret_cast<const unsigned short*>(d) + (size_t)ra * B + 2 * q_l;
    db_p = reinterpret_cast<const unsigned short*>(d) + (size_t)rb * B + 2 * q_l;
  };
  set_rows();
  // block scales as raw fp16 bits, converted when the stage is consumed (the
  // loads then have the whole ring depth to land)
  unsigned short dv[S][2][2];                          // [stage][block h][row half]
  auto issue = [&](int s, bool commit) {
    if (il < n_units) {
      const uint32_t st = ring + s * C::kWStage + lane * 16;
      const bool h1 = !(odd_b && q_l == P - 1);       // odd B: the last pair has one block
      const uint32_t s1a = h1 ? szA : 0u, s1b = h1 ? szB : 0u;
      const int o1 = h1 ? 64 : 0;
      cp_async_cg16(st, pa, szA);
      cp_async_cg16(st + 512, pb, szB);
      cp_async_cg16(st + 1024, pa + o1, s1a);
      cp_async_cg16(st + 1536, pb + o1, s1b);
      // unconditional loads from clamped addresses (a select on the loaded
      // value would wait for it); rows outside the matrix are never stored
      // and a missing block has zero weights and zero activation scalars
      dv[s][0][0] = __ldg(da_p);
      dv[s][0][1] = __ldg(db_p);
      dv[s][1][0] = __ldg(da_p + (h1 ? 1 : 0));
      dv[s][1][1] = __ldg(db_p + (h1 ? 1 : 0));
      ++il;
      if (++q_l == P) {
        q_l = 0;
        ++rt_l;
        set_rows();
      } else {
        pa += 128;
        pb += 128;
        da_p += 2;
        db_p += 2;
      }
    }
    if (commit) cp_async_commit();                    // one group per stage (empty at the end)
  };
  // The weights do not depend on X: the whole ring is copied before waiting
  // for the grid that produced X (programmatic dependent launch), so a CTA
  // that launched early has its first weights in place when the wait ends.
  // (Kernels that write qs or d must therefore not let this one launch early;
  // none of this library's do.)  Every CTA lets the next grid launch as soon
  // as it runs: that grid can only start once all CTAs of this one have done
  // so, i.e. are resident, so its CTAs never take a slot that a CTA of this
  // grid (which a reducer may wait for) still needs.
  ptx::griddep_launch_dependents();
#pragma unroll
  for (int st = 0; st < S; ++st) issue(st, true);     // group s: weight stage s
  ptx::griddep_wait();
  // this call's stamp: epoch and slot (the previous grid's epoch update is visible now)
  const unsigned long long stamp =
      (unsigned long long)((*reinterpret_cast<volatile unsigned*>(p.epoch) + 1u) * (unsigned)kEpochSlots + p.slot);
  const int n_pairs = n_units < P ? n_units : P;
  {
    // zero slots, read by the lanes without a B column
    for (int it = threadIdx.x; it < n_pairs * 2 * 4; it += kThreads) {
      const int i = it & 3, hb = it >> 2;
      *reinterpret_cast<uint4*>(smem + C::kRing + (hb >> 1) * C::kPairBytes + (hb & 1) * C::kBlkBytes +
                                (i * C::kBSlots + C::kBL) * 16) = make_uint4(0, 0, 0, 0);
    }
    // Quantise one block per warp at a time; lane L holds elements 8L .. 8L+7,
    // i.e. word L/2 of the block, bytes 2(L&1) and 2(L&1)+1, fields 0..3: the
    // two bytes of field g land in one 16-bit half of fragment register
    // (p, g, r) of the thread with threadID_in_group = tig.  The X loads of up
    // to four blocks per warp are in flight together.
    const int f_word = lane >> 1, half = lane & 1;
    const int f_tig = f_word >> 2, f_p = (f_word >> 1) & 1, f_r = f_word & 1;
    constexpr int kXB = 4;
    const int n_blk = n_pairs * 2;
    for (int hb0 = warp; hb0 < n_blk; hb0 += kXB * kWarps) {
      uint4 raw[kXB][M];
#pragma unroll
      for (int x = 0; x < kXB; ++x) {
        const int hb = hb0 + x * kWarps;
        int qq = q0 + (hb >> 1);
        if (qq >= P) qq -= P;
        const int blk = 2 * qq + (hb & 1);
#pragma unroll
        for (int m = 0; m < M; ++m)
          raw[x][m] = (hb < n_blk && blk < B)
                          ? __ldg(reinterpret_cast<const uint4*>(p.X + (size_t)m * p.K + (size_t)blk * kBlock) + lane)
                          : make_uint4(0, 0, 0, 0);
      }

#pragma unroll
      for (int x = 0; x < kXB; ++x) {
        const int hb = hb0 + x * kWarps;
        if (hb >= n_blk) break;
        const int jj = hb >> 1, h = hb & 1;
        int qq = q0 + jj;
        if (qq >= P) qq -= P;
        const int blk = 2 * qq + h;
        uint8_t* rec = smem + C::kRing + jj * C::kPairBytes + h * C::kBlkBytes;
        float* sc = reinterpret_cast<float*>(smem + C::kRing + jj * C::kPairBytes + 2 * C::kBlkBytes) + h * 2 * M;
        if (blk >= B) {                               // the missing half of an odd last pair
          for (int it = lane; it < 4 * C::kBL; it += 32)
            *reinterpret_cast<uint4*>(rec + ((it / C::kBL) * C::kBSlots + it % C::kBL) * 16) = make_uint4(0, 0, 0, 0);
          if (lane < 2 * M) sc[lane] = 0.f;
          continue;
        }
#pragma unroll
        for (int m = 0; m < M; ++m) {
          const uint32_t hw[4] = {raw[x][m].x, raw[x][m].y, raw[x][m].z, raw[x][m].w};
          float xv[8];
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            const float2 f = __half22float2(*reinterpret_cast<const __half2*>(&hw[i]));
            xv[2 * i] = f.x;
            xv[2 * i + 1] = f.y;
          }
          float amax = 0.f;
#pragma unroll
          for (int e = 0; e < 8; ++e) amax = fmaxf(amax, fabsf(xv[e]));
          // |x| >= 0: the bit patterns order like the values, so one integer
          // warp reduction gives the block maximum
          amax = __uint_as_float(__reduce_max_sync(0xFFFFFFFFu, __float_as_uint(amax)));
          const float inv = amax > 0.f ? kQMax / amax : 0.f;
          // Balanced base-256 digits of q, as bytes: with u = q + 0x808080
          // (in [0, 2^24) for |q| <= 8e6), byte i of u is digit i + 128, so
          // byte i of u ^ 0x808080 is digit i as a signed byte (byte 0 the
          // lowest digit, byte 2 the highest).
          uint32_t dg[8];
          int sum = 0;
#pragma unroll
          for (int e = 0; e < 8; ++e) {
            const int q = __float2int_rn(xv[e] * inv);   // |q| <= 8e6 < 2^23
            sum += q;
            dg[e] = ((uint32_t)q + 0x808080u) ^ 0x808080u;
          }
          // level lv = column 3m + lv holds digit 2 - lv (the highest first);
          // the two bytes of field g are elements g and g + 4
#pragma unroll
          for (int lv = 0; lv < 3; ++lv)
#pragma unroll
            for (int g = 0; g < 4; ++g) {
              const int off = ((f_p * 2 + (g >> 1)) * C::kBSlots + (3 * m + lv) * 4 + f_tig) * 16 +
                              ((g & 1) * 2 + f_r) * 4 + 2 * half;
              const uint32_t sel = (uint32_t)(2 - lv) | ((uint32_t)(6 - lv) << 4);
              *reinterpret_cast<uint16_t*>(rec + off) = (uint16_t)__byte_perm(dg[g], dg[g + 4], sel);
            }
          sum = __reduce_add_sync(0xFFFFFFFFu, sum);
          if (lane == 0) {
            sc[m] = amax > 0.f ? (amax / kQMax) * (1.f / 64.f) : 0.f;   // s_b / 64
            sc[M + m] = 64.f * (float)sum;                              // 64 sum_k x^_k
          }
        }
      }
    }

  }
  __syncthreads();                                    // fragments visible to every warp

  // the columns this thread holds in C (2tig, 2tig+1): batch row and level weight
  float wA[M], wB[M];
#pragma unroll
  for (int m = 0; m < M; ++m) {
    const int la = 2 * tig - 3 * m, lb = 2 * tig + 1 - 3 * m;   // level within batch row m
    wA[m] = la == 0 ? 65536.f : la == 1 ? 256.f : la == 2 ? 1.f : 0.f;
    wB[m] = lb == 0 ? 65536.f : lb == 1 ? 256.f : lb == 2 ? 1.f : 0.f;
  }
  const float wBias = tig == 0 ? -1.f : 0.f;          // bias subtracted once per row
  const int k4 = p.k4, k16 = p.k16, k64 = p.k64;
  const uint32_t bfrag = pairs + (lane < C::kBL ? lane : C::kBL) * 16;

  float acc[2][M];
#pragma unroll
  for (int h = 0; h < 2; ++h)
#pragma unroll
    for (int m = 0; m < M; ++m) acc[h][m] = 0.f;
  int rt = (int)(u0 / P), q = q0;
  int seg_q0 = q, j = 0;
  const int r_local = warp * 16 + gid;
  // End of a segment of row tile `tile` that does not cover the whole tile
  // (side 0: it holds the tile's start, i.e. it is this CTA's last segment;
  // side 1: it continues the tile, i.e. it is this CTA's first): store the
  // warp's stamped partial sums, take the warp's ticket; the last arrival
  // adds the partials of CTAs cfirst .. clast in order and writes Y.
  auto finish_split = [&](int tile, int side) {
    const long long cfirst = cta_of_unit((long long)tile * P, U, G);
    const long long clast = cta_of_unit((long long)tile * P + P - 1, U, G);
    if (tig == 0) {
      unsigned long long* mine = p.partials + ((size_t)blockIdx.x * 2 + side) * kRT * M;
#pragma unroll
      for (int h = 0; h < 2; ++h)
#pragma unroll
        for (int m = 0; m < M; ++m)
          __stcg(mine + (r_local + 8 * h) * M + m, (stamp << 32) | __float_as_uint(acc[h][m]));
    }
    __syncwarp();
    unsigned old = 0;
    unsigned* ticket = p.epoch + 2 + cfirst * kWarps + warp;
    if (lane == 0) {
      old = atomicAdd(ticket, 1u);
      if (old == (unsigned)(clast - cfirst)) *ticket = 0u;   // nobody else touches it in this call
    }
    old = __shfl_sync(0xFFFFFFFFu, old, 0);
    if (old != (unsigned)(clast - cfirst) || tig != 0) return;
    float sum[2][M];
#pragma unroll
    for (int h = 0; h < 2; ++h)
#pragma unroll
      for (int m = 0; m < M; ++m) sum[h][m] = 0.f;
    // The partial sums of up to kBatch contributors are loaded together (one
    // round trip), then checked and added in CTA order; only a value whose
    // stamp is not yet this call's (a store still on its way) is read again.
    constexpr int kBatch = 8 / M;
    for (long long c0 = cfirst; c0 <= clast; c0 += kBatch) {
      const int nb = (int)(clast - c0 + 1 < kBatch ? clast - c0 + 1 : kBatch);
      unsigned long long v[kBatch][2][M];
#pragma unroll
      for (int k = 0; k < kBatch; ++k)
#pragma unroll
        for (int h = 0; h < 2; ++h)
#pragma unroll
          for (int m = 0; m < M; ++m)
            v[k][h][m] = (k < nb && c0 + k != (long long)blockIdx.x)
                             ? ptx::ld_relaxed_u64(p.partials + ((size_t)(c0 + k) * 2 + (c0 + k == cfirst ? 0 : 1)) * kRT * M +
                                                   (r_local + 8 * h) * M + m)
                             : 0ull;
#pragma unroll
      for (int k = 0; k < kBatch; ++k) {
        if (k >= nb) break;
        const long long c = c0 + k;
#pragma unroll
        for (int h = 0; h < 2; ++h)
#pragma unroll
          for (int m = 0; m < M; ++m) {
            if (c == (long long)blockIdx.x) {
              sum[h][m] += acc[h][m];
              continue;
            }
            unsigned long long x = v[k][h][m];
            const unsigned long long* a =
                p.partials + ((size_t)c * 2 + (c == cfirst ? 0 : 1)) * kRT * M + (r_local + 8 * h) * M + m;
            x = ptx::wait_stamp(a, x, stamp, kSpinLimit);     // an issued store, bounded
            if ((x >> 32) != stamp) ptx::record_wait_failure(p.error, 11u);
            sum[h][m] += __uint_as_float((unsigned)x);
          }
      }
    }
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const int n = tile * kRT + r_local + 8 * h;
      if (n < p.N)
#pragma unroll
        for (int m = 0; m < M; ++m) Y[(size_t)m * p.N + n] = __float2half_rn(sum[h][m]);
    }
  };

  for (int base = 0; base < n_units; base += S) {
#pragma unroll
    for (int s = 0; s < S; ++s) {
      if (base + s >= n_units) break;
      cp_async_wait<S - 1>();
      const uint32_t stg = ring + s * C::kWStage + lane * 16;
      const uint32_t pj = bfrag + j * C::kPairBytes;
      const float* sc = reinterpret_cast<const float*>(smem + C::kRing + j * C::kPairBytes + 2 * C::kBlkBytes);
      int c[2][4][4];
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const uint4 va = ptx::lds128(stg + h * 1024), vb = ptx::lds128(stg + h * 1024 + 512);
        uint4 bf[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) bf[i] = ptx::lds128(pj + h * C::kBlkBytes + i * C::kBSlots * 16);
        const uint32_t wa[4] = {va.x, va.y, va.z, va.w};
        const uint32_t wb[4] = {vb.x, vb.y, vb.z, vb.w};
        const uint32_t bw[16] = {bf[0].x, bf[0].y, bf[0].z, bf[0].w, bf[1].x, bf[1].y, bf[1].z, bf[1].w,
                                 bf[2].x, bf[2].y, bf[2].z, bf[2].w, bf[3].x, bf[3].y, bf[3].z, bf[3].w};
#pragma unroll
        for (int g = 0; g < 4; ++g) {
          const uint32_t mask = 0x03030303u << (2 * g);
          mma_u8s8_z(c[h][g], wa[0] & mask, wb[0] & mask, wa[1] & mask, wb[1] & mask, bw[g * 2],
                     bw[g * 2 + 1]);
        }
#pragma unroll
        for (int g = 0; g < 4; ++g) {
          const uint32_t mask = 0x03030303u << (2 * g);
          mma_u8s8(c[h][g], wa[2] & mask, wb[2] & mask, wa[3] & mask, wb[3] & mask, bw[(4 + g) * 2],
                   bw[(4 + g) * 2 + 1]);
        }
      }
      float da[2][2];
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        da[h][0] = __half2float(__ushort_as_half(dv[s][h][0]));
        da[h][1] = __half2float(__ushort_as_half(dv[s][h][1]));
      }
      // the stage's bytes are in registers (the MMAs consumed them): refill it
      issue(s, true);
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        float fv[4];
#pragma unroll
        for (int e = 0; e < 4; ++e)
          fv[e] = (float)(c[h][3][e] + c[h][2][e] * k4 + c[h][1][e] * k16 + c[h][0][e] * k64);
#pragma unroll
        for (int m = 0; m < M; ++m) {
          const float st = sc[h * 2 * M + m], nb = wBias * sc[h * 2 * M + M + m];
          const float f0 = fmaf(wA[m], fv[0], fmaf(wB[m], fv[1], nb));
          const float f1 = fmaf(wA[m], fv[2], fmaf(wB[m], fv[3], nb));
          acc[0][m] = fmaf(f0, st * da[h][0], acc[0][m]);
          acc[1][m] = fmaf(f1, st * da[h][1], acc[1][m]);
        }
      }

      const int u = base + s;
      const int cur_rt = rt, cur_q = q;
      if (++j == P) j = 0;                            // slot of pair q: (q - q0) mod P
      if (++q == P) { q = 0; ++rt; }
      if (cur_q != P - 1 && u != n_units - 1) continue;

      // ------------------------------------------------ end of a row-tile segment
#pragma unroll
      for (int h = 0; h < 2; ++h)
#pragma unroll
        for (int m = 0; m < M; ++m) {
          acc[h][m] += __shfl_xor_sync(0xFFFFFFFFu, acc[h][m], 1);
          acc[h][m] += __shfl_xor_sync(0xFFFFFFFFu, acc[h][m], 2);
        }
      if (seg_q0 == 0 && cur_q == P - 1) {
        // the CTA covered the whole row tile: store it
        if (tig == 0) {
#pragma unroll
          for (int h = 0; h < 2; ++h) {
            const int n = cur_rt * kRT + r_local + 8 * h;
            if (n < p.N)
#pragma unroll
              for (int m = 0; m < M; ++m) Y[(size_t)m * p.N + n] = __float2half_rn(acc[h][m]);
          }
        }
      } else {
        // a split segment: the tile's start (this CTA's last segment) or its
        // continuation (this CTA's first)
        finish_split(cur_rt, seg_q0 == 0 ? 0 : 1);
      }
#pragma unroll
      for (int h = 0; h < 2; ++h)
#pragma unroll
        for (int m = 0; m < M; ++m) acc[h][m] = 0.f;
      seg_q0 = 0;
    }
  }
  cp_async_wait<0>();
  // the last CTA to finish advances the epoch for the next call on this workspace
  __syncthreads();
  if (threadIdx.x == 0 && atomicAdd(&p.epoch[1], 1u) == (unsigned)(p.G - 1)) {
    p.epoch[1] = 0u;
    p.epoch[0] = p.epoch[0] + 1u;
  }
}

// ---------------------------------------------------------------- host side
size_t up256(size_t x) { return (x + 255) & ~size_t(255); }

struct Layout {
  int T, G, P;
  long long U;
  size_t smem;
  size_t off_part, total;
};

template <int M>
Layout layout_m(int64_t N, int64_t K, int num_sms) {
  using C = Cfg<M>;
  Layout L;
  const int64_t B = K / kBlock;
  L.P = (int)ceil_div(B, 2);
  L.T = (int)ceil_div(N, kRT);
  L.U = (long long)L.T * L.P;
  // at least two units per CTA and few enough that the CTA's block pairs fit
  // in shared memory; one CTA per SM while the work is small (up to eight
  // units per SM), so that consecutive calls' CTAs share the SMs and the next
  // call's prologue overlaps this one, else two per SM
  long long G = L.U / 2;
  const long long per_sm = L.U <= 8LL * num_sms ? 1 : 2;
  if (G > per_sm * num_sms) G = per_sm * num_sms;
  if (G < 1) G = 1;
  if (ceil_div(L.U, G) > C::kMaxPairs) G = ceil_div(L.U, C::kMaxPairs);
  if (G > kMaxG) G = kMaxG;
  L.G = (int)G;
  long long per = ceil_div(L.U, G);
  if (per > L.P) per = L.P;
  L.smem = (size_t)C::kRing + (size_t)per * C::kPairBytes;
  L.off_part = 0;
  L.total = L.off_part + up256((size_t)G * 2 * kRT * M * 8);
  return L;
}

Layout layout_for(int64_t M, int64_t N, int64_t K, int num_sms) {
  return M == 1 ? layout_m<1>(N, K, num_sms) : layout_m<2>(N, K, num_sms);
}

// ---- epoch slots: one per (device, workspace).  A slot's tickets are zero
// between calls, so a slot may pass to another workspace once the calls of
// its previous one are done: the slot reused is the least recently used one
// last used on the calling stream (ordered with this call), else the least
// recently used one.  (Calls in flight on other streams on more than
// kEpochSlots workspaces at once could share a slot: not supported.)
struct SlotTable {
  std::mutex mu;
  const void* ws[kEpochSlots] = {};
  cudaStream_t stream[kEpochSlots] = {};
  unsigned long long used[kEpochSlots] = {};
  unsigned long long clock = 0;
  unsigned* base = nullptr;
};
constexpr int kMaxDev = 64;
SlotTable g_slots[kMaxDev];

cudaError_t epoch_slot(const void* ws, cudaStream_t s, unsigned** out, unsigned* slot_out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDev) return cudaErrorInvalidDevice;
  SlotTable& t = g_slots[dev];
  std::lock_guard<std::mutex> lock(t.mu);
  if (!t.base) {
    void* ptr = nullptr;
    e = cudaGetSymbolAddress(&ptr, g_i8_epochs);
    if (e != cudaSuccess) return e;
    t.base = static_cast<unsigned*>(ptr);
  }
  int slot = -1, lru = 0, lru_same = -1;
  for (int i = 0; i < kEpochSlots; ++i) {
    if (t.ws[i] == ws) { slot = i; break; }
    if (t.used[i] < t.used[lru]) lru = i;
    if (t.stream[i] == s && (lru_same < 0 || t.used[i] < t.used[lru_same])) lru_same = i;
  }
  if (slot < 0) {
    // a reused slot keeps counting: stamps carry the slot index, so sums that
    // an earlier workspace left under another slot can never match
    slot = t.used[lru] == 0 ? lru : (lru_same >= 0 ? lru_same : lru);
    t.ws[slot] = ws;
  }
  t.stream[slot] = s;
  t.used[slot] = ++t.clock;
  *out = t.base + (size_t)kSlotWords * slot;
  *slot_out = (unsigned)slot;
  return cudaSuccess;
}

// the kernel's dynamic shared memory limit, raised once per device to the
// largest size any supported shape uses
template <int M>
size_t smem_limit() {
  return (size_t)Cfg<M>::kRing + (size_t)Cfg<M>::kMaxPairs * Cfg<M>::kPairBytes;
}

template <int M>
cudaError_t smem_attribute() {
  static std::once_flag once[kMaxDev];
  static cudaError_t err[kMaxDev];
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDev) return cudaErrorInvalidDevice;
  std::call_once(once[dev], [dev]() {
    err[dev] = cudaFuncSetAttribute(gemv_i8_kernel<M>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                    (int)smem_limit<M>());
  });
  return err[dev];
}

template <int M>
cudaError_t launch_m(const __half* X, const uint8_t* qs, const __half* d, __half* Y, int N, int K,
                     void* ws, int num_sms, cudaStream_t s) {
  const Layout L = layout_m<M>(N, K, num_sms);
  uint8_t* w = static_cast<uint8_t*>(ws);
  Params p;
  p.X = X;
  p.partials = reinterpret_cast<unsigned long long*>(w + L.off_part);
  cudaError_t e0 = epoch_slot(ws, s, &p.epoch, &p.slot);
  if (e0 != cudaSuccess) return e0;
  e0 = wait_status_word(&p.error);
  if (e0 != cudaSuccess) return e0;
  p.N = N; p.K = K; p.B = K / kBlock; p.P = L.P; p.T = L.T; p.G = L.G; p.U = L.U;
  p.k4 = 4; p.k16 = 16; p.k64 = 64;
  cudaError_t e = smem_attribute<M>();
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)L.G);
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = L.smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, gemv_i8_kernel<M>, qs, d, Y, p);
}

}  // namespace

// Shapes whose per-CTA block pairs fit in shared memory with two CTAs per SM
// (within the grid size limit; no CTA waits for another, so any grid runs).
bool gemv_i8_supported(int64_t M, int64_t N, int64_t K) {
  if (M >= 3) return gemv_i8n_supported(M, N, K);
  if (M < 1 || N < 1 || K < kBlock || K % kBlock) return false;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDev) return false;
  static std::once_flag once[kMaxDev];
  static int sm_count[kMaxDev];
  std::call_once(once[dev], [dev]() {
    if (cudaDeviceGetAttribute(&sm_count[dev], cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
      sm_count[dev] = 0;
  });
  const int sms = sm_count[dev];
  if (sms < 1) return false;
  const Layout L = layout_for(M, N, K, sms);
  long long per = ceil_div(L.U, L.G);
  if (per > L.P) per = L.P;
  return per <= (M == 1 ? Cfg<1>::kMaxPairs : Cfg<2>::kMaxPairs);
}

size_t gemv_i8_ws_bytes(int64_t M, int64_t N, int64_t K, int num_sms) {
  if (M >= 3) return gemv_i8n_ws_bytes(M, N, K, num_sms);
  return layout_for(M, N, K, num_sms).total;
}

cudaError_t launch_gemv_i8(const __half* X, const uint8_t* qs, const __half* d, __half* Y, int M,
                           int N, int K, void* ws, int num_sms, cudaStream_t s) {
  if (M == 1) return launch_m<1>(X, qs, d, Y, N, K, ws, num_sms, s);
  if (M == 2) return launch_m<2>(X, qs, d, Y, N, K, ws, num_sms, s);
  return launch_gemv_i8n(X, qs, d, Y, M, N, K, ws, num_sms, s);
}

}  // namespace tri
