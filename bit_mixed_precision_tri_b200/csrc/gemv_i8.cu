// Decode-regime ternary GEMV for one or two activation rows on the integer
// tensor-core path: exact int8 products of the packed weights (TQ2 fields, or
// TQ1 digit prefixes, see tq1_slot below) with fixed-point activation digits.
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
//    keeps four units of cp.async copies in flight (weights, and the rows'
//    block scales in the last 128 bytes of each stage), the first four
//    copied before the wait for the preceding grid.  The ring is walked with
//    a run-time stage index, so the loop body exists once in the instruction
//    stream.  A row tile split
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
// TQ1 weight stage: [row 0..15][112 bytes] (the pair's 104 bytes at offset 0
// or 8), spare words at 1792, block scales [row 0..15][8 bytes] at 1920
constexpr int kTq1RowStride = 112;
constexpr int kTq1ScaleOff = 1920;

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
template <int M, bool kTQ1> struct Cfg {
  static constexpr int kStages = 4;                       // pairs of weights in flight per warp
  // TQ2: [block h][row half][32 lanes][16 B], then the block scales
  // [row 0..15][8 B]; TQ1: rows of 112 B, spare words, then the scales
  static constexpr int kWStage = kTQ1 ? 2048 : 2176;
  static constexpr int kScaleOff = kTQ1 ? kTq1ScaleOff : 2048;
  static constexpr int kRing = kWarps * kStages * kWStage;
  static constexpr int kLevels = kTQ1 ? 4 : 3;            // activation digit levels per batch row
  static constexpr int kBL = 4 * kLevels * M;             // lanes with a B column (gid < kLevels M)
  static constexpr int kBSlots = kBL + 1;                 // + a zero slot
  static constexpr int kBlkBytes = 4 * kBSlots * 16;      // [i][slot][16 B]
  static constexpr int kPairBytes = 2 * kBlkBytes + 2 * 2 * M * 4;   // + [h][step M, bias M]
  static constexpr int kXs = kTQ1 ? kWarps * 256 * 4 : 0; // TQ1: per-warp staging of a block's x^
  // pairs whose records fit beside the ring with two CTAs per SM
  static constexpr int kMaxPairs = kTQ1 ? (M == 1 ? 17 : 9) : (M == 1 ? 27 : 14);
  static_assert(2 * (kRing + kXs + kMaxPairs * kPairBytes + 1024) <= 233472, "two CTAs per SM");
};

// TQ1 decode by digit prefixes.  For a TQ1 byte b ("Scaling Laws and
// Efficient Inference for Ternary Language Models", "1.6 bits per weight":
// the decoder multiplies by 3 and keeps the high byte), the j-th prefix
// F_j = floor(3^j b / 256) (j = 1..5, F_5 = the 5-digit number N) satisfies
// d_j = F_j - 3 F_{j-1} (F_0 = 0) for the j-th digit (first digit most
// significant).  Hence sum_j d_j x_j = sum_{j=1..5} F_j x'_j with
// x'_j = x_j - 3 x_{j+1} (x_6 = 0): the prefixes, each a byte, are the
// MMA's u8 operand and x' (from X, once per block) its activation.  Two
// bytes sit in the 16-bit halves of a word (b 3^j < 2^16 never carries
// across them), so a word of four TQ1 bytes gives its five prefix registers
// in two masks, ten multiplies and five byte permutes.
//
// Lane tig of a row owns 64 of the block's 256 prefix slots (51 full bytes
// x 5, and byte 51's F_1, whose other four digits are padding with x = 0):
// F_1..F_5 of the twelve bytes of words 3 tig .. 3 tig + 2 (registers
// 0..14), and one register from word 12 (bytes 48..51): F_{tig+1} of bytes
// 48, 49, 50, then F_1 of byte 51 (tig 0) or F_5 of byte 47 + tig.
// (TQ1 byte g, prefix j) of slot bi of prefix register ri of lane tig
__host__ __device__ inline void tq1_slot(int tig, int ri, int bi, int& g, int& jj) {
  if (ri < 15) {
    g = 4 * (3 * tig + ri / 5) + bi;
    jj = ri % 5 + 1;
  } else if (bi < 3) {
    g = 48 + bi;
    jj = tig + 1;
  } else if (tig == 0) {
    g = 51;
    jj = 1;
  } else {
    g = 47 + tig;
    jj = 5;
  }
}

__device__ __forceinline__ void cp_async_cg16(uint32_t dst, const void* src, uint32_t src_bytes) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src), "r"(src_bytes)
               : "memory");
}
__device__ __forceinline__ void cp_async_ca4(uint32_t dst, const void* src, uint32_t src_bytes) {
  asm volatile("cp.async.ca.shared.global [%0], [%1], 4, %2;" ::"r"(dst), "l"(src), "r"(src_bytes)
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

// The sixteen prefix registers of one row's block: words 3 tig .. 3 tig + 2
// (w0..w2) and word 12 (w12); emul = 3^(tig + 1), esel the permute that
// puts F_5 of byte 47 + tig into byte 3 (tig > 0).
__device__ __forceinline__ void tq1_prefixes(uint32_t w0, uint32_t w1, uint32_t w2, uint32_t w12,
                                             uint32_t emul, uint32_t esel, uint32_t (&A)[16]) {
  const uint32_t w[3] = {w0, w1, w2};
#pragma unroll
  for (int k = 0; k < 3; ++k) {
    const uint32_t ev = w[k] & 0x00FF00FFu;              // bytes 0, 2
    const uint32_t od = __byte_perm(w[k], 0u, 0x4341);   // bytes 1, 3
    uint32_t m = 1u;
#pragma unroll
    for (int jp = 1; jp <= 5; ++jp) {
      m *= 3u;                                           // 3^j (a constant)
      A[5 * k + jp - 1] = __byte_perm(ev * m, od * m, 0x7351);   // F_j of bytes 0, 1, 2, 3
    }
  }
  const uint32_t ev = w12 & 0x00FF00FFu, od = __byte_perm(w12, 0u, 0x4341);
  const uint32_t P = __byte_perm(ev * emul, od * emul, 0x7351);        // F_{tig+1} of bytes 48..51
  const uint32_t Q = __byte_perm(ev * 243u, od * 243u, 0x7351);        // F_5 of bytes 48..51
  A[15] = __byte_perm(P, Q, esel);
}

template <int M, bool kTQ1, bool kWide>
__global__ void __launch_bounds__(kThreads, 2)
gemv_i8_kernel(const uint8_t* __restrict__ qs, const __half* __restrict__ d, __half* __restrict__ Y,
               const Params p) {
  using C = Cfg<M, kTQ1>;
  constexpr int S = C::kStages;
  extern __shared__ __align__(16) uint8_t smem[];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int gid = lane >> 2, tig = lane & 3;
  const long long U = p.U, G = p.G;
  const long long u0 = range_start(blockIdx.x, U, G), u1 = range_start(blockIdx.x + 1, U, G);
  const int n_units = (int)(u1 - u0);
  const int B = p.B, P = p.P;                          // blocks and block pairs per row
  // packed bytes per row and per block pair
  const size_t rs = kTQ1 ? (size_t)(p.K / kBlock) * kTq1BlockBytes : (size_t)p.K / 4;
  constexpr int kPairRow = kTQ1 ? 2 * kTq1BlockBytes : 2 * kTq2BlockBytes;
  const uint32_t ring = ptx::smem_u32(smem) + warp * (S * C::kWStage);
  uint8_t* const pair_base = smem + C::kRing + C::kXs;
  const uint32_t pairs = ptx::smem_u32(pair_base);
  const int q0 = (int)(u0 % P);

  // ---- producer state: next unit to copy
  int il = 0;                                          // units issued
  int rt_l = (int)(u0 / P), q_l = q0;
  // rows outside the matrix copy 0 bytes (zero fill) from a valid address
  const uint8_t* pa = qs;                             // row gid, block 2 q_l
  const uint8_t* pb = qs;                             // row gid + 8
  // TQ1 with 16-byte aligned rows: the warp copies its 16 rows' 112-byte
  // windows (7 chunks each) in four 16-byte copies per lane; chunk
  // i = 32 c + lane is chunk i % 7 of row i / 7
  const uint8_t* wrow[4] = {qs, qs, qs, qs};
  uint32_t wsz[4] = {0, 0, 0, 0};
  const unsigned short* ds_p = nullptr;               // this lane's scale row, block 2 q_l
  uint32_t szS = 0;
  const uintptr_t d_end = reinterpret_cast<uintptr_t>(d) + (size_t)p.N * B * 2;
  uint32_t szA = 0, szB = 0;
  const bool odd_b = (B & 1) != 0;
  auto set_rows = [&]() {
    const int rowA = rt_l * kRT + warp * 16 + gid;
    szA = rowA < p.N ? 16u : 0u;
    szB = rowA + 8 < p.N ? 16u : 0u;
    const int ra = szA ? rowA : 0, rb = szB ? rowA + 8 : 0;
    // TQ2: bytes 16 tig .. +16 of each 64-byte block row; TQ1: the pair
    pa = qs + (size_t)ra * rs + (size_t)q_l * kPairRow + (kTQ1 ? 0 : tig * 16);
    pb = qs + (size_t)rb * rs + (size_t)q_l * kPairRow + (kTQ1 ? 0 : tig * 16);
    if constexpr (kTQ1 && kWide) {
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        const int i = 32 * c + lane, row = rt_l * kRT + warp * 16 + i / 7;
        const bool ok = i < 112 && row < p.N;
        wrow[c] = qs + (size_t)(ok ? row : 0) * rs + 16 * (i % 7);
        wsz[c] = ok ? 16u : 0u;
      }
    }
    {
      // lane (gid, tig) copies word tig & 1 of the 8-byte window (from the
      // 4-byte boundary at or below the pair's two scales) of row
      // gid + 8 (tig >> 1)
      const int rowS = rt_l * kRT + warp * 16 + gid + 8 * (tig >> 1);
      szS = rowS < p.N ? 4u : 0u;
      ds_p = reinterpret_cast<const unsigned short*>(d) + (size_t)(szS ? rowS : 0) * B + 2 * q_l;
    }
  };
  set_rows();
  // weights and block scales of the next unit into ring stage s
  auto issue = [&](int s, bool commit) {
    if (il < n_units) {
      const uint32_t st = ring + s * C::kWStage + lane * 16;
      const bool h1 = !(odd_b && q_l == P - 1);       // odd B: the last pair has one block
      const uint32_t s1a = h1 ? szA : 0u, s1b = h1 ? szB : 0u;
      if constexpr (kTQ1) {
        // stage layout: row r (0..15) of the warp at 112 r, the pair's 104
        // bytes from offset 8 (q odd, wide) or 0
        const uint32_t st0 = ring + s * C::kWStage;
        if constexpr (kWide) {
          // B % 4 == 0: rows are 16-byte aligned and the pair starts 8 bytes
          // past a boundary when q is odd; the 112-byte window never leaves
          // the row
          const int qo = kPairRow * q_l - 8 * (q_l & 1);
#pragma unroll
          for (int c = 0; c < 4; ++c)
            if (c < 3 || lane < 16) cp_async_cg16(st0 + 16 * (32 * c + lane), wrow[c] + qo, wsz[c]);
        } else {
          // 4-byte rows: every lane copies the words it reads, words 3 tig ..
          // 3 tig + 2 of rows gid and gid + 8, and lane tig 0 word 12 (the
          // others copy nothing to a spare slot past the rows)
#pragma unroll
          for (int h = 0; h < 2; ++h)
#pragma unroll
            for (int rr = 0; rr < 2; ++rr) {
              const uint8_t* src = (rr ? pb : pa) + (h && h1 ? kTq1BlockBytes : 0);
              const uint32_t sz = ((rr ? szB : szA) >> 2) * (h == 0 || h1 ? 1u : 0u);
              const uint32_t dst = st0 + (gid + 8 * rr) * 112 + kTq1BlockBytes * h;
#pragma unroll
              for (int c = 0; c < 3; ++c) cp_async_ca4(dst + 12 * tig + 4 * c, src + 12 * tig + 4 * c, sz);
              cp_async_ca4(tig == 0 ? dst + 48 : st0 + 16 * 112 + 4 * lane, src + 48, tig == 0 ? sz : 0u);
            }
        }
      } else {
        const int o1 = h1 ? kTq2BlockBytes : 0;
        cp_async_cg16(st, pa, szA);
        cp_async_cg16(st + 512, pb, szB);
        cp_async_cg16(st + 1024, pa + o1, s1a);
        cp_async_cg16(st + 1536, pb + o1, s1b);
      }
      {
        // block scales into the stage's last 128 bytes: [row 0..15][8 bytes]
        const uintptr_t a4 = (reinterpret_cast<uintptr_t>(ds_p) & ~uintptr_t(3)) + 4 * (tig & 1);
        const uint32_t sz = a4 + 4 <= d_end ? szS : (a4 < d_end ? (uint32_t)(d_end - a4) : 0u) * (szS ? 1u : 0u);
        cp_async_ca4(ring + s * C::kWStage + C::kScaleOff + (gid + 8 * (tig >> 1)) * 8 + 4 * (tig & 1),
                     reinterpret_cast<const void*>(a4 < d_end ? a4 : reinterpret_cast<uintptr_t>(d)), sz);
      }
      ++il;
      if (++q_l == P) {
        q_l = 0;
        ++rt_l;
        set_rows();
      } else {
        pa += kPairRow;
        pb += kPairRow;
        ds_p += 2;
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
      *reinterpret_cast<uint4*>(pair_base + (hb >> 1) * C::kPairBytes + (hb & 1) * C::kBlkBytes +
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
    // TQ1: this lane's eight slots (prefix registers 2 (L % 8) + r of lane
    // tig = L / 8, bytes bi): the index k0 of x_j, whether x_{j+1} enters
    // (j < 5 inside the block), and the record offset of the words
    int tq_k0[8];
    uint32_t tq_two = 0;
    const int tq_rec = (((lane & 7) >> 1) * C::kBSlots + (lane >> 3)) * 16 + (lane & 1) * 8;
    if constexpr (kTQ1) {
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        int g, jp;
        tq1_slot(lane >> 3, 2 * (lane & 7) + (e >> 2), e & 3, g, jp);
        tq_k0[e] = 5 * g + jp - 1;
        if (jp < 5 && tq_k0[e] + 1 < kBlock) tq_two |= 1u << e;
      }
    }
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
        uint8_t* rec = pair_base + jj * C::kPairBytes + h * C::kBlkBytes;
        float* sc = reinterpret_cast<float*>(pair_base + jj * C::kPairBytes + 2 * C::kBlkBytes) + h * 2 * M;
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
          int sum = 0;
          if constexpr (kTQ1) {
            // x^ of the block into the warp's staging row, then each lane
            // writes the words of prefix register pair (2i, 2i+1), i = L % 8,
            // of lane tig = L / 8: x' = x^_{5g+j-1} - 3 x^_{5g+j} (x^_{5g+5}
            // for j = 5; positions past the block's 256 are padding, x = 0)
            // in four balanced base-256 digits (|x'| < 2^25), level lv =
            // column 4m + lv holding digit 3 - lv
            int* xs = reinterpret_cast<int*>(smem + C::kRing) + warp * 256;
            int qv[8];
#pragma unroll
            for (int e = 0; e < 8; ++e) {
              qv[e] = __float2int_rn(xv[e] * inv);   // |q| <= 8e6 < 2^23
              sum += qv[e];
            }
            reinterpret_cast<int4*>(xs)[2 * lane] = make_int4(qv[0], qv[1], qv[2], qv[3]);
            reinterpret_cast<int4*>(xs)[2 * lane + 1] = make_int4(qv[4], qv[5], qv[6], qv[7]);
            __syncwarp();
#pragma unroll
            for (int r = 0; r < 2; ++r) {
              uint32_t dg[4];
#pragma unroll
              for (int bi = 0; bi < 4; ++bi) {
                const int e = 4 * r + bi;
                const int a = xs[tq_k0[e]];
                const int b = (tq_two >> e) & 1u ? xs[tq_k0[e] + 1] : 0;
                dg[bi] = ((uint32_t)(a - 3 * b) + 0x80808080u) ^ 0x80808080u;
              }
#pragma unroll
              for (int lv = 0; lv < 4; ++lv) {
                const uint32_t sel = (uint32_t)(3 - lv) | ((uint32_t)(7 - lv) << 4);
                const uint32_t lo = __byte_perm(dg[0], dg[1], sel), hi = __byte_perm(dg[2], dg[3], sel);
                const uint32_t word = (lo & 0xFFFFu) | (hi << 16);
                *reinterpret_cast<uint32_t*>(rec + tq_rec + (4 * m + lv) * 4 * 16 + r * 4) = word;
              }
            }
            __syncwarp();                             // the staging row is free for the next block
          } else {
          // Balanced base-256 digits of q, as bytes: with u = q + 0x808080
          // (in [0, 2^24) for |q| <= 8e6), byte i of u is digit i + 128, so
          // byte i of u ^ 0x808080 is digit i as a signed byte (byte 0 the
          // lowest digit, byte 2 the highest).
          uint32_t dg[8];
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
          }
          sum = __reduce_add_sync(0xFFFFFFFFu, sum);
          if (lane == 0) {
            // TQ2: the field masks scale products by 4^g and the chains are
            // combined as 64 c0 + 16 c1 + 4 c2 + c3, i.e. 64 sum d' x^
            // TQ1: the step and sum_k x^_k as integer bits (the bias is
            // subtracted exactly)
            constexpr float kScale = kTQ1 ? 1.f : 64.f;
            sc[m] = amax > 0.f ? (amax / kQMax) / kScale : 0.f;   // s_b / scale
            sc[M + m] = kTQ1 ? __int_as_float(sum) : kScale * (float)sum;
          }
        }
      }
    }

  }
  __syncthreads();                                    // fragments visible to every warp

  // TQ2: the columns this thread holds in C (2tig, 2tig+1): batch row and
  // level weight (65536, 256, 1 for levels 0, 1, 2); the bias of batch row m
  // is subtracted once, by the threads with tig == 0
  float wA[M], wB[M], wBias[M];
#pragma unroll
  for (int m = 0; m < M; ++m) {
    const int la = 2 * tig - 3 * m, lb = 2 * tig + 1 - 3 * m;   // level within batch row m
    auto lw = [](int l) { return l == 0 ? 65536.f : l == 1 ? 256.f : l == 2 ? 1.f : 0.f; };
    wA[m] = la >= 0 && la < 3 ? lw(la) : 0.f;
    wB[m] = lb >= 0 && lb < 3 ? lw(lb) : 0.f;
    wBias[m] = tig == 0 ? -1.f : 0.f;
  }
  // TQ1: 3^(tig + 1), and the permute that takes byte 3 of the edge
  // register from F_5 of byte 47 + tig (tig > 0)
  const uint32_t emul = tig == 0 ? 3u : tig == 1 ? 9u : tig == 2 ? 27u : 81u;
  const uint32_t esel = tig == 0 ? 0x3210u : (0x0210u | ((3u + (uint32_t)tig) << 12));
  const int k4 = p.k4, k16 = p.k16, k64 = p.k64;
  const uint32_t bfrag = pairs + (lane < C::kBL ? lane : C::kBL) * 16;

  float acc[2][M];
#pragma unroll
  for (int h = 0; h < 2; ++h)
#pragma unroll
    for (int m = 0; m < M; ++m) acc[h][m] = 0.f;
  int rt = (int)(u0 / P), q = q0;
  int j = 0;
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

  // End of a segment of row tile `tile` (the unit just consumed closed it):
  // the four threads of a row add their sums; a segment that covered the
  // whole tile stores it, a split one (side 0: the tile's start, i.e. this
  // CTA's last segment; side 1: its continuation, i.e. this CTA's first)
  // is finished by the tile's last contributor.
  auto end_segment = [&](int tile, bool whole, int side) {
#pragma unroll
    for (int h = 0; h < 2; ++h)
#pragma unroll
      for (int m = 0; m < M; ++m) {
        acc[h][m] += __shfl_xor_sync(0xFFFFFFFFu, acc[h][m], 1);
        acc[h][m] += __shfl_xor_sync(0xFFFFFFFFu, acc[h][m], 2);
      }
    if (whole) {
      if (tig == 0) {
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          const int n = tile * kRT + r_local + 8 * h;
          if (n < p.N)
#pragma unroll
            for (int m = 0; m < M; ++m) Y[(size_t)m * p.N + n] = __float2half_rn(acc[h][m]);
        }
      }
    } else {
      finish_split(tile, side);
    }
#pragma unroll
    for (int h = 0; h < 2; ++h)
#pragma unroll
      for (int m = 0; m < M; ++m) acc[h][m] = 0.f;
  };

  // One unit per iteration with the stage index at run time, so that the
  // loop body is emitted once (unrolled over the ring's stages, the body and
  // the split-tile finish overflowed the instruction cache: ncu counted
  // 1-2.5 cycles per issued instruction waiting for instructions).  The
  // segment ends (row tile ends and the range end) are handled between the
  // inner loops.  fp16 scale pair of a row from its 8-byte window: the
  // scales start at byte 2 of it when (row B) is odd.
  const uint32_t dsel = (gid & 1) && (B & 1) ? 0x5432u : 0x3210u;
  int s = 0;
  for (int u = 0; u < n_units;) {
    const int seg_q0 = q, seg_rt = rt;
    const int seg_len = n_units - u < P - q ? n_units - u : P - q;
#pragma unroll 1
    for (int k = 0; k < seg_len; ++k) {
      cp_async_wait<S - 1>();
      __syncwarp();                                   // the scales (and TQ1 rows) are other lanes' copies
      const uint32_t st0 = ring + s * C::kWStage;
      // TQ1: words 3 tig .. 3 tig + 2 and 12 of [block h][row gid, gid + 8];
      // TQ2: this lane's 16 bytes of [block h][row gid, gid + 8]
      uint32_t tw[2][2][4];
      if constexpr (kTQ1) {
        const uint32_t r0 = st0 + gid * kTq1RowStride + (kWide ? 8 * (q & 1) : 0);
#pragma unroll
        for (int h = 0; h < 2; ++h)
#pragma unroll
          for (int rr = 0; rr < 2; ++rr) {
            const uint32_t base = r0 + rr * 8 * kTq1RowStride + kTq1BlockBytes * h;
#pragma unroll
            for (int c3 = 0; c3 < 3; ++c3) tw[h][rr][c3] = ptx::lds32(base + 12 * tig + 4 * c3);
            tw[h][rr][3] = ptx::lds32(base + 48);
          }
      } else {
#pragma unroll
        for (int h = 0; h < 2; ++h)
#pragma unroll
          for (int rr = 0; rr < 2; ++rr) {
            const uint4 v = ptx::lds128(st0 + lane * 16 + h * 1024 + rr * 512);
            tw[h][rr][0] = v.x;
            tw[h][rr][1] = v.y;
            tw[h][rr][2] = v.z;
            tw[h][rr][3] = v.w;
          }
      }
      const uint2 sa = ptx::lds64(st0 + C::kScaleOff + gid * 8);
      const uint2 sb = ptx::lds64(st0 + C::kScaleOff + (gid + 8) * 8);
      __syncwarp();                                   // read: the stage may be refilled
      issue(s, true);
      // scales [row half] as (block 0, block 1) fp16 pairs; an odd B's last
      // pair has one block, whose scale stands in for the missing one (its
      // weights and activations are zero)
      const bool h1 = !((B & 1) && q == P - 1);
      uint32_t dpair[2] = {__byte_perm(sa.x, sa.y, dsel), __byte_perm(sb.x, sb.y, dsel)};
      if (!h1) {
        dpair[0] = __byte_perm(dpair[0], 0u, 0x1010);
        dpair[1] = __byte_perm(dpair[1], 0u, 0x1010);
      }
      const uint32_t pj = bfrag + j * C::kPairBytes;
      const float* sc = reinterpret_cast<const float*>(pair_base + j * C::kPairBytes + 2 * C::kBlkBytes);
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        uint4 bf[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) bf[i] = ptx::lds128(pj + h * C::kBlkBytes + i * C::kBSlots * 16);
        const uint32_t bw[16] = {bf[0].x, bf[0].y, bf[0].z, bf[0].w, bf[1].x, bf[1].y, bf[1].z, bf[1].w,
                                 bf[2].x, bf[2].y, bf[2].z, bf[2].w, bf[3].x, bf[3].y, bf[3].z, bf[3].w};
        const float da0 = __half2float(__ushort_as_half((unsigned short)(dpair[0] >> (16 * h))));
        const float da1 = __half2float(__ushort_as_half((unsigned short)(dpair[1] >> (16 * h))));
        int c[4][4];
        if constexpr (kTQ1) {
          // prefix registers of rows gid and gid + 8; MMA i takes registers
          // 2i, 2i+1 of each row (chain i % 4)
          uint32_t Aa[16], Ab[16];
          tq1_prefixes(tw[h][0][0], tw[h][0][1], tw[h][0][2], tw[h][0][3], emul, esel, Aa);
          tq1_prefixes(tw[h][1][0], tw[h][1][1], tw[h][1][2], tw[h][1][3], emul, esel, Ab);
#pragma unroll
          for (int i = 0; i < 4; ++i)
            mma_u8s8_z(c[i], Aa[2 * i], Ab[2 * i], Aa[2 * i + 1], Ab[2 * i + 1], bw[2 * i], bw[2 * i + 1]);
#pragma unroll
          for (int i = 4; i < 8; ++i)
            mma_u8s8(c[i - 4], Aa[2 * i], Ab[2 * i], Aa[2 * i + 1], Ab[2 * i + 1], bw[2 * i], bw[2 * i + 1]);
          // The level sums of one row cancel to far below their size (the
          // prefix weights telescope), so they are combined exactly: every
          // thread forms 256 c_even + c_odd of its two columns (|.| < 2^31),
          // and the thread holding level 0 of batch row m adds its partner's
          // pair and the bias in 64-bit integers, 2^16 P_0 + P_1 - sum x^,
          // then rounds once.
          int pv[2];
#pragma unroll
          for (int r = 0; r < 2; ++r)
            pv[r] = (c[0][2 * r] + c[1][2 * r] + c[2][2 * r] + c[3][2 * r]) * 256 +
                    (c[0][2 * r + 1] + c[1][2 * r + 1] + c[2][2 * r + 1] + c[3][2 * r + 1]);
          const int po0 = __shfl_xor_sync(0xFFFFFFFFu, pv[0], 1);
          const int po1 = __shfl_xor_sync(0xFFFFFFFFu, pv[1], 1);
#pragma unroll
          for (int m = 0; m < M; ++m) {
            const float st = sc[h * 2 * M + m];
            const long long xsum = __float_as_int(sc[h * 2 * M + M + m]);
            const long long s0 = (long long)pv[0] * 65536 + po0 - xsum;
            const long long s1 = (long long)pv[1] * 65536 + po1 - xsum;
            const bool own = tig == 2 * m;
            acc[0][m] = fmaf(own ? (float)s0 : 0.f, st * da0, acc[0][m]);
            acc[1][m] = fmaf(own ? (float)s1 : 0.f, st * da1, acc[1][m]);
          }
        } else {
          // field g of rows gid (words 0..3 of tw[h][0]) and gid + 8
#pragma unroll
          for (int g = 0; g < 4; ++g) {
            const uint32_t mask = 0x03030303u << (2 * g);
            mma_u8s8_z(c[g], tw[h][0][0] & mask, tw[h][1][0] & mask, tw[h][0][1] & mask, tw[h][1][1] & mask,
                       bw[g * 2], bw[g * 2 + 1]);
          }
#pragma unroll
          for (int g = 0; g < 4; ++g) {
            const uint32_t mask = 0x03030303u << (2 * g);
            mma_u8s8(c[g], tw[h][0][2] & mask, tw[h][1][2] & mask, tw[h][0][3] & mask, tw[h][1][3] & mask,
                     bw[(4 + g) * 2], bw[(4 + g) * 2 + 1]);
          }
          float fv[4];
#pragma unroll
          for (int e = 0; e < 4; ++e)
            fv[e] = (float)(c[3][e] + c[2][e] * k4 + c[1][e] * k16 + c[0][e] * k64);
#pragma unroll
          for (int m = 0; m < M; ++m) {
            const float st = sc[h * 2 * M + m], nb = wBias[m] * sc[h * 2 * M + M + m];
            const float f0 = fmaf(wA[m], fv[0], fmaf(wB[m], fv[1], nb));
            const float f1 = fmaf(wA[m], fv[2], fmaf(wB[m], fv[3], nb));
            acc[0][m] = fmaf(f0, st * da0, acc[0][m]);
            acc[1][m] = fmaf(f1, st * da1, acc[1][m]);
          }
        }
      }
      s = (s + 1) & (S - 1);
      if (++j == P) j = 0;                            // slot of pair q: (q - q0) mod P
      ++q;
    }
    u += seg_len;
    const bool whole = seg_q0 == 0 && q == P;
    if (q == P) {
      q = 0;
      ++rt;
    }
    end_segment(seg_rt, whole, seg_q0 == 0 ? 0 : 1);
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

template <int M, bool kTQ1>
Layout layout_m(int64_t N, int64_t K, int num_sms) {
  using C = Cfg<M, kTQ1>;
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
  L.smem = (size_t)C::kRing + (size_t)C::kXs + (size_t)per * C::kPairBytes;
  L.off_part = 0;
  L.total = L.off_part + up256((size_t)G * 2 * kRT * M * 8);
  return L;
}

Layout layout_for(int64_t M, int64_t N, int64_t K, int num_sms, bool tq1) {
  if (tq1) return M == 1 ? layout_m<1, true>(N, K, num_sms) : layout_m<2, true>(N, K, num_sms);
  return M == 1 ? layout_m<1, false>(N, K, num_sms) : layout_m<2, false>(N, K, num_sms);
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
template <int M, bool kTQ1>
size_t smem_limit() {
  using C = Cfg<M, kTQ1>;
  return (size_t)C::kRing + (size_t)C::kXs + (size_t)C::kMaxPairs * C::kPairBytes;
}

template <int M, bool kTQ1, bool kWide>
cudaError_t smem_attribute() {
  static std::once_flag once[kMaxDev];
  static cudaError_t err[kMaxDev];
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDev) return cudaErrorInvalidDevice;
  std::call_once(once[dev], [dev]() {
    err[dev] = cudaFuncSetAttribute(gemv_i8_kernel<M, kTQ1, kWide>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                    (int)smem_limit<M, kTQ1>());
  });
  return err[dev];
}

template <int M, bool kTQ1>
cudaError_t launch_m(const __half* X, const uint8_t* qs, const __half* d, __half* Y, int N, int K,
                     void* ws, int num_sms, cudaStream_t s) {
  const Layout L = layout_m<M, kTQ1>(N, K, num_sms);
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
  // TQ1 rows are copied in 16-byte chunks when they start on 16-byte
  // boundaries (B % 4 == 0 and an aligned plane), else word by word
  const bool wide = kTQ1 && p.B % 4 == 0 && reinterpret_cast<uintptr_t>(qs) % 16 == 0;
  cudaError_t e = cudaSuccess;
  if constexpr (kTQ1) e = wide ? smem_attribute<M, true, true>() : smem_attribute<M, true, false>();
  else e = smem_attribute<M, false, false>();
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
  if constexpr (kTQ1) {
    if (wide) return cudaLaunchKernelEx(&cfg, gemv_i8_kernel<M, true, true>, qs, d, Y, p);
    return cudaLaunchKernelEx(&cfg, gemv_i8_kernel<M, true, false>, qs, d, Y, p);
  } else {
    return cudaLaunchKernelEx(&cfg, gemv_i8_kernel<M, false, false>, qs, d, Y, p);
  }
}

}  // namespace

// Shapes whose per-CTA block pairs fit in shared memory with two CTAs per SM
// (within the grid size limit; no CTA waits for another, so any grid runs).
// TQ1 planes are read directly at M <= 2; 3 <= M <= 16 takes TQ2 only.
bool gemv_i8_supported(int64_t M, int64_t N, int64_t K, bool tq1) {
  if (M >= 3) return !tq1 && gemv_i8n_supported(M, N, K);
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
  const Layout L = layout_for(M, N, K, sms, tq1);
  long long per = ceil_div(L.U, L.G);
  if (per > L.P) per = L.P;
  const int max_pairs = tq1 ? (M == 1 ? Cfg<1, true>::kMaxPairs : Cfg<2, true>::kMaxPairs)
                            : (M == 1 ? Cfg<1, false>::kMaxPairs : Cfg<2, false>::kMaxPairs);
  return per <= max_pairs;
}

size_t gemv_i8_ws_bytes(int64_t M, int64_t N, int64_t K, int num_sms, bool tq1) {
  if (M >= 3) return gemv_i8n_ws_bytes(M, N, K, num_sms);
  return layout_for(M, N, K, num_sms, tq1).total;
}

cudaError_t launch_gemv_i8(const __half* X, const uint8_t* qs, const __half* d, __half* Y, int M,
                           int N, int K, void* ws, int num_sms, cudaStream_t s, bool tq1) {
  if (tq1) {
    if (M == 1) return launch_m<1, true>(X, qs, d, Y, N, K, ws, num_sms, s);
    if (M == 2) return launch_m<2, true>(X, qs, d, Y, N, K, ws, num_sms, s);
    return cudaErrorInvalidValue;
  }
  if (M == 1) return launch_m<1, false>(X, qs, d, Y, N, K, ws, num_sms, s);
  if (M == 2) return launch_m<2, false>(X, qs, d, Y, N, K, ws, num_sms, s);
  return launch_gemv_i8n(X, qs, d, Y, M, N, K, ws, num_sms, s);
}

}  // namespace tri
