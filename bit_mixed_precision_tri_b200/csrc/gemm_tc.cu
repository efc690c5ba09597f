// Compute-regime ternary GEMM (M >= 17) for TQ2 weights on sm_100a.
//
// Y = X (d * W_hat)^T ("Scaling Laws and Efficient Inference for Ternary
// Language Models", section "The model", step 3) once the batch is large
// enough that arithmetic, not weight traffic, bounds the layer (section
// "TriRun: ternary inference on GPUs": the speedup falls once the product
// becomes compute-bound).  The pages' kernel used mma.sync; this one uses the
// fifth-generation tensor cores with the decoded weights in tensor memory,
// computing the transposed product Y^T = (d * W_hat) X^T tile by tile:
//
//  * a tile is 128 weight rows (the MMA's M, one TMEM lane per row) by NB <= 256
//    activation rows (the MMA's N); its K range may be split over the CTAs of
//    a thread-block cluster;
//  * two producer threads TMA-load, per 64-wide K step, the activation tile
//    (NB rows x 64 fp16, 128-byte swizzle) straight from X; a third loads the
//    packed weights one 256-wide block at a time (128 rows x 64 B, 64-byte
//    swizzle).  A single issuing thread is latency-bound near one TMA load per
//    ~300 cycles, so the loads are spread over threads;
//  * eight decoder warps (two per TMEM lane quarter, one K half each) turn
//    each byte's four 2-bit fields into two fp16 pairs (w_k, w_k+1) = t * d in
//    natural K order (byte spread + mask + OR with fp16 exponents, subtract the
//    bias, multiply by the block scale -- all exact) and store them into a
//    ring of A slots in tensor memory with tcgen05.st, so the decoded weights
//    never touch shared memory and X needs no reordering;
//  * one thread issues tcgen05.mma (M = 128, N = NB, K = 16, fp32 accumulate)
//    with A in tensor memory and the activations in shared memory.  That
//    thread is a serial latency chain, so stages move in pairs: one barrier
//    wait, eight MMAs and one commit per 128 of K; the commit frees both
//    activation buffers and both A slots of the pair;
//  * the epilogue reads the accumulator with tcgen05.ld.  When K is split, the
//    CTAs of the cluster each own some 32-column slices of the tile: the
//    others write their partial slices to an L2-resident scratch, the cluster
//    synchronises once, and each owner adds the slices in cluster-rank order,
//    so results are deterministic (no atomics, no tickets).
#include <cudaTypedefs.h>

#include "sm100_ptx.cuh"
#include "tri_internal.cuh"

namespace tri {
namespace {

constexpr int kRows = 128;                        // weight rows per tile (MMA M, TMEM lanes)
constexpr int BK = 64;                            // K per MMA stage: one 128-byte swizzle row
constexpr int kStepsPerBlock = kBlock / BK;       // 4
constexpr int kPBytes = kRows * (kBlock / 4);     // packed block tile: 8 KB
constexpr int kPStages = 4;
constexpr int kMaxStages = 8;                     // activation stages = A slots
constexpr int kAColBase = 256;                    // A slots live after the accumulator columns
constexpr int kACols = BK / 2;                    // 64 fp16 per lane = 32 columns
constexpr int kFirstDec = 4;                      // warps 0,2: X producers; 1: MMA; 3: P producer
constexpr int kDecWarps = 8;
constexpr int kThreads = (kFirstDec + kDecWarps) * 32;
constexpr int kRingBudget = 192 * 1024;
constexpr int kMinSmem = 120 * 1024;              // > half an SM: one CTA (and TMEM owner) per SM
constexpr int kChunkF4 = kRows * 8;               // one 32-column slice of a partial tile (float4)

// most chunks a rank sends (it owns at least floor(nch / sp) of the nch chunks)
__host__ __device__ constexpr int max_out_chunks(int nch, int sp) { return nch - nch / sp; }
// chunks below c that rank `rank` owns
__host__ __device__ constexpr int owned_below(int c, int rank, int sp) { return c > rank ? (c - rank + sp - 1) / sp : 0; }
constexpr uint32_t kWaitLimit = 1u << 18;   // mbarrier polls: ~4 us each when pending, ~1 s in all

struct TcParams {
  unsigned* error;
  float4* scratch;     // split-K partial slices [tile][rank][out chunk][8][128] (float4)
  int M, N, K, B;      // B = K / 256 blocks
  int NB;              // activation rows per tile (MMA N)
  int S;               // activation stages (even, <= kMaxStages)
  int splits;          // CTAs per cluster sharing one tile's K range
};

size_t smem_bytes(int NB, int S) {
  const size_t need = 1024 + (size_t)S * NB * 128 + (size_t)kPStages * kPBytes +
                      (kMaxStages + 2 * kPStages + 1) * 8 + 16;
  return need < (size_t)kMinSmem ? (size_t)kMinSmem : need;
}

// Two fp16 weights (w_k, w_k+1) of one byte (spread into both 16-bit halves):
// field 2f in the low half, field 2f+1 in the high half, each read as the low
// mantissa bits of an fp16 constant, minus (constant + 1) gives the trit
// exactly; times the block scale gives t * d exactly.
template <int F>
__device__ __forceinline__ uint32_t pair_of(uint32_t spread, __half2 dd) {
  constexpr uint32_t mask = F == 0 ? 0x000C0003u : 0x00C00030u;
  constexpr uint32_t expo = F == 0 ? 0x5C006400u : 0x4C005400u;   // 256 | 1024, 16 | 64
  constexpr uint32_t bias = F == 0 ? 0x5C046401u : 0x4C405410u;   // 257 | 1025, 17 | 65
  const uint32_t h = (spread & mask) | expo;
  const uint32_t b = bias;
  __half2 t = __hsub2(*reinterpret_cast<const __half2*>(&h), *reinterpret_cast<const __half2*>(&b));
  t = __hmul2(t, dd);
  return *reinterpret_cast<uint32_t*>(&t);
}

__device__ __forceinline__ void store_y(__half* __restrict__ Y, const uint32_t (&v)[32], int n,
                                        int mbase, int lim, int N) {
#pragma unroll
  for (int e = 0; e < 32; ++e)
    if (e < lim) Y[(size_t)(mbase + e) * N + n] = __float2half_rn(__uint_as_float(v[e]));
}

template <int G>
__global__ void __launch_bounds__(kThreads, 1)
gemm_tc_kernel(const __grid_constant__ CUtensorMap xmap, const __grid_constant__ CUtensorMap qmap,
               const __half* __restrict__ dsc, __half* __restrict__ Y, const TcParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int S = p.S, NB = p.NB, PS = S / G;          // stages move in groups of G: one barrier phase
  const uint32_t XB = (uint32_t)NB * 128;
  uint8_t* xs = smem;                                            // S x XB (1024-aligned)
  uint8_t* ps = xs + (size_t)S * XB;                             // kPStages x kPBytes
  uint64_t* full = reinterpret_cast<uint64_t*>(ps + kPStages * kPBytes);   // per stage pair
  uint64_t* empty = full + kMaxStages / 2;
  uint64_t* pfull = empty + kMaxStages / 2;
  uint64_t* pempty = pfull + kPStages;
  uint64_t* accf = pempty + kPStages;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(accf + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int n_tile = blockIdx.x, m_tile = blockIdx.y, split = blockIdx.z;
  const int b0 = (int)((int64_t)p.B * split / p.splits);
  const int nblk = (int)((int64_t)p.B * (split + 1) / p.splits) - b0;
  const int nks = nblk * kStepsPerBlock;
  const int ngroups = nks / G;

  ptx::griddep_launch_dependents();
  if (threadIdx.x == 0) {
    for (int s = 0; s < PS; ++s) {
      ptx::mbar_init(&full[s], kDecWarps + 2);     // 8 decoder warps + both X producers (with tx)
      ptx::mbar_init(&empty[s], 1);                // MMA commit
    }
    for (int s = 0; s < kPStages; ++s) {
      ptx::mbar_init(&pfull[s], 1);
      ptx::mbar_init(&pempty[s], kDecWarps);
    }
    ptx::mbar_init(accf, 1);
    ptx::fence_mbar_init();
  }
  if (warp == 1) {
    ptx::tmem_alloc(tmem_slot, 512);
    ptx::tmem_relinquish();
  }
  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  // decoder / epilogue geometry (meaningful for warps >= kFirstDec)
  const int q = warp & 3, h = (warp - kFirstDec) >> 2;
  const int r = 32 * q + lane;                         // weight row in the tile = TMEM lane
  const int n = n_tile * kRows + r;
  const uint32_t lane_base = tmem + ((uint32_t)(32 * q) << 16);
  uint32_t limit = kWaitLimit;

  if ((warp == 0 || warp == 2) && lane == 0) {
    // -------------------------------------------------- activation producers
    ptx::prefetch_tensormap(&xmap);
    uint64_t pol_x;
    asm volatile("createpolicy.fractional.L2::evict_last.b64 %0, 1.0;" : "=l"(pol_x));
    ptx::griddep_wait();           // X may be the previous kernel's output
    const int u = warp >> 1;      // this producer loads the even (0) or odd (1) steps of each group
    int pr = 0, round = 0;
    for (int k = 0; k < ngroups; ++k) {
      if (round > 0 && !ptx::mbar_wait(&empty[pr], (uint32_t)((round - 1) & 1), limit)) {
        ptx::record_wait_failure(p.error, 21u);
        limit = 1;
      }
      ptx::mbar_arrive_expect_tx(&full[pr], XB * (G / 2));
#pragma unroll
      for (int v = u; v < G; v += 2)
        ptx::tma_load_2d(xs + (size_t)(G * pr + v) * XB, &xmap, (b0 * kStepsPerBlock + G * k + v) * BK,
                         m_tile * NB, &full[pr], pol_x);
      if (++pr == PS) { pr = 0; ++round; }
    }
  } else if (warp == 3 && lane == 0) {
    // -------------------------------------------------- packed weight producer
    ptx::prefetch_tensormap(&qmap);
    const uint64_t pol_w = ptx::policy_evict_first();
    int s = 0;
    uint32_t ph = 0;
    for (int j = 0; j < nblk; ++j) {
      if (j >= kPStages && !ptx::mbar_wait(&pempty[s], ph ^ 1u, limit)) {
        ptx::record_wait_failure(p.error, 22u);
        limit = 1;
      }
      ptx::mbar_arrive_expect_tx(&pfull[s], kPBytes);
      ptx::tma_load_2d(ps + s * kPBytes, &qmap, (b0 + j) * (kBlock / 4), n_tile * kRows, &pfull[s], pol_w);
      if (++s == kPStages) { s = 0; ph ^= 1u; }
    }
  } else if (warp == 1 && lane == 0) {
    // -------------------------------------------------- MMA issuer
    const uint32_t idesc = (1u << 4)                        // D: f32
                           | ((uint32_t)(NB >> 3) << 17)     // N
                           | ((uint32_t)(kRows >> 4) << 24); // M = 128; A, B: f16, K-major
    const uint32_t xs_u = ptx::smem_u32(xs);
    int pr = 0;
    uint32_t ph = 0;
    for (int k = 0; k < ngroups; ++k) {
      if (!ptx::mbar_wait(&full[pr], ph, limit)) {
        ptx::record_wait_failure(p.error, 23u);
        limit = 1;
      }
      ptx::tc_fence_after();
#pragma unroll
      for (int u = 0; u < G; ++u) {
        const int s = G * pr + u;
        const uint64_t bdesc = ptx::sw128_kmajor_desc(xs_u + (uint32_t)s * XB);
        const uint32_t a_tm = tmem + (uint32_t)(kAColBase + s * kACols);
#pragma unroll
        for (int kk = 0; kk < BK / 16; ++kk)
          ptx::umma_f16_ts(tmem, a_tm + (uint32_t)(8 * kk), bdesc + (uint64_t)(2 * kk), idesc,
                           (k > 0 || u > 0 || kk > 0) ? 1u : 0u);
      }
      ptx::umma_commit(&empty[pr]);
      if (++pr == PS) { pr = 0; ph ^= 1u; }
    }
    ptx::umma_commit(accf);
  } else if (warp >= kFirstDec) {
    // -------------------------------------------------- decoders
    const bool nvalid = n < p.N;
    const __half* drow = dsc + (size_t)(nvalid ? n : 0) * p.B + b0;
    const uint32_t ps_u = ptx::smem_u32(ps);
    // this thread's 8 bytes of K step t: 16-byte granule t of row r, 64-byte swizzle, half h
    const uint32_t row_off = (uint32_t)(r * 64 + 8 * h);
    const uint32_t swz = (uint32_t)((r >> 1) & 3);
    __half dnext = nvalid ? __ldg(drow) : __float2half(0.f);
    int pr = 0, round = 0, pst = 0;
    uint32_t pph = 0;
    for (int j = 0; j < nblk; ++j) {
      const __half2 dd = __halves2half2(dnext, dnext);
      if (j + 1 < nblk) dnext = nvalid ? __ldg(drow + j + 1) : __float2half(0.f);
      if (!ptx::mbar_wait(&pfull[pst], pph, limit)) {
        ptx::record_wait_failure(p.error, 24u);
        limit = 1;
      }
      uint2 wv[kStepsPerBlock];
      const uint32_t pbase = ps_u + (uint32_t)(pst * kPBytes) + row_off;
#pragma unroll
      for (int t = 0; t < kStepsPerBlock; ++t) wv[t] = ptx::lds64(pbase + ((((uint32_t)t) ^ swz) << 4));
      __syncwarp();
      if (lane == 0) ptx::mbar_arrive(&pempty[pst]);
      if (++pst == kPStages) { pst = 0; pph ^= 1u; }
#pragma unroll
      for (int t2 = 0; t2 < kStepsPerBlock / G; ++t2) {
        if (round > 0 && !ptx::mbar_wait(&empty[pr], (uint32_t)((round - 1) & 1), limit)) {
          ptx::record_wait_failure(p.error, 25u);
          limit = 1;
        }
        ptx::tc_fence_after();
        __syncwarp();                    // tcgen05.st below is warp-collective
#pragma unroll
        for (int u = 0; u < G; ++u) {
          const uint2 w2 = wv[G * t2 + u];
          uint32_t a[16];
#pragma unroll
          for (int b = 0; b < 8; ++b) {
            const uint32_t w = b < 4 ? w2.x : w2.y;
            const uint32_t sel = (uint32_t)(b & 3) * 0x0101u + 0x4040u;   // byte b into both halves
            const uint32_t spread = __byte_perm(w, 0u, sel);
            a[2 * b] = pair_of<0>(spread, dd);
            a[2 * b + 1] = pair_of<1>(spread, dd);
          }
          ptx::tmem_st_32x32b_x16(lane_base + (uint32_t)(kAColBase + (G * pr + u) * kACols + 16 * h), a);
        }
        ptx::tmem_st_wait();
        ptx::tc_fence_before();
        __syncwarp();
        if (lane == 0) ptx::mbar_arrive(&full[pr]);
        if (++pr == PS) { pr = 0; ++round; }
      }
    }
    if (!ptx::mbar_wait(accf, 0, limit)) ptx::record_wait_failure(p.error, 26u);
    ptx::tc_fence_after();
    __syncwarp();
  }

  // ---------------------------------------------------------------- epilogue
  const int nch = (NB + 31) / 32;                      // 32-column accumulator chunks
  const bool dec = warp >= kFirstDec;
  const int mtile0 = m_tile * NB;
  if (p.splits > 1) {
    // Split K: chunk c of the accumulator belongs to rank c % sp.  Each CTA
    // writes the chunks it does not own to an L2-resident scratch (a warp
    // store covers 512 contiguous bytes), the cluster synchronises once, and
    // each owner adds the slices in rank order.
    const int sp = p.splits;
    const int mo = max_out_chunks(nch, sp);
    const size_t tile = (size_t)m_tile * gridDim.x + n_tile;
    if (dec) {
      float4* mine = p.scratch + (tile * sp + split) * mo * kChunkF4 + r;
      for (int c = h; c < nch; c += 2) {
        if (c % sp == split) continue;
        uint32_t v[32];
        ptx::tmem_ld_32x32b_x32(lane_base + (uint32_t)(32 * c), v);
        ptx::tmem_ld_wait();
        float4* dst = mine + (size_t)(c - owned_below(c, split, sp)) * kChunkF4;
#pragma unroll
        for (int g = 0; g < 8; ++g)
          dst[g * kRows] = make_float4(__uint_as_float(v[4 * g]), __uint_as_float(v[4 * g + 1]),
                                       __uint_as_float(v[4 * g + 2]), __uint_as_float(v[4 * g + 3]));
      }
    }
    ptx::cluster_sync();               // release / acquire at cluster scope orders the slices
    __syncwarp();
    if (dec) {                         // warp-uniform: tcgen05.ld is warp-collective
      const int nown = split < nch ? (nch - 1 - split) / sp + 1 : 0;
      for (int lc = h; lc < nown; lc += 2) {
        const int c = lc * sp + split;
        uint32_t v[32];
        ptx::tmem_ld_32x32b_x32(lane_base + (uint32_t)(32 * c), v);
        ptx::tmem_ld_wait();
        float acc[32];
#pragma unroll
        for (int e = 0; e < 32; ++e) acc[e] = 0.f;
        for (int src = 0; src < sp; ++src) {
          if (src == split) {
#pragma unroll
            for (int e = 0; e < 32; ++e) acc[e] += __uint_as_float(v[e]);
            continue;
          }
          const float4* srcp = p.scratch + ((tile * sp + src) * mo + (c - owned_below(c, src, sp))) * kChunkF4 + r;
#pragma unroll
          for (int g = 0; g < 8; ++g) {
            const float4 f = __ldcg(srcp + g * kRows);
            acc[4 * g] += f.x;
            acc[4 * g + 1] += f.y;
            acc[4 * g + 2] += f.z;
            acc[4 * g + 3] += f.w;
          }
        }
#pragma unroll
        for (int e = 0; e < 32; ++e) v[e] = __float_as_uint(acc[e]);
        const int lim = min(min(32, NB - 32 * c), p.M - (mtile0 + 32 * c));
        if (n < p.N) store_y(Y, v, n, mtile0 + 32 * c, lim, p.N);
      }
    }
  } else if (dec) {
    for (int c = h; c < nch; c += 2) {
      uint32_t v[32];
      ptx::tmem_ld_32x32b_x32(lane_base + (uint32_t)(32 * c), v);
      ptx::tmem_ld_wait();
      const int lim = min(min(32, NB - 32 * c), p.M - (mtile0 + 32 * c));
      if (n < p.N) store_y(Y, v, n, mtile0 + 32 * c, lim, p.N);
    }
  }
  ptx::tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    ptx::tc_fence_after();
    ptx::tmem_dealloc(tmem, 512);
  }
}

// ---------------------------------------------------------------- host side
struct Plan {
  int NB, S, tiles_n, tiles_m, splits;
  size_t smem, scratch;
};

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

constexpr int kMaxSmem = 232448;                  // 227 KB: the opt-in limit per block

// Raise the kernel's dynamic shared memory limit to the maximum once per device.
cudaError_t ensure_smem_attr() {
  static bool done[16] = {};
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev >= 0 && dev < 16 && done[dev]) return cudaSuccess;
  e = cudaFuncSetAttribute(gemm_tc_kernel<2>, cudaFuncAttributeMaxDynamicSharedMemorySize, kMaxSmem);
  if (e == cudaSuccess)
    e = cudaFuncSetAttribute(gemm_tc_kernel<4>, cudaFuncAttributeMaxDynamicSharedMemorySize, kMaxSmem);
  if (e == cudaSuccess && dev >= 0 && dev < 16) done[dev] = true;
  return e;
}

// CTAs that can run at once in clusters of `sp` (one CTA per SM), per device.
int cluster_slots(int sp, int num_sms) {
  static int cache[16][5] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 16) return (num_sms / sp) * sp;
  int& slot = cache[dev][sp];
  if (slot) return slot;
  int clusters = 0;
  if (ensure_smem_attr() == cudaSuccess) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(1, 1, (unsigned)sp);
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = kMinSmem;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 1;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = (unsigned)sp;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    if (cudaOccupancyMaxActiveClusters(&clusters, gemm_tc_kernel<2>, &cfg) != cudaSuccess) clusters = 0;
  }
  cudaGetLastError();
  slot = clusters > 0 ? clusters * sp : (num_sms / sp) * sp;
  return slot;
}

Plan plan_for(int64_t M, int64_t N, int64_t K, int num_sms) {
  Plan pl;
  pl.tiles_m = (int)ceil_div(M, 256);
  const int64_t per = ceil_div(M, pl.tiles_m);
  pl.NB = (int)(ceil_div(per, 16) * 16);
  const int XB = pl.NB * 128;
  int S = kRingBudget / XB;
  if (S > kMaxStages) S = kMaxStages;
  pl.S = S & ~1;
  pl.tiles_n = (int)ceil_div(N, kRows);
  const int64_t tiles = (int64_t)pl.tiles_n * pl.tiles_m;
  const int64_t B = K / kBlock;
  const int nch = (pl.NB + 31) / 32;
  // estimated time in K-step units: waves x (steps per CTA + fixed cost)
  double best = 0;
  pl.splits = 1;
  for (int sp = 1; sp <= 4; ++sp) {
    if (sp > B) break;
    const int64_t slots = sp == 1 ? num_sms : cluster_slots(sp, num_sms);
    const int64_t waves = ceil_div(tiles * sp, slots);
    const double t = (double)waves * ((double)ceil_div(B, sp) * kStepsPerBlock + (sp == 1 ? 6.0 : 9.0));
    if (sp == 1 || t < best) {
      best = t;
      pl.splits = sp;
    }
  }
  pl.smem = smem_bytes(pl.NB, pl.S);
  pl.scratch = pl.splits > 1 ? (size_t)tiles * pl.splits * max_out_chunks(nch, pl.splits) * kChunkF4 * 16 : 0;
  return pl;
}

}  // namespace

bool gemm_tc_supported(int fmt, int64_t M, int64_t N, int64_t K) {
  return fmt == TRI_TQ2 && M >= 17 && N >= 1 && K >= kBlock && K % kBlock == 0 &&
         ceil_div(M, 256) <= 65535;
}

size_t gemm_tc_ws_bytes(int fmt, int64_t M, int64_t N, int64_t K, int num_sms) {
  if (!gemm_tc_supported(fmt, M, N, K)) return 0;
  return plan_for(M, N, K, num_sms).scratch;
}

cudaError_t launch_gemm_tc(int fmt, const __half* X, const uint8_t* qs, const __half* d, __half* Y,
                           int M, int N, int K, void* ws, int num_sms, cudaStream_t s) {
  if (!gemm_tc_supported(fmt, M, N, K)) return cudaErrorNotSupported;
  const Plan pl = plan_for(M, N, K, num_sms);
  auto enc = encode_fn();
  if (!enc) return cudaErrorNotSupported;
  CUtensorMap xmap, qmap;
  {
    const cuuint64_t gdim[2] = {(cuuint64_t)K, (cuuint64_t)M};
    const cuuint64_t gstr[1] = {(cuuint64_t)K * 2};
    const cuuint32_t box[2] = {BK, (cuuint32_t)pl.NB};
    const cuuint32_t es[2] = {1, 1};
    if (enc(&xmap, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, const_cast<__half*>(X), gdim, gstr, box, es,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return cudaErrorInvalidValue;
  }
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
  TcParams p;
  const cudaError_t ew = wait_status_word(&p.error);
  if (ew != cudaSuccess) return ew;
  p.scratch = static_cast<float4*>(ws);
  p.M = M; p.N = N; p.K = K; p.B = K / kBlock;
  p.NB = pl.NB; p.S = pl.S; p.splits = pl.splits;
  if (pl.smem > (size_t)kMaxSmem) return cudaErrorInvalidValue;
  const cudaError_t e = ensure_smem_attr();
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)pl.tiles_n, (unsigned)pl.tiles_m, (unsigned)pl.splits);
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
  // small activation tiles make each MMA short: move K in groups of four
  // steps per barrier phase to amortise the issuing thread's waits
  if (pl.NB <= 128 && pl.S % 4 == 0) return cudaLaunchKernelEx(&cfg, gemm_tc_kernel<4>, xmap, qmap, d, Y, p);
  return cudaLaunchKernelEx(&cfg, gemm_tc_kernel<2>, xmap, qmap, d, Y, p);
}

}  // namespace tri
