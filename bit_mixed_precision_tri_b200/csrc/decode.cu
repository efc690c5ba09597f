// The non-linear steps of one transformer-block decode step around the
// ternary linear layers ("Scaling Laws and Efficient Inference for Ternary
// Language Models", section "The model": LLaMA-style blocks with SwiGLU,
// rotary embeddings with theta = 5e5, RMSNorm and QK-Norm, no biases;
// "Spectra: ...", section "Architecture of TriLM and FloatLM": activations
// stay in 16-bit floats).  All activations are fp16 in HBM; arithmetic is
// fp32; every kernel rounds once, where it stores.
//
//  * rmsnorm_kernel: y = x / sqrt(mean(x^2) + eps) * g per row, optionally
//    after the residual sum h = x + r (fp16 add: the exact sum rounded once),
//    which it stores too.  One CTA per row.
//  * rope_table_kernel: (cos, sin) of p * theta^(-2i/dh) for every position p
//    and pair i, angles in float64, stored as float32 pairs.
//  * qknorm_rope_kernel: one warp per (token, head) of the fused QKV product:
//    query and key heads are RMS-normalised over their 128 features (gains
//    gq / gk) and rotated ("rotate half": pairs (i, i + 64)); the key and
//    the value go into the caches at the token's position.  Lane l holds
//    features 2l, 2l + 1, 64 + 2l, 65 + 2l: both members of its two pairs.
//  * attn_decode_kernel: grouped-query attention of each sequence's new
//    token over its cached positions 0..pos, split over positions.  A CTA
//    (4 warps) owns (split, key/value head, sequence); 64-position tiles of
//    K and V are double-buffered in shared memory with cp.async (rows padded
//    to 272 bytes: conflict-free fragment reads), and each warp takes 16
//    positions of every tile: Q K^T and P V on the tensor cores
//    (mma.sync m16n8k16, fp32 accumulation; the group's query heads are the
//    A rows), the running softmax in fp32.  attn_combine_kernel merges the
//    (max, sum, output) triples of every split and warp.
#include "tri_internal.cuh"

namespace tri {
namespace {

constexpr int kDh = 128;            // head dimension served
constexpr int kTP = 64;             // positions per attention tile
constexpr int kRowB = 272;          // shared-memory row stride of K / V tiles, bytes
constexpr int kAttnWarps = 8;       // query heads per key/value head served: up to 8

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xFFFFFFFFu, v, o);
  return v;
}
__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xFFFFFFFFu, v, o));
  return v;
}

// ---------------------------------------------------------------- RMSNorm
__global__ void __launch_bounds__(256)
rmsnorm_kernel(const __half* __restrict__ x, const __half* __restrict__ r, const __half* __restrict__ g,
               __half* __restrict__ h_out, __half* __restrict__ y, int D, float eps) {
  __shared__ float red[8];
  const size_t row = (size_t)blockIdx.x * D;
  const uint4* x8 = reinterpret_cast<const uint4*>(x + row);
  const uint4* r8 = r ? reinterpret_cast<const uint4*>(r + row) : nullptr;
  uint4* h8 = h_out ? reinterpret_cast<uint4*>(h_out + row) : nullptr;
  const int n8 = D / 8;
  float ss = 0.f;
  for (int i = threadIdx.x; i < n8; i += blockDim.x) {
    uint4 v = x8[i];
    if (r8) {
      const uint4 w = r8[i];
      __half2* a = reinterpret_cast<__half2*>(&v);
      const __half2* b = reinterpret_cast<const __half2*>(&w);
#pragma unroll
      for (int k = 0; k < 4; ++k) a[k] = __hadd2(a[k], b[k]);   // exact sum, rounded once
      h8[i] = v;
    }
    const __half2* a = reinterpret_cast<const __half2*>(&v);
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const float2 f = __half22float2(a[k]);
      ss = fmaf(f.x, f.x, fmaf(f.y, f.y, ss));
    }
  }
  ss = warp_sum(ss);
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = ss;
  __syncthreads();
  if (threadIdx.x < 32) {
    float t = threadIdx.x < (blockDim.x >> 5) ? red[threadIdx.x] : 0.f;
    t = warp_sum(t);
    if (threadIdx.x == 0) red[0] = t;
  }
  __syncthreads();
  const float rstd = 1.f / sqrtf(red[0] / (float)D + eps);
  const uint4* g8 = reinterpret_cast<const uint4*>(g);
  uint4* y8 = reinterpret_cast<uint4*>(y + row);
  for (int i = threadIdx.x; i < n8; i += blockDim.x) {
    const uint4 v = h8 ? h8[i] : x8[i];      // h: written above by this thread
    const uint4 gv = g8[i];
    const __half2* a = reinterpret_cast<const __half2*>(&v);
    const __half2* b = reinterpret_cast<const __half2*>(&gv);
    uint4 o;
    __half2* c = reinterpret_cast<__half2*>(&o);
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const float2 f = __half22float2(a[k]), w = __half22float2(b[k]);
      c[k] = __floats2half2_rn(f.x * rstd * w.x, f.y * rstd * w.y);
    }
    y8[i] = o;
  }
}

// ---------------------------------------------------------------- RoPE table
__global__ void rope_table_kernel(float2* __restrict__ cs, int Lmax, int half_dh, double theta) {
  const int64_t idx = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (idx >= (int64_t)Lmax * half_dh) return;
  const int p = (int)(idx / half_dh), i = (int)(idx % half_dh);
  const double inv = pow(theta, -2.0 * (double)i / (double)(2 * half_dh));
  double s, c;
  sincos((double)p * inv, &s, &c);
  cs[idx] = make_float2((float)c, (float)s);
}

// ---------------------------------------------------------------- QK-Norm + RoPE + cache append
__global__ void __launch_bounds__(256)
qknorm_rope_kernel(const __half* __restrict__ qkv, const int* __restrict__ pos, const __half* __restrict__ gq,
                   const __half* __restrict__ gk, const float2* __restrict__ cs, __half* __restrict__ q_out,
                   __half* __restrict__ kc, __half* __restrict__ vc, int M, int H, int Hkv, int Lmax, float eps) {
  const int lane = threadIdx.x & 31;
  const int nh = H + 2 * Hkv;
  const int64_t wid = (int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  if (wid >= (int64_t)M * nh) return;
  const int m = (int)(wid / nh), j = (int)(wid % nh);
  const __half* src = qkv + ((size_t)m * nh + j) * kDh;
  const __half2 a = *reinterpret_cast<const __half2*>(src + 2 * lane);
  const __half2 b = *reinterpret_cast<const __half2*>(src + 64 + 2 * lane);
  const int p = pos[m];
  const bool in_range = p >= 0 && p < Lmax;            // else: nothing is cached, q unspecified
  if (j >= H + Hkv) {                                  // value head: into the cache as is
    if (in_range) {
      __half* dst = vc + (((size_t)m * Hkv + (j - H - Hkv)) * Lmax + p) * kDh;
      *reinterpret_cast<__half2*>(dst + 2 * lane) = a;
      *reinterpret_cast<__half2*>(dst + 64 + 2 * lane) = b;
    }
    return;
  }
  const float2 fa = __half22float2(a), fb = __half22float2(b);
  const float ss = warp_sum(fa.x * fa.x + fa.y * fa.y + fb.x * fb.x + fb.y * fb.y);
  const float rstd = 1.f / sqrtf(ss / (float)kDh + eps);
  const __half* g = j < H ? gq : gk;
  const float2 ga = __half22float2(*reinterpret_cast<const __half2*>(g + 2 * lane));
  const float2 gb = __half22float2(*reinterpret_cast<const __half2*>(g + 64 + 2 * lane));
  const float x0 = fa.x * rstd * ga.x, x1 = fa.y * rstd * ga.y;    // features 2l, 2l + 1
  const float y0 = fb.x * rstd * gb.x, y1 = fb.y * rstd * gb.y;    // features 64 + 2l, 65 + 2l
  const int pc = in_range ? p : 0;
  const float2 c0 = cs[(size_t)pc * 64 + 2 * lane], c1 = cs[(size_t)pc * 64 + 2 * lane + 1];
  const __half2 oa = __floats2half2_rn(x0 * c0.x - y0 * c0.y, x1 * c1.x - y1 * c1.y);
  const __half2 ob = __floats2half2_rn(y0 * c0.x + x0 * c0.y, y1 * c1.x + x1 * c1.y);
  __half* dst;
  if (j < H) {
    dst = q_out + ((size_t)m * H + j) * kDh;
  } else {
    if (!in_range) return;
    dst = kc + (((size_t)m * Hkv + (j - H)) * Lmax + p) * kDh;
  }
  *reinterpret_cast<__half2*>(dst + 2 * lane) = oa;
  *reinterpret_cast<__half2*>(dst + 64 + 2 * lane) = ob;
}

// ---------------------------------------------------------------- attention
__device__ __forceinline__ void cp16(uint32_t dst, const void* src, uint32_t n) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src), "r"(n) : "memory");
}
__device__ __forceinline__ uint32_t s_addr(const void* p) {
  return (uint32_t)__cvta_generic_to_shared(p);
}

constexpr int kTileBytes = kTP * kRowB;                                    // one K or V tile
constexpr int kAttnThreads = 128;                                          // 4 warps x 16 positions
constexpr int kAttnParts = kAttnThreads / 32;                              // partial results per split
constexpr int kAttnSmem = 2 * 2 * kTileBytes + kAttnWarps * kDh * 2;
static_assert(kTP == 16 * kAttnParts, "one 16-position slice per warp");
static_assert(kTP * 16 % kAttnThreads == 0, "whole copies per thread");

__device__ __forceinline__ void mma_f16(float (&c)[4], uint32_t a0, uint32_t a2, uint32_t b0, uint32_t b1) {
  // rows 8..15 of A are zero (at most 8 query heads per group)
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a0), "r"(0u), "r"(a2), "r"(0u), "r"(b0), "r"(b1));
}
__device__ __forceinline__ void ldsm_x4_trans(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2,
                                              uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3) : "r"(addr) : "memory");
}
__device__ __forceinline__ uint32_t lds_u32(uint32_t addr) {
  uint32_t v;
  asm volatile("ld.shared.u32 %0, [%1];" : "=r"(v) : "r"(addr) : "memory");
  return v;
}
__device__ __forceinline__ uint32_t pack_half2(float lo, float hi) {
  const __half2 h = __floats2half2_rn(lo, hi);
  return *reinterpret_cast<const uint32_t*>(&h);
}

// grid (splits, Hkv, M), 4 warps.  The group's G <= 8 query heads are the
// rows of the MMAs' A operand (rows 8..15 zero).  Warp w takes positions
// 16w .. 16w + 15 of every 64-position tile: S = Q K^T over them (two n8
// tiles, eight k16 steps, the B fragments read straight from the K tile:
// lane (gid, tig) reads position gid, features 2 tig, 2 tig + 1 (+8), which
// hit 32 distinct banks with 272-byte rows), the running softmax per head
// row (the four lanes of a quad hold a row), then O += P V with P taken from
// the S accumulators as the A operand and V's B fragments by ldmatrix.trans.
// Each warp leaves its own (max, sum, output) partial.
__global__ void __launch_bounds__(kAttnThreads)
attn_decode_kernel(const __half* __restrict__ q, const __half* __restrict__ kc, const __half* __restrict__ vc,
                   const int* __restrict__ pos, float* __restrict__ part_o, float2* __restrict__ part_ml,
                   int H, int Hkv, int Lmax, int max_len, int tiles_per_split) {
  extern __shared__ __align__(16) uint8_t sm[];
  uint8_t* qsm = sm + 4 * kTileBytes;                                    // [G][128] fp16
  const int s = blockIdx.x, kvh = blockIdx.y, m = blockIdx.z, splits = gridDim.x;
  const int G = H / Hkv;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, gid = lane >> 2, tig = lane & 3;
  int L = pos[m] + 1;                                  // clamped to [1, max_len] (max_len <= Lmax)
  L = L < 1 ? 1 : (L > max_len ? max_len : L);
  const int t0 = s * tiles_per_split * kTP;
  const int t1 = min(L, t0 + tiles_per_split * kTP);
  const int ntiles = t1 > t0 ? (t1 - t0 + kTP - 1) / kTP : 0;
  for (int i = threadIdx.x; i < G * 16; i += kAttnThreads)
    reinterpret_cast<uint4*>(qsm)[i] =
        reinterpret_cast<const uint4*>(q + ((size_t)m * H + (size_t)kvh * G) * kDh)[i];
  const __half* kb = kc + ((size_t)m * Hkv + kvh) * Lmax * kDh;
  const __half* vb = vc + ((size_t)m * Hkv + kvh) * Lmax * kDh;
  // tile `it` into buffer it & 1: 64 rows x 16 chunks of K and of V, i.e.
  // 1024 chunks each, 8 + 8 copies per thread (rows 0..63, chunks 0..15)
  auto issue = [&](int it) {
    const int base = t0 + it * kTP;
    uint8_t* kt = sm + (it & 1) * 2 * kTileBytes;
#pragma unroll
    for (int c = 0; c < kTP * 16 / kAttnThreads; ++c) {
      const int idx = c * kAttnThreads + threadIdx.x, row = idx >> 4, col = idx & 15;
      const bool ok = base + row < t1;
      const size_t off = (size_t)(ok ? base + row : 0) * kDh + col * 8;
      cp16(s_addr(kt + row * kRowB + col * 16), kb + off, ok ? 16u : 0u);
      cp16(s_addr(kt + kTileBytes + row * kRowB + col * 16), vb + off, ok ? 16u : 0u);
    }
    asm volatile("cp.async.commit_group;" ::: "memory");
  };
  if (ntiles > 0) issue(0);
  __syncthreads();                                     // q staged
  // A fragments of Q: row gid (a query head, zero past G), k step kk:
  // features 16 kk + 2 tig, +1 (a0) and 16 kk + 8 + 2 tig, +1 (a2)
  uint32_t qa[8][2];
  {
    const uint32_t qrow = s_addr(qsm) + (uint32_t)gid * kDh * 2 + 4 * tig;
#pragma unroll
    for (int kk = 0; kk < 8; ++kk) {
      qa[kk][0] = gid < G ? lds_u32(qrow + 32 * kk) : 0u;
      qa[kk][1] = gid < G ? lds_u32(qrow + 32 * kk + 16) : 0u;
    }
  }
  const float scale = rsqrtf((float)kDh);
  float mrun = -INFINITY, lrun = 0.f;
  float o[16][4];
#pragma unroll
  for (int nf = 0; nf < 16; ++nf) o[nf][0] = o[nf][1] = o[nf][2] = o[nf][3] = 0.f;
  for (int it = 0; it < ntiles; ++it) {
    if (it + 1 < ntiles) {
      issue(it + 1);
      asm volatile("cp.async.wait_group 1;" ::: "memory");
    } else {
      asm volatile("cp.async.wait_group 0;" ::: "memory");
    }
    __syncthreads();
    const uint32_t kt = s_addr(sm + (it & 1) * 2 * kTileBytes) + 16 * warp * kRowB;   // this warp's 16 rows
    const uint32_t vt = kt + kTileBytes;
    const int p0 = t0 + it * kTP + 16 * warp;          // position of the warp's first row
    // S = Q K^T: n tile nt = positions p0 + 8 nt .. + 7
    float sacc[2][4];
#pragma unroll
    for (int nt = 0; nt < 2; ++nt) {
      sacc[nt][0] = sacc[nt][1] = sacc[nt][2] = sacc[nt][3] = 0.f;
      const uint32_t krow = kt + (uint32_t)(8 * nt + gid) * kRowB + 4 * tig;
#pragma unroll
      for (int kk = 0; kk < 8; ++kk)
        mma_f16(sacc[nt], qa[kk][0], qa[kk][1], lds_u32(krow + 32 * kk), lds_u32(krow + 32 * kk + 16));
    }
    // row gid's scores at positions p0 + 8 nt + 2 tig + e
    float sc[2][2];
    float mt = -INFINITY;
#pragma unroll
    for (int nt = 0; nt < 2; ++nt)
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        sc[nt][e] = p0 + 8 * nt + 2 * tig + e < t1 ? sacc[nt][e] * scale : -INFINITY;
        mt = fmaxf(mt, sc[nt][e]);
      }
    mt = fmaxf(mt, __shfl_xor_sync(0xFFFFFFFFu, mt, 1));
    mt = fmaxf(mt, __shfl_xor_sync(0xFFFFFFFFu, mt, 2));
    const float mnew = fmaxf(mrun, mt);
    // no valid position seen yet (a slice past the end): nothing changes
    const float alpha = mnew == -INFINITY ? 1.f : expf(mrun - mnew);
    float pr[2][2], ps = 0.f;
#pragma unroll
    for (int nt = 0; nt < 2; ++nt)
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        pr[nt][e] = mnew == -INFINITY ? 0.f : expf(sc[nt][e] - mnew);
        ps += pr[nt][e];
      }
    ps += __shfl_xor_sync(0xFFFFFFFFu, ps, 1);
    ps += __shfl_xor_sync(0xFFFFFFFFu, ps, 2);
    lrun = lrun * alpha + ps;
    mrun = mnew;
    // O = alpha O + P V: A = P (row gid, k = positions 2 tig, +1 and 8 + 2 tig, +1)
    // as two fp16 parts, P = hi + lo (lo = the rounding error of hi, itself
    // rounded): the products keep ~22 bits of P, so the fp32 accumulation,
    // not an fp16 rounding of the weights, bounds the error
    const uint32_t pa0 = pack_half2(pr[0][0], pr[0][1]), pa2 = pack_half2(pr[1][0], pr[1][1]);
    const float2 h0 = __half22float2(*reinterpret_cast<const __half2*>(&pa0));
    const float2 h2 = __half22float2(*reinterpret_cast<const __half2*>(&pa2));
    const uint32_t pl0 = pack_half2(pr[0][0] - h0.x, pr[0][1] - h0.y);
    const uint32_t pl2 = pack_half2(pr[1][0] - h2.x, pr[1][1] - h2.y);
    // ldmatrix.trans: lane l addresses row (l & 7) + 8 ((l >> 3) & 1) of the
    // slice at feature 8 (l >> 4) of the pair of n tiles
    const uint32_t vrow = vt + (uint32_t)((lane & 7) + 8 * ((lane >> 3) & 1)) * kRowB + 16 * (lane >> 4);
#pragma unroll
    for (int nf = 0; nf < 16; nf += 2) {
      uint32_t v0, v1, v2, v3;
      ldsm_x4_trans(vrow + 16 * nf, v0, v1, v2, v3);
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        o[nf][e] *= alpha;
        o[nf + 1][e] *= alpha;
      }
      mma_f16(o[nf], pa0, pa2, v0, v1);
      mma_f16(o[nf], pl0, pl2, v0, v1);
      mma_f16(o[nf + 1], pa0, pa2, v2, v3);
      mma_f16(o[nf + 1], pl0, pl2, v2, v3);
    }
    __syncthreads();                                   // the buffer may be refilled
  }
  if (gid < G) {
    const size_t slot = (((size_t)m * H + (size_t)kvh * G + gid) * splits + s) * kAttnParts + warp;
    float* dst = part_o + slot * kDh + 2 * tig;
#pragma unroll
    for (int nf = 0; nf < 16; ++nf) *reinterpret_cast<float2*>(dst + 8 * nf) = make_float2(o[nf][0], o[nf][1]);
    if (tig == 0) part_ml[slot] = make_float2(mrun, lrun);
  }
}

// One CTA of 128 threads per (sequence, query head) merges the `nparts`
// partials: the block reduces their maxima, each thread turns a strided share
// of them into weights exp(max_s - max) in shared memory (dynamic, nparts
// floats) and sums the weighted row sums; then thread d adds feature d over
// the partials (coalesced rows of 128 floats).
__device__ __forceinline__ float block_reduce_128(float v, float* red, bool is_max) {
  v = is_max ? warp_max(v) : warp_sum(v);
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = v;
  __syncthreads();
  const float r = is_max ? fmaxf(fmaxf(red[0], red[1]), fmaxf(red[2], red[3]))
                         : (red[0] + red[1]) + (red[2] + red[3]);
  __syncthreads();                                     // red may be reused
  return r;
}

__global__ void __launch_bounds__(128)
attn_combine_kernel(const float* __restrict__ part_o, const float2* __restrict__ part_ml, __half* __restrict__ out,
                    int nparts) {
  extern __shared__ float wsm[];                       // [nparts]
  __shared__ float red[4];
  const size_t mh = blockIdx.x;
  const int t = threadIdx.x;
  const float2* ml = part_ml + mh * nparts;
  float mx = -INFINITY;
  for (int s = t; s < nparts; s += 128)
    if (ml[s].y > 0.f) mx = fmaxf(mx, ml[s].x);
  mx = block_reduce_128(mx, red, true);
  float l = 0.f;
  for (int s = t; s < nparts; s += 128) {
    const float2 v = ml[s];
    const float w = v.y > 0.f ? expf(v.x - mx) : 0.f;
    wsm[s] = w;
    l = fmaf(w, v.y, l);
  }
  l = block_reduce_128(l, red, false);                 // its barriers also publish wsm
  const float* po = part_o + mh * nparts * kDh + t;
  float acc = 0.f;
#pragma unroll 4
  for (int s = 0; s < nparts; ++s) acc = fmaf(wsm[s], po[(size_t)s * kDh], acc);
  out[mh * kDh + t] = __float2half_rn(acc / l);
}

struct AttnPlan {
  int splits, tiles_per_split;
  size_t off_ml, total;
};

AttnPlan attn_plan(int64_t M, int64_t H, int64_t Hkv, int64_t max_len, int sms) {
  AttnPlan pl;
  const int64_t tiles = (max_len + kTP - 1) / kTP;
  int64_t sp = (2 * (int64_t)sms + M * Hkv - 1) / (M * Hkv);   // about two CTAs per SM
  if (sp > tiles) sp = tiles;
  if (sp < 1) sp = 1;
  pl.tiles_per_split = (int)((tiles + sp - 1) / sp);
  pl.splits = (int)((tiles + pl.tiles_per_split - 1) / pl.tiles_per_split);
  const size_t n = (size_t)M * H * pl.splits * kAttnParts;
  pl.off_ml = (n * kDh * 4 + 255) & ~size_t(255);
  pl.total = pl.off_ml + ((n * 8 + 255) & ~size_t(255));
  return pl;
}

}  // namespace

cudaError_t launch_rmsnorm(const __half* x, const __half* r, const __half* g, __half* h_out, __half* y,
                           int64_t M, int64_t D, float eps, cudaStream_t s) {
  rmsnorm_kernel<<<(unsigned)M, 256, 0, s>>>(x, r, g, h_out, y, (int)D, eps);
  return cudaGetLastError();
}

cudaError_t launch_rope_table(float2* cs, int64_t Lmax, int64_t dh, double theta, cudaStream_t s) {
  const int64_t n = Lmax * (dh / 2);
  rope_table_kernel<<<(unsigned)((n + 255) / 256), 256, 0, s>>>(cs, (int)Lmax, (int)(dh / 2), theta);
  return cudaGetLastError();
}

cudaError_t launch_qknorm_rope(const __half* qkv, const int* pos, const __half* gq, const __half* gk,
                               const float2* cs, __half* q_out, __half* kc, __half* vc, int64_t M, int64_t H,
                               int64_t Hkv, int64_t Lmax, float eps, cudaStream_t s) {
  const int64_t warps = M * (H + 2 * Hkv);
  qknorm_rope_kernel<<<(unsigned)((warps + 7) / 8), 256, 0, s>>>(qkv, pos, gq, gk, cs, q_out, kc, vc, (int)M,
                                                                  (int)H, (int)Hkv, (int)Lmax, eps);
  return cudaGetLastError();
}

size_t attention_decode_ws_bytes(int64_t M, int64_t H, int64_t Hkv, int64_t max_len, int sms) {
  return attn_plan(M, H, Hkv, max_len, sms).total;
}

cudaError_t launch_attention_decode(const __half* q, const __half* kc, const __half* vc, const int* pos,
                                    __half* out, int64_t M, int64_t H, int64_t Hkv, int64_t Lmax,
                                    int64_t max_len, void* ws, int sms, cudaStream_t s) {
  const AttnPlan pl = attn_plan(M, H, Hkv, max_len, sms);
  static bool attr_done[64] = {};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 0 || dev >= 64 || !attr_done[dev]) {
    const cudaError_t e = cudaFuncSetAttribute(attn_decode_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                               kAttnSmem);
    if (e != cudaSuccess) return e;
    if (dev >= 0 && dev < 64) attr_done[dev] = true;
  }
  float* part_o = static_cast<float*>(ws);
  float2* part_ml = reinterpret_cast<float2*>(static_cast<uint8_t*>(ws) + pl.off_ml);
  attn_decode_kernel<<<dim3((unsigned)pl.splits, (unsigned)Hkv, (unsigned)M), kAttnThreads, kAttnSmem, s>>>(
      q, kc, vc, pos, part_o, part_ml, (int)H, (int)Hkv, (int)Lmax, (int)max_len, pl.tiles_per_split);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  const int nparts = pl.splits * kAttnParts;           // at most ~2 x SMs x 4: a few KB of weights
  attn_combine_kernel<<<(unsigned)(M * H), kDh, (size_t)nparts * sizeof(float), s>>>(part_o, part_ml, out, nparts);
  return cudaGetLastError();
}

}  // namespace tri
