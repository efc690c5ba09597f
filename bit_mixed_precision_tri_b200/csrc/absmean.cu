// Absmean scale and ternarization on sm_100a.
//
// "Scaling Laws and Efficient Inference for Ternary Language Models",
// section "The model", steps 1-2: gamma = eps + mean|W| over the whole matrix
// ("Spectra ...", section "Architecture of TriLM and FloatLM": one scale per
// matrix), then W_hat = round(clip(W / gamma, -1, 1)).
//
// Exactness.  A trit flips if gamma moves by one ulp near |W/gamma| = 0.5, so
// gamma must not depend on the reduction order.  Every finite float32 |w| is
// m * 2^(e-150) with a 24-bit integer m and e = max(biased exponent, 1), i.e.
// m * 2^(e-1) in units of 2^-149.  All sums are of such integers (integer adds
// commute, so the result is identical for every grid and every run): a bin
// b holds integers worth 2^(b-1) units each, and a one-thread finalize
// expands sum_b bin[b] * 2^(b-1) into a 384-bit integer and rounds it once to
// the nearest double.  Then mean = RN64(S / (N*K)) and gamma =
// RN32(RN64(mean + eps)).
//
// The bins pass keeps, per lane, a window of 24 exponents [lo, lo + 23]
// placed below the largest exponent the lane has seen: the lane adds
// m << (e - lo) (< 2^47) into a 64-bit register, which is flushed as two
// 32-bit halves into the warp's shared bins lo and lo + 32 when the window
// moves up, every 2^16 values and at the end.  A value below the window (for
// real weights, below 2^-22 of the lane's largest magnitude: rare) is added
// to its own bin at once (one shared atomic).  No warp collective runs in the
// loop.
//
// Traffic: the bins pass reads W once (4 B/weight); ternarize reads W again
// and writes one int8 per weight (5 B/weight).  Both are HBM-bound streams
// with warp-contiguous accesses.
#include "tri_internal.cuh"

namespace tri {
namespace {

constexpr int kBins = 288;          // exponents 1..254, and flushed high halves up to 254 + 10
constexpr int kThreads = 256;
constexpr int kWarps = kThreads / 32;

struct AbsmeanWs {
  unsigned long long bins[kBins];
  unsigned int nonfinite;
  unsigned int pad[3];
};

__device__ __forceinline__ float4 ld_stream_f4(const float4* p) {
  float4 v;
  asm volatile("ld.global.nc.L1::no_allocate.v4.f32 {%0,%1,%2,%3}, [%4];"
               : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w) : "l"(p));
  return v;
}

// One lane's window accumulator: exponents lo .. lo + 23 (placed below the
// largest exponent the lane has seen), acc = sum of m << (e - lo) < 2^63
// (at most 2^16 values of < 2^47 between flushes).  A flush adds the two
// 32-bit halves to bins lo and lo + 32; a value below the window goes to its
// own bin at once (rare for real weights: below 2^-22 of the lane's largest).
struct LaneAcc {
  int lo = 0;                    // 0: no window yet
  int cnt = 0;                   // values added since the last flush
  unsigned long long acc = 0ull;

  __device__ __forceinline__ void flush(unsigned long long* wb) {
    if (acc) {
      atomicAdd(&wb[lo], acc & 0xFFFFFFFFull);
      if (acc >> 32) atomicAdd(&wb[lo + 32], acc >> 32);
    }
    acc = 0ull;
    cnt = 0;
  }

  template <int K>
  __device__ __forceinline__ void add(unsigned long long* wb, const float (&x)[K], unsigned& bad) {
    unsigned e[K], m[K];
    unsigned emax = 1u;
#pragma unroll
    for (int i = 0; i < K; ++i) {
      // e = max(biased exponent, 1); m = fraction plus the hidden bit
      // exactly when the biased exponent is not 0 (zero and denormals)
      const unsigned bits = __float_as_uint(x[i]);
      const unsigned er = (bits >> 23) & 0xFFu;
      e[i] = er > 1u ? er : 1u;
      m[i] = (bits & 0x7FFFFFu) + 0x800000u - ((e[i] - er) << 23);
      emax = e[i] > emax ? e[i] : emax;
    }
    if (emax == 255u) {          // Inf or NaN somewhere: gamma becomes NaN (rare)
      bad = 1u;
      emax = 1u;
#pragma unroll
      for (int i = 0; i < K; ++i) {
        if (e[i] == 255u) {
          m[i] = 0u;
          e[i] = 1u;
        }
        emax = e[i] > emax ? e[i] : emax;
      }
    }
    if (lo == 0 || (int)emax > lo + 23 || cnt > (1 << 16) - K) {
      flush(wb);
      lo = (int)emax - 22 > 1 ? (int)emax - 22 : 1;
    }
    cnt += K;
#pragma unroll
    for (int i = 0; i < K; ++i) {
      const int dsh = (int)e[i] - lo;
      if (dsh >= 0) acc += (unsigned long long)m[i] << dsh;
      else if (m[i]) atomicAdd(&wb[e[i]], (unsigned long long)m[i]);
    }
  }
};

__global__ void __launch_bounds__(kThreads)
absmean_bins_kernel(const float* __restrict__ W, int64_t n, AbsmeanWs* ws) {
  __shared__ unsigned long long sbins[kWarps][kBins];
  for (int i = threadIdx.x; i < kWarps * kBins; i += kThreads) (&sbins[0][0])[i] = 0ull;
  __syncthreads();
  unsigned long long* wb = sbins[threadIdx.x >> 5];
  unsigned bad = 0u;
  const int64_t n4 = n >> 2;
  const float4* W4 = reinterpret_cast<const float4*>(W);
  const int64_t stride = (int64_t)gridDim.x * kThreads;
  LaneAcc la;
  // Chunks of 4 x kThreads float4: every thread has four 16-byte loads in
  // flight, each warp-wide load one contiguous 512 bytes.
  // The next chunk's loads are issued before the current one is added up.
  const int64_t chunks = n4 / (4 * kThreads);
  float4 v[4];
  if ((int64_t)blockIdx.x < chunks) {
#pragma unroll
    for (int q = 0; q < 4; ++q) v[q] = ld_stream_f4(W4 + (int64_t)blockIdx.x * 4 * kThreads + threadIdx.x + q * kThreads);
  }
  for (int64_t c = blockIdx.x; c < chunks; c += gridDim.x) {
    const int64_t cn = c + gridDim.x;
    float4 w[4];
    if (cn < chunks) {
#pragma unroll
      for (int q = 0; q < 4; ++q) w[q] = ld_stream_f4(W4 + cn * 4 * kThreads + threadIdx.x + q * kThreads);
    }
    const float x[16] = {v[0].x, v[0].y, v[0].z, v[0].w, v[1].x, v[1].y, v[1].z, v[1].w,
                         v[2].x, v[2].y, v[2].z, v[2].w, v[3].x, v[3].y, v[3].z, v[3].w};
    la.add<16>(wb, x, bad);
#pragma unroll
    for (int q = 0; q < 4; ++q) v[q] = w[q];
  }
  for (int64_t i = chunks * 4 * kThreads + (int64_t)blockIdx.x * kThreads + threadIdx.x; i < n4; i += stride) {
    const float4 v = ld_stream_f4(W4 + i);
    const float x[4] = {v.x, v.y, v.z, v.w};
    la.add<4>(wb, x, bad);
  }
  for (int64_t i = (n4 << 2) + (int64_t)blockIdx.x * kThreads + threadIdx.x; i < n; i += stride) {
    const float x[1] = {W[i]};
    la.add<1>(wb, x, bad);
  }
  la.flush(wb);
  const int any_bad = __syncthreads_or((int)bad);
  for (int b = threadIdx.x; b < kBins; b += kThreads) {
    unsigned long long s = 0ull;
#pragma unroll
    for (int w = 0; w < kWarps; ++w) s += sbins[w][b];
    if (s) atomicAdd(&ws->bins[b], s);
  }
  if (threadIdx.x == 0 && any_bad) atomicOr(&ws->nonfinite, 1u);
}

// 64 bits of a little-endian multi-limb integer starting at bit `pos` (pos >= 0)
__device__ unsigned long long limb_window(const unsigned* L, int nl, int pos) {
  const int w = pos >> 5, off = pos & 31;
  unsigned long long lo = 0ull, mid = 0ull, hi = 0ull;
  if (w < nl) lo = L[w];
  if (w + 1 < nl) mid = L[w + 1];
  if (w + 2 < nl) hi = L[w + 2];
  const unsigned long long v = lo | (mid << 32);
  return off ? ((v >> off) | (hi << (64 - off))) : v;
}

// true if any bit below `pos` is set
__device__ bool limb_any_below(const unsigned* L, int pos) {
  const int w = pos >> 5, off = pos & 31;
  for (int i = 0; i < w; ++i)
    if (L[i]) return true;
  return off && (L[w] & ((1u << off) - 1u));
}

// Launched with one warp.  S = sum_b bin[b] 2^(b-1) (units of 2^-149) as a
// 384-bit integer in 32-bit limbs: bin b = 32 li + bi + 1 adds bin << bi at
// limb li.  Lane bi takes the bins 32 li + bi + 1 (li = 0..8) and adds the
// three 32-bit parts of each shifted value to its limb sums (static indices:
// registers); the lanes' limb sums are added over the warp in 64 bits
// (< 2^39), and lane 0 carries them once and rounds.
__global__ void absmean_finalize_kernel(AbsmeanWs* ws, int64_t n, float eps, float* gamma) {
  constexpr int NL = 12;  // 384 bits: bins up to 287 (2^286 units) times 64-bit values, plus carries
  const int lane = threadIdx.x & 31;
  unsigned long long part[NL];
#pragma unroll
  for (int i = 0; i < NL; ++i) part[i] = 0ull;
#pragma unroll
  for (int li = 0; li < 9; ++li) {
    const int b = 32 * li + lane + 1;
    const unsigned long long v = b < kBins ? ws->bins[b] : 0ull;
    const unsigned long long lo = v << lane;
    const unsigned long long hi = lane ? (v >> (64 - lane)) : 0ull;
    part[li] += lo & 0xFFFFFFFFull;
    part[li + 1] += lo >> 32;
    part[li + 2] += hi;
  }
#pragma unroll
  for (int i = 0; i < NL; ++i)
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) part[i] += __shfl_xor_sync(0xFFFFFFFFu, part[i], o);
  if (threadIdx.x != 0 || blockIdx.x != 0) return;
  if (ws->nonfinite) { *gamma = __int_as_float(0x7FC00000); return; }
  unsigned L[NL];
  unsigned long long carry = 0ull;
#pragma unroll
  for (int i = 0; i < NL; ++i) {
    const unsigned long long t = part[i] + carry;
    L[i] = (unsigned)t;
    carry = t >> 32;
  }
  int top = -1;
  for (int i = NL - 1; i >= 0 && top < 0; --i)
    if (L[i]) top = i * 32 + (31 - __clz(L[i]));
  double s64 = 0.0;
  if (top >= 0) {
    if (top <= 52) {
      s64 = ldexp((double)limb_window(L, NL, 0), -149);   // exact: fits in 53 bits
    } else {
      const int sh = top - 52;
      unsigned long long mant = limb_window(L, NL, sh) & ((1ull << 53) - 1ull);
      const bool rbit = (limb_window(L, NL, sh - 1) & 1ull) != 0ull;
      const bool sticky = limb_any_below(L, sh - 1);
      if (rbit && (sticky || (mant & 1ull))) ++mant;     // round half to even
      s64 = ldexp((double)mant, sh - 149);
    }
  }
  const double mean = __ddiv_rn(s64, (double)n);
  const double g = __dadd_rn(mean, (double)eps);
  *gamma = __double2float_rn(g);
}

__device__ __forceinline__ int8_t trit_of(float w, float g) {
  float x = __fdiv_rn(w, g);
  if (isnan(x)) return 0;
  x = fminf(fmaxf(x, -1.0f), 1.0f);
  return (int8_t)__float2int_rn(x);
}

// Each thread handles four float4 of a 4 x kThreads-float4 chunk, at
// stride kThreads, so every load and every 32-bit store of a warp is one
// contiguous 512-byte (or 128-byte) run: W is read exactly once.
__global__ void __launch_bounds__(kThreads)
ternarize_kernel(const float* __restrict__ W, int64_t n, const float* __restrict__ gamma,
                 int8_t* __restrict__ trits) {
  const float g = *gamma;
  const int64_t n4 = n >> 2;
  const int64_t chunks = n4 / (4 * kThreads);
  const float4* W4 = reinterpret_cast<const float4*>(W);
  unsigned* T4 = reinterpret_cast<unsigned*>(trits);
  for (int64_t c = blockIdx.x; c < chunks; c += gridDim.x) {
    const int64_t base = c * 4 * kThreads + threadIdx.x;
    float4 v[4];
#pragma unroll
    for (int q = 0; q < 4; ++q) v[q] = ld_stream_f4(W4 + base + q * kThreads);
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const unsigned b0 = (unsigned)(uint8_t)trit_of(v[q].x, g);
      const unsigned b1 = (unsigned)(uint8_t)trit_of(v[q].y, g);
      const unsigned b2 = (unsigned)(uint8_t)trit_of(v[q].z, g);
      const unsigned b3 = (unsigned)(uint8_t)trit_of(v[q].w, g);
      T4[base + q * kThreads] = b0 | (b1 << 8) | (b2 << 16) | (b3 << 24);
    }
  }
  // the float4 after the last whole chunk, then single elements
  for (int64_t i = chunks * 4 * kThreads + (int64_t)blockIdx.x * kThreads + threadIdx.x; i < n4;
       i += (int64_t)gridDim.x * kThreads) {
    const float4 v = ld_stream_f4(W4 + i);
    T4[i] = (unsigned)(uint8_t)trit_of(v.x, g) | ((unsigned)(uint8_t)trit_of(v.y, g) << 8) |
            ((unsigned)(uint8_t)trit_of(v.z, g) << 16) | ((unsigned)(uint8_t)trit_of(v.w, g) << 24);
  }
  for (int64_t i = (n4 << 2) + (int64_t)blockIdx.x * kThreads + threadIdx.x; i < n;
       i += (int64_t)gridDim.x * kThreads)
    trits[i] = trit_of(W[i], g);
}

int grid_for(int64_t work_items) {
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  int64_t g = ceil_div(work_items, kThreads);
  const int64_t cap = (int64_t)sms * 8;
  if (g > cap) g = cap;
  if (g < 1) g = 1;
  return (int)g;
}

}  // namespace

size_t absmean_ws_bytes() { return sizeof(AbsmeanWs); }

cudaError_t launch_absmean(const float* W, int64_t n, float eps, float* gamma, void* ws,
                           cudaStream_t s) {
  AbsmeanWs* w = static_cast<AbsmeanWs*>(ws);
  cudaError_t e = cudaMemsetAsync(w, 0, sizeof(AbsmeanWs), s);
  if (e != cudaSuccess) return e;
  absmean_bins_kernel<<<grid_for(n >> 4), kThreads, 0, s>>>(W, n, w);   // one block per 4 x 256 float4
  absmean_finalize_kernel<<<1, 32, 0, s>>>(w, n, eps, gamma);
  return cudaGetLastError();
}

cudaError_t launch_ternarize(const float* W, int64_t n, const float* gamma, int8_t* trits,
                             cudaStream_t s) {
  ternarize_kernel<<<grid_for(n >> 4), kThreads, 0, s>>>(W, n, gamma, trits);   // one block per 4 x 256 float4
  return cudaGetLastError();
}

}  // namespace tri
