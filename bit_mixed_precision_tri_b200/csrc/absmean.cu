// Absmean scale and ternarization on sm_100a.
//
// "Scaling Laws and Efficient Inference for Ternary Language Models",
// section "The model", steps 1-2: gamma = eps + mean|W| over the whole matrix
// ("Spectra ...", section "Architecture of TriLM and FloatLM": one scale per
// matrix), then W_hat = round(clip(W / gamma, -1, 1)).
//
// Exactness.  A trit flips if gamma moves by one ulp near |W/gamma| = 0.5, so
// gamma must not depend on the reduction order.  Every finite float32 |w| is
// m * 2^(e-150) with a 24-bit integer m and e = max(biased exponent, 1); the
// kernel sums the integers m per exponent e into 64-bit bins (integer adds
// commute, so the bins are identical for every grid and every run), and a
// one-thread finalize expands sum_e bin[e] * 2^(e-1) into a 352-bit integer
// (units of 2^-149) and rounds it once to the nearest double.  Then
// mean = RN64(S / (N*K)) and gamma = RN32(RN64(mean + eps)).
//
// Traffic: the bins pass reads W once (4 B/weight); ternarize reads W again
// and writes one int8 per weight (5 B/weight).  Both are HBM-bound streams
// with warp-contiguous accesses.
#include "tri_internal.cuh"

namespace tri {
namespace {

constexpr int kBins = 256;
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

// Add |x| to the warp's exponent bins.  Lanes holding the same exponent are
// grouped with match.any, their 24-bit mantissas summed with redux.sync
// (< 2^29, exact in 32 bits), and one lane per group issues the atomic, so a
// warp step costs one shared atomic per distinct exponent instead of 32.
// All 32 lanes must call this together.
__device__ __forceinline__ void bin_add_warp(unsigned long long* wbins, float x, unsigned& bad) {
  const unsigned u = __float_as_uint(x) & 0x7FFFFFFFu;
  unsigned e = u >> 23;
  unsigned m = (u & 0x7FFFFFu) | (e ? 0x800000u : 0u);
  if (e == 255u) { bad = 1u; m = 0u; }
  if (e == 0u) e = 1u;
  const unsigned grp = __match_any_sync(0xFFFFFFFFu, e);
  const unsigned sum = __reduce_add_sync(grp, m);
  if ((threadIdx.x & 31) == (unsigned)(__ffs(grp) - 1) && sum != 0u)
    atomicAdd(&wbins[e], (unsigned long long)sum);
}

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
  // whole warps iterate together (the bins update is a warp collective)
  for (int64_t base = (int64_t)blockIdx.x * kThreads; base < n4; base += stride) {
    const int64_t i = base + threadIdx.x;
    float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
    if (i < n4) v = ld_stream_f4(W4 + i);
    bin_add_warp(wb, v.x, bad);
    bin_add_warp(wb, v.y, bad);
    bin_add_warp(wb, v.z, bad);
    bin_add_warp(wb, v.w, bad);
  }
  for (int64_t base = (n4 << 2) + (int64_t)blockIdx.x * kThreads; base < n; base += stride) {
    const int64_t i = base + threadIdx.x;
    bin_add_warp(wb, i < n ? W[i] : 0.f, bad);
  }
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

__global__ void absmean_finalize_kernel(AbsmeanWs* ws, int64_t n, float eps, float* gamma) {
  if (threadIdx.x != 0 || blockIdx.x != 0) return;
  if (ws->nonfinite) { *gamma = __int_as_float(0x7FC00000); return; }
  constexpr int NL = 12;  // 384 bits >= 253 + 64 + carries
  unsigned L[NL];
#pragma unroll
  for (int i = 0; i < NL; ++i) L[i] = 0u;
  for (int e = 1; e < 255; ++e) {
    const unsigned long long v = ws->bins[e];
    if (!v) continue;
    const int sh = e - 1;               // value = v * 2^(e-1) units of 2^-149
    const int li = sh >> 5, bi = sh & 31;
    // v << bi spans up to three limbs
    unsigned long long lo = v << bi;
    unsigned long long hi = bi ? (v >> (64 - bi)) : 0ull;
    unsigned parts[3] = {(unsigned)lo, (unsigned)(lo >> 32), (unsigned)hi};
    unsigned long long carry = 0ull;
    for (int j = 0; li + j < NL; ++j) {
      unsigned long long add = carry + (j < 3 ? parts[j] : 0u);
      if (add == 0ull && j >= 3) break;
      unsigned long long t = (unsigned long long)L[li + j] + add;
      L[li + j] = (unsigned)t;
      carry = t >> 32;
    }
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
  absmean_bins_kernel<<<grid_for(n >> 2), kThreads, 0, s>>>(W, n, w);
  absmean_finalize_kernel<<<1, 32, 0, s>>>(w, n, eps, gamma);
  return cudaGetLastError();
}

cudaError_t launch_ternarize(const float* W, int64_t n, const float* gamma, int8_t* trits,
                             cudaStream_t s) {
  ternarize_kernel<<<grid_for(n >> 4), kThreads, 0, s>>>(W, n, gamma, trits);   // one block per 4 x 256 float4
  return cudaGetLastError();
}

}  // namespace tri
