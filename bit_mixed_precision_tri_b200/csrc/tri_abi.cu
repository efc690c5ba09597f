// The C ABI (include/tri.h): host-side validation and dispatch.
//
// Every entry point checks its arguments before enqueuing anything, launches
// on the caller's stream and never allocates; only tri_wait_status
// synchronizes (it exists to read a device-side result).
#include <mutex>

#include "tri_internal.cuh"

namespace {

using tri::ceil_div;

constexpr int64_t kMaxDim = (int64_t(1) << 31) - 1;

bool aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

struct DevInfo {
  int sms = 0;
  int major = 0;
  int minor = 0;
};

constexpr int kMaxDevices = 64;
DevInfo g_dev[kMaxDevices];
std::once_flag g_once[kMaxDevices];

tri_status device_info(DevInfo* out) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) {
    cudaGetLastError();
    return TRI_ERR_CUDA;
  }
  std::call_once(g_once[dev], [dev]() {
    cudaDeviceGetAttribute(&g_dev[dev].sms, cudaDevAttrMultiProcessorCount, dev);
    cudaDeviceGetAttribute(&g_dev[dev].major, cudaDevAttrComputeCapabilityMajor, dev);
    cudaDeviceGetAttribute(&g_dev[dev].minor, cudaDevAttrComputeCapabilityMinor, dev);
  });
  *out = g_dev[dev];
  if (out->major != 10 || out->minor != 0) return TRI_ERR_NO_DEVICE;
  return TRI_OK;
}

thread_local cudaError_t g_last_cuda = cudaSuccess;

tri_status from_cuda(cudaError_t e) {
  if (e == cudaSuccess) return TRI_OK;
  g_last_cuda = e;
  cudaGetLastError();
  return TRI_ERR_CUDA;
}

tri_status check_nk(int64_t N, int64_t K) {
  if (N < 1 || K < tri::kBlock || K % tri::kBlock != 0) return TRI_ERR_SHAPE;
  if (N > kMaxDim || K > kMaxDim) return TRI_ERR_SHAPE;
  if (N * K >= (int64_t(1) << 40)) return TRI_ERR_SHAPE;
  return TRI_OK;
}

size_t up256(size_t x) { return (x + 255) & ~size_t(255); }

// The integer path reads TQ1 planes directly for M <= 2 (the decode
// regime, where the weight stream is the cost); the other tensor-core kernels
// consume TQ2 planes, and TQ1 weights reach them through a transcode into the
// head of the workspace (N*K/4 bytes).
bool tq1_direct(int fmt, int path, int64_t M) { return fmt == TRI_TQ1 && path == TRI_PATH_I8 && M <= 2; }

bool path_supported(int fmt, int path, int64_t M, int64_t N, int64_t K) {
  switch (path) {
    case TRI_PATH_SIMT: return true;
    case TRI_PATH_MMA: return tri::gemv_mma_supported(TRI_TQ2, M, N, K);
    case TRI_PATH_TCGEN05: return tri::gemm_tc_supported(TRI_TQ2, M, N, K);
    case TRI_PATH_I8: return tri::gemv_i8_supported(M, N, K, tq1_direct(fmt, path, M));
    default: return false;
  }
}

size_t transcode_bytes(int fmt, int path, int64_t M, int64_t N, int64_t K) {
  return (fmt == TRI_TQ1 && path != TRI_PATH_SIMT && !tq1_direct(fmt, path, M))
             ? up256((size_t)N * (size_t)K / 4)
             : 0;
}

size_t path_ws_bytes(int fmt, int path, int64_t M, int64_t N, int64_t K, int sms) {
  size_t inner = 0;
  if (path == TRI_PATH_MMA) inner = tri::gemv_mma_ws_bytes(TRI_TQ2, M, N, K, sms);
  if (path == TRI_PATH_TCGEN05) inner = tri::gemm_tc_ws_bytes(TRI_TQ2, M, N, K, sms);
  if (path == TRI_PATH_I8) inner = tri::gemv_i8_ws_bytes(M, N, K, sms, tq1_direct(fmt, path, M));
  return transcode_bytes(fmt, path, M, N, K) + inner;
}

// shapes the decode-step attention serves
tri_status attn_shape(int64_t M, int64_t H, int64_t Hkv, int64_t Lmax, int64_t max_len) {
  if (M < 1 || M > 65535 || H < 1 || Hkv < 1 || Hkv > 65535 || H % Hkv != 0 || H / Hkv > 8) return TRI_ERR_SHAPE;
  if (Lmax < 1 || Lmax > (int64_t(1) << 24) || max_len < 1 || max_len > Lmax) return TRI_ERR_SHAPE;
  if (M * Hkv * Lmax > (int64_t(1) << 40) / 128 || M * H > (int64_t(1) << 31) - 1) return TRI_ERR_SHAPE;
  return TRI_OK;
}

int auto_path(int fmt, int64_t M, int64_t N, int64_t K) {
  if (M <= 16 && path_supported(fmt, TRI_PATH_I8, M, N, K)) return TRI_PATH_I8;
  if (M <= 16 && path_supported(fmt, TRI_PATH_MMA, M, N, K)) return TRI_PATH_MMA;
  if (M > 16 && path_supported(fmt, TRI_PATH_TCGEN05, M, N, K)) return TRI_PATH_TCGEN05;
  return TRI_PATH_SIMT;
}

}  // namespace

extern "C" {

const char* tri_status_string(int status) {
  switch (status) {
    case TRI_OK: return "ok";
    case TRI_ERR_INVALID_ARG: return "invalid argument";
    case TRI_ERR_SHAPE: return "invalid shape (need N,M >= 1, K >= 256, K % 256 == 0)";
    case TRI_ERR_ALIGNMENT: return "misaligned pointer";
    case TRI_ERR_NONFINITE: return "non-finite weights";
    case TRI_ERR_INVALID_CODE: return "invalid packed code";
    case TRI_ERR_CUDA: return "CUDA runtime error";
    case TRI_ERR_NOT_IMPLEMENTED: return "kernel path not available for this shape";
    case TRI_ERR_WORKSPACE: return "workspace missing or too small";
    case TRI_ERR_NO_DEVICE: return "current device is not an sm_100 GPU";
    case TRI_ERR_SCRATCH_LIMIT: return "shape needs more scratch than the no-alloc entry point's static 8 MiB array";
    default: return "unknown status";
  }
}

int tri_version(void) { return 100; }

const char* tri_last_cuda_error(void) { return cudaGetErrorString(g_last_cuda); }

size_t tri_absmean_workspace_bytes(int64_t, int64_t) { return tri::absmean_ws_bytes(); }

tri_status tri_absmean(const float* W, int64_t N, int64_t K, float eps, float* gamma,
                       void* workspace, size_t workspace_bytes, void* stream) {
  if (!W || !gamma) return TRI_ERR_INVALID_ARG;
  if (!(eps >= 0.f) || eps > 3.0e38f) return TRI_ERR_INVALID_ARG;
  tri_status st = check_nk(N, K);
  if (st != TRI_OK) return st;
  if (!workspace || workspace_bytes < tri::absmean_ws_bytes()) return TRI_ERR_WORKSPACE;
  if (!aligned(W, 16) || !aligned(workspace, 16) || !aligned(gamma, 4)) return TRI_ERR_ALIGNMENT;
  DevInfo di;
  if ((st = device_info(&di)) != TRI_OK) return st;
  return from_cuda(tri::launch_absmean(W, N * K, eps, gamma, workspace,
                                       static_cast<cudaStream_t>(stream)));
}

tri_status tri_ternarize(const float* W, int64_t N, int64_t K, float eps, int8_t* trits,
                         float* gamma, void* workspace, size_t workspace_bytes, void* stream) {
  if (!trits) return TRI_ERR_INVALID_ARG;
  if (!aligned(trits, 16)) return TRI_ERR_ALIGNMENT;
  tri_status st = tri_absmean(W, N, K, eps, gamma, workspace, workspace_bytes, stream);
  if (st != TRI_OK) return st;
  return from_cuda(tri::launch_ternarize(W, N * K, gamma, trits, static_cast<cudaStream_t>(stream)));
}

static tri_status pack_common(int fmt, const int8_t* trits, int64_t N, int64_t K,
                              const float* scales, int64_t n_scales, uint8_t* qs, uint16_t* d,
                              int32_t* invalid_count, void* stream) {
  if (!trits || !scales || !qs || !d) return TRI_ERR_INVALID_ARG;
  tri_status st = check_nk(N, K);
  if (st != TRI_OK) return st;
  if (n_scales != 1 && n_scales != N * (K / tri::kBlock)) return TRI_ERR_INVALID_ARG;
  if (!aligned(trits, 16) || !aligned(scales, 4) || !aligned(d, 4)) return TRI_ERR_ALIGNMENT;
  if (!aligned(qs, fmt == TRI_TQ2 ? 16 : 4)) return TRI_ERR_ALIGNMENT;
  if (invalid_count && !aligned(invalid_count, 4)) return TRI_ERR_ALIGNMENT;
  DevInfo di;
  if ((st = device_info(&di)) != TRI_OK) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (fmt == TRI_TQ2)
    return from_cuda(tri::launch_pack_tq2(trits, N, K, scales, n_scales, qs, d, invalid_count, s));
  return from_cuda(tri::launch_pack_tq1(trits, N, K, scales, n_scales, qs, d, invalid_count, s));
}

tri_status tri_pack_tq2(const int8_t* trits, int64_t N, int64_t K, const float* scales,
                        int64_t n_scales, uint8_t* qs, uint16_t* d, int32_t* invalid_count,
                        void* stream) {
  return pack_common(TRI_TQ2, trits, N, K, scales, n_scales, qs, d, invalid_count, stream);
}

tri_status tri_pack_tq1(const int8_t* trits, int64_t N, int64_t K, const float* scales,
                        int64_t n_scales, uint8_t* qs, uint16_t* d, int32_t* invalid_count,
                        void* stream) {
  return pack_common(TRI_TQ1, trits, N, K, scales, n_scales, qs, d, invalid_count, stream);
}

tri_status tri_unpack(int format, const uint8_t* qs, int64_t N, int64_t K, int8_t* trits,
                      int32_t* invalid_count, void* stream) {
  if (format != TRI_TQ2 && format != TRI_TQ1) return TRI_ERR_INVALID_ARG;
  if (!qs || !trits) return TRI_ERR_INVALID_ARG;
  tri_status st = check_nk(N, K);
  if (st != TRI_OK) return st;
  if (!aligned(trits, 16) || !aligned(qs, format == TRI_TQ2 ? 16 : 4)) return TRI_ERR_ALIGNMENT;
  if (invalid_count && !aligned(invalid_count, 4)) return TRI_ERR_ALIGNMENT;
  DevInfo di;
  if ((st = device_info(&di)) != TRI_OK) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (format == TRI_TQ2) return from_cuda(tri::launch_unpack_tq2(qs, N, K, trits, invalid_count, s));
  return from_cuda(tri::launch_unpack_tq1(qs, N, K, trits, invalid_count, s));
}

int tri_gemm_auto_path(int format, int64_t M, int64_t N, int64_t K) {
  if (format != TRI_TQ2 && format != TRI_TQ1) return -1;
  if (M < 1 || M > kMaxDim || check_nk(N, K) != TRI_OK) return -1;
  return auto_path(format, M, N, K);
}

size_t tri_gemm_workspace_bytes(int format, int64_t M, int64_t N, int64_t K) {
  if (tri_gemm_auto_path(format, M, N, K) < 0) return 0;
  DevInfo di;
  int sms = 148;
  if (device_info(&di) == TRI_OK) sms = di.sms;
  size_t r = 0;
  for (int path = TRI_PATH_SIMT; path <= TRI_PATH_I8; ++path)
    if (path_supported(format, path, M, N, K)) {
      const size_t b = path_ws_bytes(format, path, M, N, K, sms);
      if (b > r) r = b;
    }
  return r < 256 ? 256 : r;
}

tri_status tri_gemm(int format, int path, const uint16_t* X, const uint8_t* qs, const uint16_t* d,
                    uint16_t* Y, int64_t M, int64_t N, int64_t K, void* workspace,
                    size_t workspace_bytes, void* stream) {
  if (format != TRI_TQ2 && format != TRI_TQ1) return TRI_ERR_INVALID_ARG;
  if (path < TRI_PATH_AUTO || path > TRI_PATH_I8) return TRI_ERR_INVALID_ARG;
  if (!X || !qs || !d || !Y) return TRI_ERR_INVALID_ARG;
  if (M < 1 || M > kMaxDim) return TRI_ERR_SHAPE;
  tri_status st = check_nk(N, K);
  if (st != TRI_OK) return st;
  if (!aligned(X, 16) || !aligned(Y, 16) || !aligned(d, 4)) return TRI_ERR_ALIGNMENT;
  if (!aligned(qs, format == TRI_TQ2 ? 16 : 4)) return TRI_ERR_ALIGNMENT;
  DevInfo di;
  if ((st = device_info(&di)) != TRI_OK) return st;
  if (path == TRI_PATH_AUTO) path = auto_path(format, M, N, K);
  if (!path_supported(format, path, M, N, K)) return TRI_ERR_NOT_IMPLEMENTED;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const __half* Xh = reinterpret_cast<const __half*>(X);
  const __half* dh = reinterpret_cast<const __half*>(d);
  __half* Yh = reinterpret_cast<__half*>(Y);
  if (path == TRI_PATH_SIMT)
    return from_cuda(tri::launch_gemm_simt(format, Xh, qs, dh, Yh, (int)M, (int)N, (int)K, s));
  const size_t need = path_ws_bytes(format, path, M, N, K, di.sms);
  if (need && (!workspace || workspace_bytes < need)) return TRI_ERR_WORKSPACE;
  if (workspace && !aligned(workspace, 256)) return TRI_ERR_ALIGNMENT;
  const uint8_t* q2 = qs;
  uint8_t* inner = static_cast<uint8_t*>(workspace);
  const bool direct = tq1_direct(format, path, M);
  if (format == TRI_TQ1 && !direct) {
    uint8_t* t = static_cast<uint8_t*>(workspace);
    const cudaError_t e = tri::launch_transcode_tq1_tq2(qs, N, K, t, s);
    if (e != cudaSuccess) return from_cuda(e);
    q2 = t;
    inner = t + transcode_bytes(format, path, M, N, K);
  }
  switch (path) {
    case TRI_PATH_MMA:
      return from_cuda(tri::launch_gemv_mma(TRI_TQ2, Xh, q2, dh, Yh, (int)M, (int)N, (int)K, inner,
                                            di.sms, s));
    case TRI_PATH_I8:
      return from_cuda(
          tri::launch_gemv_i8(Xh, q2, dh, Yh, (int)M, (int)N, (int)K, inner, di.sms, s, direct));
    case TRI_PATH_TCGEN05:
      return from_cuda(tri::launch_gemm_tc(TRI_TQ2, Xh, q2, dh, Yh, (int)M, (int)N, (int)K, inner,
                                           di.sms, s));
    default:
      return TRI_ERR_INVALID_ARG;
  }
}

namespace {
// the fused epilogue serves 3 <= M <= 16 on the integer path
bool swiglu_fused(int path, int64_t M) { return path == TRI_PATH_I8 && M >= 3 && M <= 16; }
}  // namespace

size_t tri_gemm_swiglu_workspace_bytes(int format, int64_t M, int64_t F, int64_t K) {
  if (F < 8 || F % 8 != 0) return 0;
  const size_t g = tri_gemm_workspace_bytes(format, M, 2 * F, K);
  if (g == 0) return 0;
  return up256(g) + up256((size_t)M * 2 * F * 2);
}

tri_status tri_gemm_swiglu(int format, int path, const uint16_t* X, const uint8_t* qs, const uint16_t* d,
                           uint16_t* Y, int64_t M, int64_t F, int64_t K, void* workspace,
                           size_t workspace_bytes, void* stream) {
  if (format != TRI_TQ2 && format != TRI_TQ1) return TRI_ERR_INVALID_ARG;
  if (path < TRI_PATH_AUTO || path > TRI_PATH_I8) return TRI_ERR_INVALID_ARG;
  if (!X || !qs || !d || !Y) return TRI_ERR_INVALID_ARG;
  if (M < 1 || M > kMaxDim) return TRI_ERR_SHAPE;
  if (F < 8 || F % 8 != 0 || F > kMaxDim / 2) return TRI_ERR_SHAPE;
  const int64_t N = 2 * F;
  tri_status st = check_nk(N, K);
  if (st != TRI_OK) return st;
  if (!aligned(X, 16) || !aligned(Y, 16) || !aligned(d, 4)) return TRI_ERR_ALIGNMENT;
  if (!aligned(qs, format == TRI_TQ2 ? 16 : 4)) return TRI_ERR_ALIGNMENT;
  DevInfo di;
  if ((st = device_info(&di)) != TRI_OK) return st;
  if (path == TRI_PATH_AUTO) path = auto_path(format, M, N, K);
  if (!path_supported(format, path, M, N, K)) return TRI_ERR_NOT_IMPLEMENTED;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const __half* Xh = reinterpret_cast<const __half*>(X);
  const __half* dh = reinterpret_cast<const __half*>(d);
  __half* Yh = reinterpret_cast<__half*>(Y);
  const size_t gemm_need = path == TRI_PATH_SIMT ? 0 : path_ws_bytes(format, path, M, N, K, di.sms);
  const bool fused = swiglu_fused(path, M);
  const size_t need = fused ? gemm_need : up256(gemm_need) + up256((size_t)M * N * 2);
  if (need && (!workspace || workspace_bytes < need)) return TRI_ERR_WORKSPACE;
  if (workspace && !aligned(workspace, 256)) return TRI_ERR_ALIGNMENT;
  const uint8_t* q2 = qs;
  uint8_t* inner = static_cast<uint8_t*>(workspace);
  const bool direct = tq1_direct(format, path, M);
  if (format == TRI_TQ1 && path != TRI_PATH_SIMT && !direct) {
    uint8_t* t = static_cast<uint8_t*>(workspace);
    const cudaError_t e = tri::launch_transcode_tq1_tq2(qs, N, K, t, s);
    if (e != cudaSuccess) return from_cuda(e);
    q2 = t;
    inner = t + transcode_bytes(format, path, M, N, K);
  }
  if (fused)
    return from_cuda(tri::launch_gemv_i8n(Xh, q2, dh, Yh, (int)M, (int)N, (int)K, inner, di.sms, s, true));
  // unfused: the [M][2F] product into the workspace tail, then the combine
  __half* G2 = reinterpret_cast<__half*>(static_cast<uint8_t*>(workspace) + up256(gemm_need));
  cudaError_t e = cudaSuccess;
  switch (path) {
    case TRI_PATH_SIMT:
      e = tri::launch_gemm_simt(format, Xh, qs, dh, G2, (int)M, (int)N, (int)K, s);
      break;
    case TRI_PATH_MMA:
      e = tri::launch_gemv_mma(TRI_TQ2, Xh, q2, dh, G2, (int)M, (int)N, (int)K, inner, di.sms, s);
      break;
    case TRI_PATH_I8:
      e = tri::launch_gemv_i8(Xh, q2, dh, G2, (int)M, (int)N, (int)K, inner, di.sms, s, direct);
      break;
    case TRI_PATH_TCGEN05:
      e = tri::launch_gemm_tc(TRI_TQ2, Xh, q2, dh, G2, (int)M, (int)N, (int)K, inner, di.sms, s);
      break;
    default:
      return TRI_ERR_INVALID_ARG;
  }
  if (e != cudaSuccess) return from_cuda(e);
  return from_cuda(tri::launch_swiglu_combine(G2, Yh, M, F, s));
}

int tri_gemm_tq2_noalloc_fits(int64_t M, int64_t N, int64_t K) {
  if (M < 1 || M > 16 || check_nk(N, K) != TRI_OK) return 0;
  DevInfo di;
  if (device_info(&di) != TRI_OK) return 0;
  return tri::gemv_noalloc_scratch_need(M, N, K, di.sms) <= tri::gemv_noalloc_scratch_limit() ? 1 : 0;
}

tri_status tri_gemm_tq2_noalloc(const uint16_t* X, const uint8_t* qs, const uint16_t* d, uint16_t* Y,
                                int64_t M, int64_t N, int64_t K, void* stream) {
  if (!X || !qs || !d || !Y) return TRI_ERR_INVALID_ARG;
  if (M < 1 || M > 16) return TRI_ERR_SHAPE;
  tri_status st = check_nk(N, K);
  if (st != TRI_OK) return st;
  if (!aligned(X, 16) || !aligned(Y, 16) || !aligned(d, 4) || !aligned(qs, 16)) return TRI_ERR_ALIGNMENT;
  DevInfo di;
  if ((st = device_info(&di)) != TRI_OK) return st;
  if (tri::gemv_noalloc_scratch_need(M, N, K, di.sms) > tri::gemv_noalloc_scratch_limit())
    return TRI_ERR_SCRATCH_LIMIT;
  return from_cuda(tri::launch_gemv_mma_noalloc(
      reinterpret_cast<const __half*>(X), qs, reinterpret_cast<const __half*>(d),
      reinterpret_cast<__half*>(Y), (int)M, (int)N, (int)K, di.sms, static_cast<cudaStream_t>(stream)));
}

tri_status tri_wait_status(uint32_t* code, int clear, void* stream) {
  if (!code) return TRI_ERR_INVALID_ARG;
  DevInfo di;
  tri_status st = device_info(&di);
  if (st != TRI_OK) return st;
  unsigned c = 0;
  st = from_cuda(tri::read_wait_status(&c, clear != 0, static_cast<cudaStream_t>(stream)));
  if (st == TRI_OK) *code = c;
  return st;
}

tri_status tri_selftest_wait_timeout(int which, void* scratch, void* stream) {
  if ((which != 0 && which != 1) || !scratch) return TRI_ERR_INVALID_ARG;
  if (!aligned(scratch, 8)) return TRI_ERR_ALIGNMENT;
  DevInfo di;
  tri_status st = device_info(&di);
  if (st != TRI_OK) return st;
  return from_cuda(tri::launch_expire_wait(which, scratch, static_cast<cudaStream_t>(stream)));
}

tri_status tri_gemm_tq2(const uint16_t* X, const uint8_t* qs, const uint16_t* d, uint16_t* Y,
                        int64_t M, int64_t N, int64_t K, void* workspace, size_t workspace_bytes,
                        void* stream) {
  return tri_gemm(TRI_TQ2, TRI_PATH_AUTO, X, qs, d, Y, M, N, K, workspace, workspace_bytes, stream);
}

tri_status tri_gemm_tq1(const uint16_t* X, const uint8_t* qs, const uint16_t* d, uint16_t* Y,
                        int64_t M, int64_t N, int64_t K, void* workspace, size_t workspace_bytes,
                        void* stream) {
  return tri_gemm(TRI_TQ1, TRI_PATH_AUTO, X, qs, d, Y, M, N, K, workspace, workspace_bytes, stream);
}

// ---------------------------------------------------------------- decode step
tri_status tri_rmsnorm(const uint16_t* x, const uint16_t* r, const uint16_t* g, uint16_t* h_out, uint16_t* y,
                       int64_t M, int64_t D, float eps, void* stream) {
  if (!x || !g || !y || (r && !h_out)) return TRI_ERR_INVALID_ARG;
  if (!(eps >= 0.f) || !(eps < 1e30f)) return TRI_ERR_INVALID_ARG;
  if (r && (h_out == x || h_out == r)) return TRI_ERR_INVALID_ARG;
  if (M < 1 || M > kMaxDim || D < 8 || D > (int64_t(1) << 20) || D % 8 != 0) return TRI_ERR_SHAPE;
  if (!aligned(x, 16) || !aligned(g, 16) || !aligned(y, 16) || (r && !aligned(r, 16)) ||
      (h_out && !aligned(h_out, 16)))
    return TRI_ERR_ALIGNMENT;
  DevInfo di;
  tri_status st = device_info(&di);
  if (st != TRI_OK) return st;
  return from_cuda(tri::launch_rmsnorm(reinterpret_cast<const __half*>(x), reinterpret_cast<const __half*>(r),
                                       reinterpret_cast<const __half*>(g), r ? reinterpret_cast<__half*>(h_out) : nullptr,
                                       reinterpret_cast<__half*>(y), M, D, eps, static_cast<cudaStream_t>(stream)));
}

tri_status tri_rope_table(float* cs, int64_t Lmax, int64_t dh, double theta, void* stream) {
  if (!cs || !(theta > 1.0) || !(theta < 1e300)) return TRI_ERR_INVALID_ARG;
  if (dh != 128 || Lmax < 1 || Lmax > (int64_t(1) << 24)) return TRI_ERR_SHAPE;
  if (!aligned(cs, 8)) return TRI_ERR_ALIGNMENT;
  DevInfo di;
  tri_status st = device_info(&di);
  if (st != TRI_OK) return st;
  return from_cuda(tri::launch_rope_table(reinterpret_cast<float2*>(cs), Lmax, dh, theta,
                                          static_cast<cudaStream_t>(stream)));
}

tri_status tri_qknorm_rope(const uint16_t* qkv, const int32_t* pos, const uint16_t* gq, const uint16_t* gk,
                           const float* cs, uint16_t* q_out, uint16_t* kcache, uint16_t* vcache, int64_t M,
                           int64_t H, int64_t Hkv, int64_t Lmax, float eps, void* stream) {
  if (!qkv || !pos || !gq || !gk || !cs || !q_out || !kcache || !vcache) return TRI_ERR_INVALID_ARG;
  if (!(eps >= 0.f) || !(eps < 1e30f)) return TRI_ERR_INVALID_ARG;
  if (M < 1 || H < 1 || Hkv < 1 || H % Hkv != 0 || Lmax < 1 || Lmax > (int64_t(1) << 24)) return TRI_ERR_SHAPE;
  if (M * (H + 2 * Hkv) > kMaxDim || M * Hkv * Lmax > (int64_t(1) << 40) / 128) return TRI_ERR_SHAPE;
  if (!aligned(qkv, 16) || !aligned(gq, 16) || !aligned(gk, 16) || !aligned(q_out, 16) ||
      !aligned(kcache, 16) || !aligned(vcache, 16) || !aligned(pos, 4) || !aligned(cs, 8))
    return TRI_ERR_ALIGNMENT;
  DevInfo di;
  tri_status st = device_info(&di);
  if (st != TRI_OK) return st;
  return from_cuda(tri::launch_qknorm_rope(
      reinterpret_cast<const __half*>(qkv), pos, reinterpret_cast<const __half*>(gq),
      reinterpret_cast<const __half*>(gk), reinterpret_cast<const float2*>(cs), reinterpret_cast<__half*>(q_out),
      reinterpret_cast<__half*>(kcache), reinterpret_cast<__half*>(vcache), M, H, Hkv, Lmax, eps,
      static_cast<cudaStream_t>(stream)));
}

size_t tri_attention_decode_workspace_bytes(int64_t M, int64_t H, int64_t Hkv, int64_t max_len) {
  if (attn_shape(M, H, Hkv, max_len, max_len) != TRI_OK) return 0;
  DevInfo di;
  int sms = 148;
  if (device_info(&di) == TRI_OK) sms = di.sms;
  return tri::attention_decode_ws_bytes(M, H, Hkv, max_len, sms);
}

tri_status tri_attention_decode(const uint16_t* q, const uint16_t* kcache, const uint16_t* vcache,
                                const int32_t* pos, uint16_t* out, int64_t M, int64_t H, int64_t Hkv,
                                int64_t Lmax, int64_t max_len, void* workspace, size_t workspace_bytes,
                                void* stream) {
  if (!q || !kcache || !vcache || !pos || !out) return TRI_ERR_INVALID_ARG;
  tri_status st = attn_shape(M, H, Hkv, Lmax, max_len);
  if (st != TRI_OK) return st;
  if (!aligned(q, 16) || !aligned(kcache, 16) || !aligned(vcache, 16) || !aligned(out, 16) || !aligned(pos, 4))
    return TRI_ERR_ALIGNMENT;
  DevInfo di;
  if ((st = device_info(&di)) != TRI_OK) return st;
  const size_t need = tri::attention_decode_ws_bytes(M, H, Hkv, max_len, di.sms);
  if (!workspace || workspace_bytes < need) return TRI_ERR_WORKSPACE;
  if (!aligned(workspace, 256)) return TRI_ERR_ALIGNMENT;
  return from_cuda(tri::launch_attention_decode(
      reinterpret_cast<const __half*>(q), reinterpret_cast<const __half*>(kcache),
      reinterpret_cast<const __half*>(vcache), pos, reinterpret_cast<__half*>(out), M, H, Hkv, Lmax, max_len,
      workspace, di.sms, static_cast<cudaStream_t>(stream)));
}

}  // extern "C"
