// Internal declarations shared by the library's translation units.
// Everything here is device/host plumbing for sm_100a; the public C ABI is
// include/tri.h.
#pragma once

#include <cstdint>
#include <cstddef>
#include <cuda_runtime.h>
#include <cuda_fp16.h>

#include "../../include/tri.h"

namespace tri {

constexpr int kBlock = 256;          // weights per block (one fp16 scale each)
constexpr int kTq2BlockBytes = 64;   // 256 x 2 bits
constexpr int kTq1BlockBytes = 52;   // 51 five-trit bytes + 1 byte for trit 255
constexpr int kTq1Groups = 51;

// ---- launchers (each returns cudaSuccess or the launch error) -------------
cudaError_t launch_absmean(const float* W, int64_t n, float eps, float* gamma,
                           void* ws, cudaStream_t s);
cudaError_t launch_ternarize(const float* W, int64_t n, const float* gamma,
                             int8_t* trits, cudaStream_t s);
size_t absmean_ws_bytes();

cudaError_t launch_pack_tq2(const int8_t* trits, int64_t N, int64_t K, const float* scales,
                            int64_t n_scales, uint8_t* qs, uint16_t* d, int32_t* invalid,
                            cudaStream_t s);
cudaError_t launch_pack_tq1(const int8_t* trits, int64_t N, int64_t K, const float* scales,
                            int64_t n_scales, uint8_t* qs, uint16_t* d, int32_t* invalid,
                            cudaStream_t s);
cudaError_t launch_unpack_tq2(const uint8_t* qs, int64_t N, int64_t K, int8_t* trits,
                              int32_t* invalid, cudaStream_t s);
cudaError_t launch_unpack_tq1(const uint8_t* qs, int64_t N, int64_t K, int8_t* trits,
                              int32_t* invalid, cudaStream_t s);

// TQ1 plane -> TQ2 plane (N*K/4 bytes, 16-B aligned), for the tensor-core paths
cudaError_t launch_transcode_tq1_tq2(const uint8_t* qs1, int64_t N, int64_t K, uint8_t* qs2,
                                     cudaStream_t s);

cudaError_t launch_gemm_simt(int fmt, const __half* X, const uint8_t* qs, const __half* d,
                             __half* Y, int M, int N, int K, cudaStream_t s);

// decode-regime tensor-core path (M <= 16)
bool gemv_mma_supported(int fmt, int64_t M, int64_t N, int64_t K);
size_t gemv_mma_ws_bytes(int fmt, int64_t M, int64_t N, int64_t K, int num_sms);
cudaError_t launch_gemv_mma(int fmt, const __half* X, const uint8_t* qs, const __half* d,
                            __half* Y, int M, int N, int K, void* ws, int num_sms,
                            cudaStream_t s);

// decode-regime integer tensor-core path (M <= 16: gemv_i8.cu for M <= 2, TQ2
// or TQ1 planes read directly; gemv_i8n.cu for 3 <= M <= 16, TQ2)
bool gemv_i8n_supported(int64_t M, int64_t N, int64_t K);
size_t gemv_i8n_ws_bytes(int64_t M, int64_t N, int64_t K, int num_sms);
// swiglu: N = 2F rows of gate and up interleaved in groups of 8, Y = silu(gate) * up [M][F]
cudaError_t launch_gemv_i8n(const __half* X, const uint8_t* qs, const __half* d, __half* Y, int M, int N,
                            int K, void* ws, int num_sms, cudaStream_t s, bool swiglu = false);
// silu(G) * U from a [M][2F] fp16 product in the interleaved row order, into Y [M][F]
cudaError_t launch_swiglu_combine(const __half* G2, __half* Y, int64_t M, int64_t F, cudaStream_t s);
// tq1: qs is a TQ1 plane (M <= 2 only)
bool gemv_i8_supported(int64_t M, int64_t N, int64_t K, bool tq1 = false);
size_t gemv_i8_ws_bytes(int64_t M, int64_t N, int64_t K, int num_sms, bool tq1 = false);
cudaError_t launch_gemv_i8(const __half* X, const uint8_t* qs, const __half* d, __half* Y, int M,
                           int N, int K, void* ws, int num_sms, cudaStream_t s, bool tq1 = false);

// one-block decode step around the ternary layers (decode.cu); head dim 128
cudaError_t launch_rmsnorm(const __half* x, const __half* r, const __half* g, __half* h_out, __half* y,
                           int64_t M, int64_t D, float eps, cudaStream_t s);
cudaError_t launch_rope_table(float2* cs, int64_t Lmax, int64_t dh, double theta, cudaStream_t s);
cudaError_t launch_qknorm_rope(const __half* qkv, const int* pos, const __half* gq, const __half* gk,
                               const float2* cs, __half* q_out, __half* kc, __half* vc, int64_t M, int64_t H,
                               int64_t Hkv, int64_t Lmax, float eps, cudaStream_t s);
size_t attention_decode_ws_bytes(int64_t M, int64_t H, int64_t Hkv, int64_t max_len, int sms);
cudaError_t launch_attention_decode(const __half* q, const __half* kc, const __half* vc, const int* pos,
                                    __half* out, int64_t M, int64_t H, int64_t Hkv, int64_t Lmax,
                                    int64_t max_len, void* ws, int sms, cudaStream_t s);

// decode-regime path with library-owned static scratch (no allocation)
size_t gemv_noalloc_scratch_limit();
size_t gemv_noalloc_scratch_need(int64_t M, int64_t N, int64_t K, int num_sms);
cudaError_t launch_gemv_mma_noalloc(const __half* X, const uint8_t* qs, const __half* d, __half* Y,
                                    int M, int N, int K, int num_sms, cudaStream_t s);

// compute-regime tcgen05 path (M >= 64)
bool gemm_tc_supported(int fmt, int64_t M, int64_t N, int64_t K);
size_t gemm_tc_ws_bytes(int fmt, int64_t M, int64_t N, int64_t K, int num_sms);
cudaError_t launch_gemm_tc(int fmt, const __half* X, const uint8_t* qs, const __half* d,
                           __half* Y, int M, int N, int K, void* ws, int num_sms,
                           cudaStream_t s);

// ---- device wait status (status.cu) ----------------------------------------
// codes recorded by a bounded wait that ran out; the values name the wait:
// 1-2 gemv_mma.cu, 11 gemv_i8.cu, 21-26 gemm_tc.cu, 41-42 gemv_i8n.cu
constexpr unsigned kSelfTestMbarCode = 90;
constexpr unsigned kSelfTestStampCode = 91;
// the current device's status word (device address)
cudaError_t wait_status_word(unsigned** out);
// synchronizes `s`, then copies the word to *code and optionally zeroes it
cudaError_t read_wait_status(unsigned* code, bool clear, cudaStream_t s);
// a one-block kernel whose wait (0: mbarrier, 1: stamped word) runs out;
// `scratch` is 8 device bytes the stamped word lives in
cudaError_t launch_expire_wait(int which, void* scratch, cudaStream_t s);

// ---- small helpers ---------------------------------------------------------
__host__ __device__ inline int64_t ceil_div(int64_t a, int64_t b) { return (a + b - 1) / b; }

}  // namespace tri
