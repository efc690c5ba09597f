/*
 * tri.h -- C ABI of the B200 ternary-weight linear-layer library (libtri_b200.so).
 *
 * The library implements, for NVIDIA B200 (sm_100a), the inference path of a
 * ternary linear layer as described on the page "Scaling Laws and Efficient
 * Inference for Ternary Language Models" (Spectra-1.1 / TriTera project page)
 * and on "Spectra: Surprising Effectiveness of Pretraining Ternary Language
 * Models at Scale" (section "Architecture of TriLM and FloatLM"):
 *
 *   absmean scale      gamma = eps + mean|W|                   ("The model", step 1)
 *   ternarize          W_hat = round(clip(W / gamma, -1, 1))   ("The model", step 2)
 *   TQ2 / TQ1 packing  2 bits or 1.6 bits per weight           ("Packing ternary weights")
 *   ternary GEMM       Y = X (gamma W_hat)^T, fp32 accumulation ("The model", step 3;
 *                      "TriRun: ternary inference on GPUs")
 *
 * Conventions for every entry point
 * ---------------------------------
 *  - Shapes: W is N x K (N output features, K input features), row-major.
 *    X is M x K fp16 row-major, Y is M x N fp16 row-major.  K must be a
 *    positive multiple of 256 (one block = 256 consecutive weights of a row).
 *  - Every data pointer is a DEVICE pointer, allocated and owned by the
 *    caller.  The library allocates nothing and, except in tri_wait_status,
 *    never synchronizes the host; all work is enqueued on `stream` (a
 *    cudaStream_t; NULL = legacy default stream) in call order.
 *  - fp16 tensors are passed as uint16_t bit patterns (IEEE binary16).
 *  - Arguments are validated on the host before anything is enqueued; a
 *    non-OK status means nothing was launched.  A launch failure reported by
 *    the CUDA runtime returns TRI_ERR_CUDA.  No kernel traps or asserts:
 *    data errors (non-finite weights, invalid packed codes) are reported
 *    through device-side results described per function, and every wait of
 *    one thread block on another or on an asynchronous copy is bounded and
 *    reports through the device wait status word (tri_wait_status).
 *  - Buffers given to one call must not overlap unless stated.
 *
 * Packed formats (readings of the pages, fixed by this library)
 * -------------------------------------------------------------
 *  TQ2 ("2 bits per weight"): the shifted digit d' = t + 1 in {0,1,2} of
 *    weight k of a row is stored in bits 2*(k%4) .. 2*(k%4)+1 of byte k/4 of
 *    that row, so a little-endian 32-bit word holds sixteen consecutive
 *    weights, weight j at bits 2j ("TriRun": "each 32-bit word holds sixteen
 *    2-bit weights").  qs is uint8[N][K/4] (64 bytes per 256-block).
 *  TQ1 ("1.6 bits per weight"): five consecutive weights form a base-3 number
 *    N5 = sum_j d'_j 3^(4-j) (first weight most significant), stored as the
 *    byte floor((256*N5 + 242)/243).  Each 256-block takes 52 bytes: bytes
 *    0..50 hold weights 5g..5g+4 of the block, byte 51 holds weight 255 as its
 *    leading digit followed by four zero weights.  qs is uint8[N][52*K/256].
 *  Scales (section "Fast inference on CPUs": one 16-bit scale per 256-block):
 *    d is fp16[N][K/256]; the weight of row n, column k is d[n][k/256] * t.
 */
#ifndef TRI_B200_H
#define TRI_B200_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define TRI_API __attribute__((visibility("default")))
#else
#define TRI_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum tri_status {
    TRI_OK = 0,
    TRI_ERR_INVALID_ARG = 1,      /* null pointer, bad enum, eps < 0 ...      */
    TRI_ERR_SHAPE = 2,            /* M, N, K out of range or K % 256 != 0     */
    TRI_ERR_ALIGNMENT = 3,        /* a pointer is not 16-byte aligned         */
    TRI_ERR_NONFINITE = 4,        /* reserved for wrappers (see tri_absmean)  */
    TRI_ERR_INVALID_CODE = 5,     /* reserved for wrappers (see tri_unpack)   */
    TRI_ERR_CUDA = 6,             /* the CUDA runtime reported an error       */
    TRI_ERR_NOT_IMPLEMENTED = 7,  /* the requested kernel path does not exist */
    TRI_ERR_WORKSPACE = 8,        /* workspace null or smaller than required  */
    TRI_ERR_NO_DEVICE = 9,        /* current device is not sm_100             */
    TRI_ERR_SCRATCH_LIMIT = 10    /* shape needs more than the static scratch */
} tri_status;

typedef enum tri_format { TRI_TQ1 = 1, TRI_TQ2 = 2 } tri_format;

/* Kernel choice for tri_gemm: AUTO picks by M (see tri_gemm). */
typedef enum tri_gemm_path {
    TRI_PATH_AUTO = 0,
    TRI_PATH_SIMT = 1,     /* CUDA-core kernel, any M (correctness baseline)           */
    TRI_PATH_MMA = 2,      /* decode-regime tensor-core kernel, M <= 16                */
    TRI_PATH_TCGEN05 = 3,  /* compute-regime kernel: tcgen05 MMA, TMEM accumulators    */
    TRI_PATH_I8 = 4        /* decode-regime int8 tensor-core kernels (exact integer
                              products with 24-bit fixed-point X), M <= 16           */
} tri_gemm_path;

/* Human-readable name of a status code (static string, never NULL). */
TRI_API const char* tri_status_string(int status);

/* Library ABI version (major*100 + minor). */
TRI_API int tri_version(void);

/* The CUDA runtime's message for the last error behind a TRI_ERR_CUDA
 * returned on the calling host thread (static string, never NULL). */
TRI_API const char* tri_last_cuda_error(void);

/* ------------------------------------------------------------------------
 * Absmean scale ("The model", step 1; Spectra "Architecture": one scale per
 * matrix, the mean absolute value of the latent weights).
 *
 *   gamma = RN32( RN64( RN64(S) / (N*K) ) + eps ),  S = sum |W[n][k]| exactly.
 *
 * The sum is formed exactly (integer accumulation per float exponent), so
 * gamma does not depend on the order of the reduction and is bit-identical
 * across runs and grid sizes.
 *   W         device float32[N][K], read only.
 *   eps       >= 0, finite (1e-6 in the pages' workloads).
 *   gamma     device float32[1], written.  If W holds Inf or NaN, *gamma is
 *             set to NaN (check it on the host to detect non-finite weights).
 *   workspace device scratch of at least tri_absmean_workspace_bytes(N, K)
 *             bytes, 16-byte aligned; its contents on entry do not matter.
 * N*K must be below 2^40.
 * ---------------------------------------------------------------------- */
TRI_API size_t tri_absmean_workspace_bytes(int64_t N, int64_t K);
TRI_API tri_status tri_absmean(const float* W, int64_t N, int64_t K, float eps, float* gamma,
                       void* workspace, size_t workspace_bytes, void* stream);

/* ------------------------------------------------------------------------
 * Absmean ternarization ("The model", steps 1-2):
 *   gamma as in tri_absmean, then trits[n][k] = rint(clip(W/gamma, -1, 1))
 *   with an IEEE float32 division and round-half-to-even; a NaN quotient
 *   (non-finite W, or gamma = 0) gives trit 0.
 *   trits     device int8[N][K], written, values in {-1, 0, 1}.
 * Other arguments as for tri_absmean (same workspace size).
 * ---------------------------------------------------------------------- */
TRI_API tri_status tri_ternarize(const float* W, int64_t N, int64_t K, float eps,
                         int8_t* trits, float* gamma,
                         void* workspace, size_t workspace_bytes, void* stream);

/* ------------------------------------------------------------------------
 * Packing ("Packing ternary weights": "2 bits per weight" for TQ2,
 * "1.6 bits per weight" for TQ1; block scale per "Fast inference on CPUs").
 *   trits     device int8[N][K] in {-1,0,1}; any other value is counted as
 *             invalid and packed as 0.
 *   scales    device float32, n_scales values: 1 (one scale for the matrix,
 *             e.g. gamma from tri_ternarize) or N*K/256 (one per block,
 *             row-major [N][K/256]).  d = fp16(scale), round to nearest even.
 *   qs        device uint8: N*K/4 bytes (TQ2) or N*(K/256)*52 bytes (TQ1).
 *   d         device fp16[N][K/256], written.
 *   invalid_count  device int32[1] or NULL; set to the number of invalid
 *             input trits.
 * qs must be 16-byte aligned for TQ2 and 4-byte aligned for TQ1; d 4-byte.
 * ---------------------------------------------------------------------- */
TRI_API tri_status tri_pack_tq2(const int8_t* trits, int64_t N, int64_t K,
                        const float* scales, int64_t n_scales,
                        uint8_t* qs, uint16_t* d, int32_t* invalid_count, void* stream);
TRI_API tri_status tri_pack_tq1(const int8_t* trits, int64_t N, int64_t K,
                        const float* scales, int64_t n_scales,
                        uint8_t* qs, uint16_t* d, int32_t* invalid_count, void* stream);

/* ------------------------------------------------------------------------
 * Unpacking ("2 bits per weight": d' = (b >> 2j) & 3; "1.6 bits per weight":
 * the multiply-by-3 / high-byte digit extraction).
 *   format    TRI_TQ2 or TRI_TQ1.
 *   qs        packed plane as written by tri_pack_*.
 *   trits     device int8[N][K], written.
 *   invalid_count  device int32[1] or NULL; set to the number of invalid
 *             codes: TQ2 fields equal to 3; TQ1 bytes outside the encoder's
 *             243-value image, plus block-final bytes whose four padding
 *             digits are not the zero weight.  Invalid codes are still decoded
 *             by the same rule (t = d' - 1, so a TQ2 field of 3 gives 2), so
 *             the output is defined for every input byte.
 * ---------------------------------------------------------------------- */
TRI_API tri_status tri_unpack(int format, const uint8_t* qs, int64_t N, int64_t K,
                      int8_t* trits, int32_t* invalid_count, void* stream);

/* ------------------------------------------------------------------------
 * Ternary GEMM ("The model", step 3: Y = X (gamma W_hat)^T; "TriRun": fp16
 * activations, fp32 accumulation, fp16 output):
 *
 *   Y[m][n] = fp16_RN( sum_b d[n][b] * sum_{k in block b} X[m][k] * t[n][k] )
 *
 * accumulated in float32 (the summation order is the kernel's; results are
 * deterministic for a given device, path and shape).
 *   X         device fp16[M][K], 16-byte aligned.
 *   qs, d     packed weights in `format`, as written by tri_pack_*; qs
 *             16-byte aligned (TQ2) or 4-byte aligned (TQ1).  Codes that
 *             are invalid give unspecified (but finite, non-faulting) output.
 *   Y         device fp16[M][N], 16-byte aligned, written.
 *   M >= 1, N >= 1, K >= 256 with K % 256 == 0; M, N, K < 2^31.
 *   workspace device scratch of at least tri_gemm_workspace_bytes(format, M,
 *             N, K) bytes, 256-byte aligned; its contents on entry do not
 *             matter (each call initialises what it uses).  Calls that share
 *             one workspace must be ordered (same stream, or events).
 *   path      TRI_PATH_AUTO chooses TRI_PATH_I8 for M <= 16 (TRI_PATH_MMA
 *             where it cannot serve the shape) and TRI_PATH_TCGEN05 above
 *             (TQ1 weights are first
 *             transcoded to TQ2 in the workspace on those three paths); an
 *             explicit path that cannot serve the shape returns
 *             TRI_ERR_NOT_IMPLEMENTED.  TRI_PATH_I8 quantises each
 *             256-element block of X to 24-bit fixed point (step = block
 *             max / 8e6) and forms the block dot products exactly in int32,
 *             an error of at most 2^-24 of sum_k |X[m][k] d[n][b]| per output.
 * ---------------------------------------------------------------------- */
TRI_API size_t tri_gemm_workspace_bytes(int format, int64_t M, int64_t N, int64_t K);
TRI_API tri_status tri_gemm(int format, int path, const uint16_t* X, const uint8_t* qs,
                    const uint16_t* d, uint16_t* Y, int64_t M, int64_t N, int64_t K,
                    void* workspace, size_t workspace_bytes, void* stream);
TRI_API tri_status tri_gemm_tq2(const uint16_t* X, const uint8_t* qs, const uint16_t* d,
                        uint16_t* Y, int64_t M, int64_t N, int64_t K,
                        void* workspace, size_t workspace_bytes, void* stream);
TRI_API tri_status tri_gemm_tq1(const uint16_t* X, const uint8_t* qs, const uint16_t* d,
                        uint16_t* Y, int64_t M, int64_t N, int64_t K,
                        void* workspace, size_t workspace_bytes, void* stream);

/* ------------------------------------------------------------------------
 * Ternary GEMM without any caller-provided workspace (TQ2, 1 <= M <= 16).
 * The pages have no counterpart: this is a deployment variant of the
 * decode-regime kernel for callers that may not allocate device memory (for
 * example a plugin whose host framework owns every device allocation and
 * passes in only the call's tensors, or a real-time loop that must keep a
 * fixed, preallocated memory footprint).
 *   Same result and argument meaning as tri_gemm_tq2 for these shapes; the
 *   scratch the kernel needs lives in a static 8 MiB device array inside the
 *   library, held on every device that loads it until the process exits.
 *   Returns TRI_ERR_SHAPE for M > 16 and TRI_ERR_SCRATCH_LIMIT when the shape
 *   needs more scratch than that array holds (tri_gemm_tq2_noalloc_fits
 *   answers beforehand).  It allocates nothing: the first call on a device
 *   looks up the array's device address for that device (and may load the
 *   module), so make that call before any stream capture; a lookup that
 *   fails returns TRI_ERR_CUDA and is retried by the next call.  All calls
 *   on a device share the array and each clears what it needs cleared:
 *   calls that can run at the same time on that device (other streams,
 *   other host threads) race, so order them.
 * ---------------------------------------------------------------------- */
TRI_API tri_status tri_gemm_tq2_noalloc(const uint16_t* X, const uint8_t* qs, const uint16_t* d,
                                        uint16_t* Y, int64_t M, int64_t N, int64_t K,
                                        void* stream);
/* 1 if tri_gemm_tq2_noalloc accepts this shape on the current device, else 0. */
TRI_API int tri_gemm_tq2_noalloc_fits(int64_t M, int64_t N, int64_t K);

/* ------------------------------------------------------------------------
 * Fused gate/up projection with a SwiGLU epilogue: the gated feed-forward
 * unit of "Scaling Laws and Efficient Inference for Ternary Language
 * Models" (section "The model"; its MLP is a SwiGLU over two ternary
 * projections):
 *   Y[m][f] = silu(G[m][f]) * U[m][f],  silu(g) = g / (1 + e^-g),
 *   G = X (d_g W_hat_g)^T, U = X (d_u W_hat_u)^T, fp32 accumulation, fp16 Y.
 *   qs, d     the 2F rows of both packed weight matrices (format as in
 *             tri_gemm), interleaved in groups of eight rows: fused row
 *             16j + i is gate row 8j + i and fused row 16j + 8 + i is up row
 *             8j + i (i < 8).  F % 8 == 0.
 *   Y         device fp16[M][F], 16-byte aligned, written.
 *   workspace at least tri_gemm_swiglu_workspace_bytes(format, M, F, K).
 *   path      as in tri_gemm for the 2F-row product.  For 3 <= M <= 16 the
 *             integer kernel applies silu(g) * u to the fp32 sums in its
 *             epilogue; other paths write the [M][2F] product (fp16) into
 *             the workspace and a second kernel combines it.
 *   Errors as tri_gemm; F % 8 != 0 returns TRI_ERR_SHAPE.
 * ---------------------------------------------------------------------- */
TRI_API size_t tri_gemm_swiglu_workspace_bytes(int format, int64_t M, int64_t F, int64_t K);
TRI_API tri_status tri_gemm_swiglu(int format, int path, const uint16_t* X, const uint8_t* qs,
                                   const uint16_t* d, uint16_t* Y, int64_t M, int64_t F, int64_t K,
                                   void* workspace, size_t workspace_bytes, void* stream);

/* ------------------------------------------------------------------------
 * Device wait status.  The GEMM kernels wait on asynchronous copies, on the
 * tensor-core pipeline and on partial sums of other thread blocks; each such
 * wait gives up after an iteration limit far beyond any wait a healthy call
 * sees (a second or more).  A wait that gives up stores a non-zero code in a
 * 32-bit word the library keeps on each device (the first code stays until
 * cleared; later ones are dropped), lets the kernel drain and return, and
 * leaves that call's output unspecified.  Codes name the wait: 1-2 and 11
 * the decode kernels (M <= 2), 41-42 the integer kernel for 3 <= M <= 16,
 * 21-26 the tcgen05 kernel (M > 16), 90-91 tri_selftest_wait_timeout.
 *
 * tri_wait_status: reads the current device's word in `stream` order (after
 *   the work already enqueued there), zeroes it there if `clear` is
 *   non-zero, waits for the stream to finish (cudaStreamSynchronize) and
 *   stores the value read in *code (0 = no wait has given up since the last
 *   clear).  The one entry point that synchronizes the host.  Word reads and
 *   clears race with kernels of this library running on other streams.
 * tri_selftest_wait_timeout: enqueues on `stream` one kernel whose wait can
 *   never complete, through the same bounded routines the GEMM kernels use:
 *   which = 0 waits on an mbarrier phase nothing arrives on (code 90),
 *   which = 1 on a stamped word nothing writes (code 91; the word is the
 *   first 8 bytes of `scratch`, device memory, 8-byte aligned, zeroed by the
 *   call).  The wait runs out within about a second, records its code and
 *   returns; nothing faults.  It lets a caller check the detection path.
 * ---------------------------------------------------------------------- */
TRI_API tri_status tri_wait_status(uint32_t* code, int clear, void* stream);
TRI_API tri_status tri_selftest_wait_timeout(int which, void* scratch, void* stream);

/* Kernel that tri_gemm would launch for this call under TRI_PATH_AUTO
 * (one of tri_gemm_path), or -1 if the shape is invalid. */
TRI_API int tri_gemm_auto_path(int format, int64_t M, int64_t N, int64_t K);

/* ----------------------------------------------------------------------
 * One transformer-block decode step around the ternary layers
 * ("Scaling Laws and Efficient Inference for Ternary Language Models",
 * section "The model": LLaMA-style blocks with SwiGLU MLPs, rotary
 * embeddings with theta = 5e5, RMSNorm and QK-Norm, no biases; "Spectra:
 * ...", section "Architecture of TriLM and FloatLM": activations in 16-bit
 * floats).  The linear layers of the block are tri_gemm / tri_gemm_swiglu
 * calls; these entry points are the steps between them.  All tensors are
 * caller-owned device memory, fp16 unless stated, row-major, 16-byte
 * aligned (pos: 4, cs: 8); arithmetic is fp32 and each result is rounded
 * to fp16 once, where it is stored.  Head dimension 128 throughout.
 *
 * tri_rmsnorm: y[m] = h[m] / sqrt(mean(h[m]^2) + eps) * g, where h = x, or,
 *   when r is not NULL, h = x + r (each element the exact sum rounded once),
 *   which is also written to h_out (required then; it may not alias x or r).
 *   x, r, h_out, y: [M][D]; g: [D]; 8 <= D <= 2^20, D % 8 == 0, M >= 1,
 *   0 <= eps < 1e30.  y may alias x when r is NULL.
 * tri_rope_table: cs[p][i] = (cos, sin)(p * theta^(-2 i / dh)) as float
 *   pairs for p < Lmax, i < dh / 2, the angles computed in float64
 *   (rotate-half RoPE: pair i is (feature i, feature i + dh / 2)); dh = 128,
 *   1 <= Lmax <= 2^24, theta > 1.
 * tri_qknorm_rope: qkv [M][(H + 2 Hkv) * 128] is the fused QKV product
 *   (query heads, then key heads, then value heads).  Each query and key
 *   head is RMS-normalised over its 128 features with gain gq or gk ([128],
 *   shared by the heads) and rotated at position pos[m] with the table cs
 *   ([>= Lmax][64] float pairs); queries go to q_out [M][H][128], the key
 *   and the value (as given) to kcache / vcache [M][Hkv][Lmax][128] at
 *   position pos[m] (device int32 [M]).  A position outside [0, Lmax)
 *   writes nothing to the caches and leaves that q unspecified.  H % Hkv == 0.
 * tri_attention_decode: out[m][h] = softmax(K q[m][h] / sqrt(128)) V over
 *   positions 0..pos[m] of sequence m's caches, key/value head h / (H / Hkv)
 *   (grouped queries, H / Hkv <= 8); out: [M][H * 128].  max_len (host) is
 *   an upper bound of pos[m] + 1 over the batch, 1 <= max_len <= Lmax: it
 *   sizes the split over positions and the workspace
 *   (tri_attention_decode_workspace_bytes, 256-byte aligned, contents on
 *   entry irrelevant); a pos[m] + 1 above max_len is clamped to it.  Calls
 *   that share a workspace must be ordered.
 * Errors: TRI_ERR_INVALID_ARG (null pointer, eps or theta out of range,
 *   missing h_out), TRI_ERR_SHAPE, TRI_ERR_ALIGNMENT, TRI_ERR_WORKSPACE,
 *   TRI_ERR_CUDA; nothing traps.
 * ---------------------------------------------------------------------- */
TRI_API tri_status tri_rmsnorm(const uint16_t* x, const uint16_t* r, const uint16_t* g, uint16_t* h_out,
                               uint16_t* y, int64_t M, int64_t D, float eps, void* stream);
TRI_API tri_status tri_rope_table(float* cs, int64_t Lmax, int64_t dh, double theta, void* stream);
TRI_API tri_status tri_qknorm_rope(const uint16_t* qkv, const int32_t* pos, const uint16_t* gq,
                                   const uint16_t* gk, const float* cs, uint16_t* q_out, uint16_t* kcache,
                                   uint16_t* vcache, int64_t M, int64_t H, int64_t Hkv, int64_t Lmax,
                                   float eps, void* stream);
TRI_API size_t tri_attention_decode_workspace_bytes(int64_t M, int64_t H, int64_t Hkv, int64_t max_len);
TRI_API tri_status tri_attention_decode(const uint16_t* q, const uint16_t* kcache, const uint16_t* vcache,
                                        const int32_t* pos, uint16_t* out, int64_t M, int64_t H,
                                        int64_t Hkv, int64_t Lmax, int64_t max_len, void* workspace,
                                        size_t workspace_bytes, void* stream);

#ifdef __cplusplus
}
#endif
#endif /* TRI_B200_H */
