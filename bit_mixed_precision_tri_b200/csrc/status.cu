// The device wait status word and its self-test.
//
// Kernels that wait on work of other thread blocks or on asynchronous copies
// (mbarrier pipelines, split-K and stream-K reductions) bound every wait by
// an iteration limit.  A wait that runs out records a non-zero code here (the
// first one sticks), drains and returns: the call's output is then
// unspecified, but nothing traps and the context stays usable.  The word is
// per device (one copy per loaded module), looked up once per device with
// that device current; the host reads and clears it with tri_wait_status.
#include <mutex>

#include "sm100_ptx.cuh"
#include "tri_internal.cuh"

namespace tri {

static __device__ unsigned g_wait_status;

namespace {

constexpr int kMaxDev = 64;
unsigned* g_word[kMaxDev];
cudaError_t g_word_err[kMaxDev];
std::once_flag g_word_once[kMaxDev];

// One block of 32 threads waits on something nothing completes: an mbarrier
// phase no thread arrives on (which = 0) or a stamped word no block writes
// (which = 1), each through the bounded routine the GEMM kernels use, and
// records the code the kernels' own waits would.
__global__ void expire_wait_kernel(unsigned* word, const unsigned long long* never, int which,
                                   int limit) {
  __shared__ __align__(8) uint64_t bar;
  if (threadIdx.x == 0) {
    ptx::mbar_init(&bar, 1);
    ptx::fence_mbar_init();
  }
  __syncthreads();
  if (threadIdx.x != 0) return;
  if (which == 0) {
    if (!ptx::mbar_wait(&bar, 0, (uint32_t)limit)) ptx::record_wait_failure(word, kSelfTestMbarCode);
  } else {
    const unsigned long long x = ptx::wait_stamp(never, ptx::ld_relaxed_u64(never), 1u, limit);
    if ((unsigned)(x >> 32) != 1u) ptx::record_wait_failure(word, kSelfTestStampCode);
  }
}

}  // namespace

cudaError_t wait_status_word(unsigned** out) {
  int dev = -1;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDev) return cudaErrorInvalidDevice;
  std::call_once(g_word_once[dev], [dev]() {
    void* ptr = nullptr;
    g_word_err[dev] = cudaGetSymbolAddress(&ptr, g_wait_status);
    g_word[dev] = static_cast<unsigned*>(ptr);
  });
  if (g_word_err[dev] != cudaSuccess) return g_word_err[dev];
  *out = g_word[dev];
  return cudaSuccess;
}

cudaError_t read_wait_status(unsigned* code, bool clear, cudaStream_t s) {
  unsigned* w = nullptr;
  cudaError_t e = wait_status_word(&w);
  if (e != cudaSuccess) return e;
  // read (and clear) in the stream's order, then wait: the word seen is the
  // one left by the work enqueued on `s` before this call, and the clear is
  // complete before returning
  unsigned v = 0;
  e = cudaMemcpyAsync(&v, w, sizeof(unsigned), cudaMemcpyDeviceToHost, s);
  if (e == cudaSuccess && clear) e = cudaMemsetAsync(w, 0, sizeof(unsigned), s);
  const cudaError_t es = cudaStreamSynchronize(s);
  if (e == cudaSuccess) e = es;
  if (e == cudaSuccess) *code = v;
  return e;
}

cudaError_t launch_expire_wait(int which, void* scratch, cudaStream_t s) {
  unsigned* w = nullptr;
  cudaError_t e = wait_status_word(&w);
  if (e != cudaSuccess) return e;
  // the stamped word starts at zero, so stamp 1 never appears
  e = cudaMemsetAsync(scratch, 0, sizeof(unsigned long long), s);
  if (e != cudaSuccess) return e;
  // far shorter limits than the GEMM kernels' own (a poll of the stamp is a
  // 64 ns sleep plus an L2 round trip; an mbarrier poll suspends in hardware
  // for a while), so the self-test ends within a fraction of a second
  const int limit = which == 0 ? (1 << 12) : (1 << 18);
  expire_wait_kernel<<<1, 32, 0, s>>>(w, static_cast<const unsigned long long*>(scratch), which,
                                      limit);
  return cudaGetLastError();
}

}  // namespace tri
