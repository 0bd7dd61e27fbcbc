// Host <-> device staging of a decode step's query and output by kernels, for
// tw_decode_step_host.  A decode step moves a few KB each way (B x Hq x 128
// fp16); a copy-engine transfer of that size costs more than the copy itself
// and cuts the chain of programmatic dependent launches between the step's
// kernels.  These copies are ordinary kernels in that chain instead: they read
// or write page-locked host memory through its device mapping.
#include "tw_common.cuh"
#include "tw_kernels.h"

namespace tw {

constexpr int kCopyThreads = 256;
constexpr int kCopyPerThread = 4;   // 16-byte words in flight per thread

// dst[i] = src[i] for 16-byte words i < n16.  With `early`, the source words
// are loaded before the wait on the preceding kernel (the source is a host
// buffer that no kernel of the stream writes, so its read can overlap the
// previous kernel's tail); the stores always come after the wait, because the
// preceding kernels may still read dst (the step's query) or write src (the
// step's output, read only with early = 0).
__global__ void __launch_bounds__(kCopyThreads)
k_copy16(const uint4* src, uint4* dst, int64_t n16, int early) {
  const int64_t base = (int64_t)blockIdx.x * (kCopyThreads * kCopyPerThread) + threadIdx.x;
  uint4 v[kCopyPerThread];
  if (!early) griddep_wait();
#pragma unroll
  for (int k = 0; k < kCopyPerThread; ++k) {
    const int64_t i = base + (int64_t)k * kCopyThreads;
    if (i < n16) v[k] = src[i];
  }
  if (early) griddep_wait();
#pragma unroll
  for (int k = 0; k < kCopyPerThread; ++k) {
    const int64_t i = base + (int64_t)k * kCopyThreads;
    if (i < n16) dst[i] = v[k];
  }
  griddep_launch();
}

cudaError_t launch_copy16(const void* src, void* dst, int64_t bytes, bool early, cudaStream_t st,
                          bool pdl) {
  const int64_t n16 = bytes / 16;
  if (n16 <= 0) return cudaSuccess;
  const int64_t per = (int64_t)kCopyThreads * kCopyPerThread;
  const int64_t blocks = (n16 + per - 1) / per;
  if (blocks > 0x7FFFFFFF) return cudaErrorInvalidValue;
  return launch_k(k_copy16, dim3((unsigned)blocks), dim3(kCopyThreads), 0, st, pdl,
                  static_cast<const uint4*>(src), static_cast<uint4*>(dst), n16, early ? 1 : 0);
}

}  // namespace tw
