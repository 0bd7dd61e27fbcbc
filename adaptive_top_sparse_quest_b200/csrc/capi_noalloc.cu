// tw_topp_prune_noalloc: the top-p pruner for callers that cannot allocate
// device memory (declared in include/twilight.h).
//
// Some callers have no way to hand the library a workspace: a runtime that
// records the decode step into a CUDA graph and forbids allocation while it
// records, a plugin whose enqueue hook may not allocate, or an embedded
// server that fixes its device memory at start-up.  This entry point takes the
// same inputs and outputs as tw_topp_prune but keeps its scratch (a status
// word and the selection sets' logits) in one fixed array compiled into the
// library.
//
// The array lives in device memory on every GPU that loads the library, for
// the life of the process.  In host code its name stands for a host-side
// placeholder, not a device address, so the first call on each device asks the
// runtime for the array's device address with that device current and reuses
// it afterwards.  That first call should therefore happen before any stream
// capture, and the cached address is valid for the life of the device's
// primary context (a cudaDeviceReset between calls would leave it stale).
// All calls share the array, so calls whose work overlaps on the GPU
// (different streams, or different host threads) race on it; the array keeps
// whatever the last call left in it, and nothing in it needs to start at zero
// because every byte this call reads was written by the same call (the
// status word is only ever or-ed into).
#include <atomic>

#include "twilight.h"
#include "tw_kernels.h"

namespace {

static __device__ __align__(256) unsigned char tw_noalloc_scratch[TW_NOALLOC_SCRATCH_BYTES];

std::atomic<void*> g_scratch_addr[128];

// Device address of tw_noalloc_scratch on the current device (looked up once per device).
void* scratch_address(int* status) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess || dev < 0 || dev >= 128) {
    *status = e != cudaSuccess ? TW_ERR_CUDA : TW_ERR_UNSUPPORTED;
    return nullptr;
  }
  void* p = g_scratch_addr[dev].load(std::memory_order_acquire);
  if (p == nullptr) {
    e = cudaGetSymbolAddress(&p, tw_noalloc_scratch);
    if (e != cudaSuccess || p == nullptr) {
      *status = TW_ERR_CUDA;
      return nullptr;
    }
    g_scratch_addr[dev].store(p, std::memory_order_release);
  }
  *status = TW_OK;
  return p;
}

}  // namespace

extern "C" int tw_topp_prune_noalloc(const uint16_t* q, int32_t num_q_heads, const tw_kv* kv,
                                     const uint8_t* codes, const uint16_t* scales,
                                     const uint16_t* zeros, const int32_t* cand_pages,
                                     int32_t cand_stride, const int32_t* ncand, double p,
                                     int32_t group_mode, int32_t* idx, int32_t capacity,
                                     int32_t* count, void* stream) {
  if (kv == nullptr) return TW_ERR_INVALID_ARG;
  // a request whose scratch does not fit is rejected before any device work:
  // tw_topp_prune checks the bytes it needs against the size given here
  int status = TW_OK;
  if (kv->batch == 0)
    return tw_topp_prune(q, num_q_heads, kv, codes, scales, zeros, cand_pages, cand_stride, ncand,
                         p, group_mode, idx, capacity, count, nullptr, 0, stream);
  void* ws = scratch_address(&status);
  if (status != TW_OK) return status;
  return tw_topp_prune(q, num_q_heads, kv, codes, scales, zeros, cand_pages, cand_stride, ncand, p,
                       group_mode, idx, capacity, count, ws, TW_NOALLOC_SCRATCH_BYTES, stream);
}
