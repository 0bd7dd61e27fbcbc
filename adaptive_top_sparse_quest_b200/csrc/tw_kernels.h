// Internal launch interface between the C ABI (capi.cu) and the kernels.
#pragma once

#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <atomic>
#include <utility>

#include "tw_common.cuh"

namespace tw {

// Launch with an optional programmatic-stream-serialization attribute (PDL):
// the kernel may start while its predecessor drains; it calls griddep_wait()
// before touching anything the predecessor writes.
template <typename... KArgs, typename... Args>
cudaError_t launch_k(void (*k)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st,
                     bool pdl, Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = pdl ? 1 : 0;
  return cudaLaunchKernelEx(&cfg, k, std::forward<Args>(args)...);
}

// Kernel attributes such as the dynamic shared-memory limit are per device:
// run `set` once on each device the process launches on (a repeated call from
// a racing thread only sets the same value again).
constexpr int kMaxDevices = 64;
template <typename F>
inline cudaError_t once_per_device(std::atomic<int> (&done)[kMaxDevices], F&& set) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return set();
  if (done[dev].load(std::memory_order_acquire)) return cudaSuccess;
  e = set();
  if (e == cudaSuccess) done[dev].store(1, std::memory_order_release);
  return e;
}

constexpr int kEstTile = 256;        // candidates per estimate work item
constexpr int kStatSpan = 32;        // candidates per softmax-statistics record
constexpr int kPartStride = 132;     // floats per split record: m, l, 2 pad, acc[128]
constexpr int kPartAcc = 4;
constexpr int kTargetSms = 148;      // B200 SM count used to size decode splits
constexpr int kMaxSetCandidates = 8 * 512 * 32;   // cluster of 8 x 512 threads x 32 weights
constexpr uint32_t kNoRow = 0xFFFFFFFFu;           // physical row list: "no token here"

void launch_quantize_keys(const Layout& L, const __half* K, uint8_t* codes, __half* scales,
                          __half* zeros, cudaStream_t st, int num_sms);
void launch_page_meta(const Layout& L, const __half* K, __half* meta, cudaStream_t st,
                      int num_sms);
cudaError_t launch_append_keys(const Layout& L, const __half* K, uint8_t* codes, __half* scales,
                               __half* zeros, __half* meta, cudaStream_t st, int num_sms,
                               bool pdl);
cudaError_t launch_estimate(const Layout& L, const __half* q, int Hq, const uint8_t* codes,
                            const __half* scales, const __half* zeros, const int32_t* cand,
                            int cand_stride, const int32_t* ncand, const uint32_t* row0,
                            int lcap, int cmax, float* logits, float2* stats, cudaStream_t st,
                            int num_sms, bool pdl);
int topp_shape(int cmax, int sets, int* R, int* CS);
cudaError_t launch_topp(const Layout& L, int Hq, int group_sets, const int32_t* cand,
                        int cand_stride, const int32_t* ncand, const uint32_t* row0, int lcap,
                        int cmax, const float* logits, const float2* stats, double p,
                        int32_t* idx, uint32_t* rows, int icap, int32_t* count, int32_t* done,
                        cudaStream_t st, bool pdl);
constexpr int kDecCtas = 4 * kTargetSms;   // CTAs sharing the concatenated selected tokens
size_t decode_part_floats(int B, int Hq, int Hk);
cudaError_t launch_sparse_decode(const Layout& L, const __half* q, int Hq, int group_sets,
                                 const __half* K, const __half* V, const uint32_t* rows, int icap,
                                 const int32_t* count, float* part, int32_t* done, __half* out,
                                 float* lse, cudaStream_t st, bool pdl);
cudaError_t launch_page_scores(const Layout& L, const __half* q, int Hq, const __half* meta,
                               float* scores, cudaStream_t st, int num_sms, bool pdl);
cudaError_t launch_page_topk(const Layout& L, const float* scores, int budget_pages,
                             int32_t* cand, int cand_stride, int32_t* ncand, uint32_t* row0,
                             cudaStream_t st, bool pdl);
cudaError_t launch_resolve_pages(const Layout& L, const int32_t* cand, int cand_stride,
                                 uint32_t* row0, cudaStream_t st, bool pdl);
cudaError_t launch_copy16(const void* src, void* dst, int64_t bytes, bool early, cudaStream_t st,
                          bool pdl);
cudaError_t launch_resolve_rows(const Layout& L, int Hq, int group_sets, const int32_t* idx,
                                int icap, const int32_t* count, uint32_t* rows, cudaStream_t st,
                                bool pdl);

}  // namespace tw
