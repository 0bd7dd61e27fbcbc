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

constexpr int kPartStride = 132;     // floats per split record: m, l, 2 pad, acc[128]
constexpr int kPartAcc = 4;
constexpr int kTargetSms = 148;      // B200 SM count used to size decode splits
constexpr int kMaxSetCandidates = 16 * 512 * 16;  // cluster of 16 CTAs x 512 pages x 16 tokens
constexpr uint32_t kNoRow = 0xFFFFFFFFu;           // physical row list: "no token here"

void launch_quantize_keys(const Layout& L, const __half* K, uint8_t* codes, __half* scales,
                          __half* zeros, cudaStream_t st, int num_sms);
void launch_page_meta(const Layout& L, const __half* K, __half* meta, cudaStream_t st,
                      int num_sms);
cudaError_t launch_append_keys(const Layout& L, const __half* K, uint8_t* codes, __half* scales,
                               __half* zeros, __half* meta, cudaStream_t st, int num_sms,
                               bool pdl);
// Selection stages on one thread-block cluster per (sequence, KV head) unit
// (select_prune.cu): phase 1 = Quest page scores + top-K_p pages, phase 2 =
// quantised-key weight estimate + top-p threshold + compaction.
constexpr int kSpThreads = 256;
constexpr int kSpMaxStages = 8;          // ring stages per phase (upper bound)
constexpr int kSpSharePages = 512;       // candidate pages one CTA estimates (8192 tokens)
constexpr int kSpMaxCluster = 16;
constexpr int kSpKeysCap = 8192;         // pages whose score keys a CTA keeps in shared memory
constexpr int kSpLogitsSmem = 32 * 1024; // a share's logits stay in shared memory up to this size
constexpr int kSpMaxSmem = 227 * 1024;

struct SpArgs {
  Layout L;
  const __half* q;
  int Hq;
  // phase 1 (meta == null: no selection; the candidates are cand / ncand, or every page)
  const __half* meta;
  int budget_pages;
  int32_t* cand;            // [B*Hk][cand_stride] logical page ids (written by phase 1)
  int cand_stride;
  int32_t* ncand;           // [B*Hk]
  uint32_t* gkeys;          // [B*Hk][max_pages] score keys when they exceed shared memory
  // phase 2 (codes == null: no pruning)
  const uint8_t* codes;
  const __half* scales;
  const __half* zeros;
  int group_sets;           // 1: one set per KV unit (group mode or G == 1)
  double p;
  int32_t* idx;             // [sets][icap] kept token ids, ascending
  uint32_t* rows;           // [sets][icap] their physical K/V rows (or null)
  int icap;
  int32_t* count;           // [sets]
  int32_t* done;            // [sets] attention completion counters to reset (or null)
  float* glogits;           // [B*Hk][G][lcap] when a share's logits exceed shared memory
  int lcap;
  int* status;              // device status word (bounded waits that gave up)
  int s1, s2;               // ring stages of the two phases
  int share_cap;            // candidate pages per CTA share (shared-memory logits stride / 16)
};

struct SpShape {
  int cs, share_cap, s1, s2;
  bool keys_in_smem, logits_in_smem;
  size_t smem;
};

cudaError_t launch_wait_selftest(int* status, cudaStream_t st);

// Launch the selection stages (shape chosen from the sizes and the device):
// sel_pages = candidate pages per unit at most.  a.gkeys / a.glogits point to
// workspace regions, used only when the keys / logits exceed shared memory.
cudaError_t launch_select_prune(const SpArgs& a, int sel_pages, int num_sms, cudaStream_t st,
                                bool pdl);
int select_prune_max_pages();

constexpr int kDecCtas = 4 * kTargetSms;   // CTAs sharing the concatenated selected tokens
size_t decode_part_floats(int B, int Hq, int Hk);
cudaError_t launch_sparse_decode(const Layout& L, const __half* q, int Hq, int group_sets,
                                 const __half* K, const __half* V, const uint32_t* rows, int icap,
                                 const int32_t* count, float* part, int32_t* done, __half* out,
                                 float* lse, cudaStream_t st, bool pdl);
cudaError_t launch_copy16(const void* src, void* dst, int64_t bytes, bool early, cudaStream_t st,
                          bool pdl);
cudaError_t launch_resolve_rows(const Layout& L, int Hq, int group_sets, const int32_t* idx,
                                int icap, const int32_t* count, uint32_t* rows, cudaStream_t st,
                                bool pdl);

}  // namespace tw
