// Shared device helpers of the Twilight sm_100a kernels: KV-cache addressing for
// the contiguous and paged layouts, fp16 totalOrder keys, warp reductions.
#pragma once

#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace tw {

constexpr int kHeadDim = 128;
constexpr int kPage = 16;
constexpr int kGroup = 32;
constexpr int kGroups = kHeadDim / kGroup;

// Row addressing of one (sequence, KV head) in either layout.  A "row" is one
// token of one KV head: 128 fp16 of K or V, 128 * kbits / 8 B of codes (64 B
// at 4 bits, 32 B at 2 bits), 4 scales, 4 zeros.
struct Layout {
  int32_t B, Hk, N;                 // N = max_seq_len
  const int32_t* seq_lens;          // [B] or null
  const int32_t* page_table;        // [B][max_pages] or null
  int32_t max_pages;                // ceil(N / 16)
  int32_t pool_pages;               // paged: pages in the pool
  int32_t kbits;                    // key-cache width: 4 or 2 (host-side dispatch only)

  // Valid length of sequence b, clamped to [0, N] so that a bad length can
  // never address outside the cache.
  __device__ __forceinline__ int len(int b) const {
    const int l = seq_lens ? seq_lens[b] : N;
    return l < 0 ? 0 : (l > N ? N : l);
  }

  // Pool page of logical page pg; an id outside the pool reads pool page 0
  // instead of leaving the allocation.
  __device__ __forceinline__ int64_t pool_page(int b, int pg) const {
    const int p = page_table[(int64_t)b * max_pages + pg];
    return (unsigned)p < (unsigned)pool_pages ? p : 0;
  }

  // Global row index of token t of (b, h).
  __device__ __forceinline__ int64_t row(int b, int h, int t) const {
    if (page_table) return (pool_page(b, t >> 4) * Hk + h) * kPage + (t & 15);
    return ((int64_t)b * Hk + h) * N + t;
  }

  // Row index of the first token of logical page pg (tokens of a page are
  // consecutive rows in both layouts).
  __device__ __forceinline__ int64_t page_row(int b, int h, int pg) const {
    if (page_table) return (pool_page(b, pg) * Hk + h) * kPage;
    return ((int64_t)b * Hk + h) * N + (int64_t)pg * kPage;
  }

  // Index of the metadata record (2 x 128 fp16) of logical page pg.
  __device__ __forceinline__ int64_t meta_index(int b, int h, int pg) const {
    if (page_table) return pool_page(b, pg) * Hk + h;
    return ((int64_t)b * Hk + h) * max_pages + pg;
  }
};

// fp16 bits -> int key ordered like IEEE totalOrder on non-NaN values
// (-0 sorts just below +0).  The map is its own inverse on the low 16 bits.
__device__ __forceinline__ int h_key(uint32_t bits16) {
  const int s = (int)(int16_t)(uint16_t)bits16;
  return s ^ ((s >> 31) & 0x7FFF);
}
__device__ __forceinline__ uint32_t h_from_key(int key) {
  return (uint32_t)(uint16_t)(key ^ ((key >> 31) & 0x7FFF));
}

// fp32 -> uint32 key ordered like the float value, with -0 folded onto +0.
__device__ __forceinline__ uint32_t f_key(float f) {
  const uint32_t u = __float_as_uint(__fadd_rn(f, 0.0f));
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

template <typename T>
__device__ __forceinline__ T warp_sum(T v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}

// 16-byte global load that bypasses L1 allocation (streamed once).
__device__ __forceinline__ uint4 ld_stream16(const void* p) {
  uint4 r;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
               : "l"(p));
  return r;
}

__device__ __forceinline__ uint2 ld_stream8(const void* p) {
  uint2 r;
  asm volatile("ld.global.nc.L1::no_allocate.v2.u32 {%0,%1}, [%2];"
               : "=r"(r.x), "=r"(r.y)
               : "l"(p));
  return r;
}

// Programmatic dependent launch: wait until the preceding kernel in the stream
// has completed and its writes are visible (a no-op without the launch
// attribute), and let the next kernel begin launching.
__device__ __forceinline__ void griddep_wait() {
  asm volatile("griddepcontrol.wait;" ::: "memory");
}
__device__ __forceinline__ void griddep_launch() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

}  // namespace tw
