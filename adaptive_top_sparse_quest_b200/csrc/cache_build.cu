// Cache-build kernels (prefill time, once per token): the quantised key cache
// and the Quest page metadata.
//
// Key cache: Twilight estimates attention weights from INT4 keys
// (atlas.scime.ai summary of "Twilight: Adaptive Attention Sparsity with
// Hierarchical Top-p Pruning", "Approach"); the 2-bit width its quantisation
// ablation compares against (table of measured effects) is built by the same
// kernels with 3 levels instead of 15.  Quest page metadata: per-page
// channel-wise key min / max, the layout Quest's page selection works on
// ("Surprising findings").
//
// Both kernels stream K once with 16-byte loads; one half-warp owns one token
// row (or one page), lane l owns channels 8l..8l+7, so a group of 32 channels
// is 4 adjacent lanes and its min / max needs two xor-shuffles.  The decode-
// time append kernel applies the same row quantisation to each sequence's
// newest token and folds that row into its page's min / max.
#include "tw_common.cuh"
#include "tw_kernels.h"

namespace tw {

// Quantise one token row held by a half-warp (lane l16 holds channels
// 8 l16 .. 8 l16 + 7 in `raw`) to BITS-bit codes (levels 0 .. 2^BITS - 1) and
// store its codes, scales and zeros at `row`.  Every value is a fixed sequence
// of IEEE round-to-nearest operations, so it is bit-exact with the CPU
// definition.  Code j of the lane sits at bits BITS * j of its 4 (BITS = 4) or
// 2 (BITS = 2) bytes: channel c at bits BITS * (c % (8 / BITS)) of byte
// c / (8 / BITS).
template <int BITS>
__device__ __forceinline__ void quantize_row(const uint4 raw, int64_t row, int lane,
                                             unsigned hmask, uint8_t* __restrict__ codes,
                                             __half* __restrict__ scales,
                                             __half* __restrict__ zeros) {
  static_assert(BITS == 4 || BITS == 2, "key-cache width");
  constexpr int kLevels = (1 << BITS) - 1;
  const int l16 = lane & 15;
  const uint32_t w[4] = {raw.x, raw.y, raw.z, raw.w};
  int kmin = 0x7FFFFFFF, kmax = -0x7FFFFFFF - 1;
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    const int kk = h_key((w[j >> 1] >> (16 * (j & 1))) & 0xFFFFu);
    kmin = min(kmin, kk);
    kmax = max(kmax, kk);
  }
#pragma unroll
  for (int o = 1; o <= 2; o <<= 1) {
    kmin = min(kmin, __shfl_xor_sync(hmask, kmin, o));
    kmax = max(kmax, __shfl_xor_sync(hmask, kmax, o));
  }
  const uint32_t mn_bits = h_from_key(kmin);
  const uint32_t mx_bits = h_from_key(kmax);
  const float mnf = __half2float(__ushort_as_half((unsigned short)mn_bits));
  const float mxf = __half2float(__ushort_as_half((unsigned short)mx_bits));
  const float s32 = __fdiv_rn(__fsub_rn(mxf, mnf), (float)kLevels);
  const __half sc = __float2half_rn(s32);
  const float scf = __half2float(sc);
  uint32_t packed = 0;
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    const float x =
        __half2float(__ushort_as_half((unsigned short)((w[j >> 1] >> (16 * (j & 1))) & 0xFFFFu)));
    int c = 0;
    if (scf != 0.0f) {
      c = __float2int_rn(__fdiv_rn(__fsub_rn(x, mnf), scf));
      c = min(max(c, 0), kLevels);
    }
    packed |= (uint32_t)c << (BITS * j);
  }
  if (BITS == 4)
    *reinterpret_cast<uint32_t*>(codes + row * (kHeadDim / 2) + l16 * 4) = packed;
  else
    *reinterpret_cast<uint16_t*>(codes + row * (kHeadDim / 4) + l16 * 2) = (uint16_t)packed;
  // gather the 4 groups' scale / zero to lane 0 of the half-warp: one 8-byte store each
  const uint32_t sc_bits = __half_as_ushort(sc);
  const int base = lane & 16;
  uint32_t s[4], z[4];
#pragma unroll
  for (int g = 0; g < 4; ++g) {
    s[g] = __shfl_sync(hmask, sc_bits, base + 4 * g);
    z[g] = __shfl_sync(hmask, mn_bits, base + 4 * g);
  }
  if (l16 == 0) {
    *reinterpret_cast<uint2*>(scales + row * kGroups) =
        make_uint2(s[0] | (s[1] << 16), s[2] | (s[3] << 16));
    *reinterpret_cast<uint2*>(zeros + row * kGroups) =
        make_uint2(z[0] | (z[1] << 16), z[2] | (z[3] << 16));
  }
}

template <int BITS>
__global__ void __launch_bounds__(256)
k_quantize_keys(Layout L, const __half* __restrict__ K, uint8_t* __restrict__ codes,
                __half* __restrict__ scales, __half* __restrict__ zeros) {
  const int lane = threadIdx.x & 31;
  const int l16 = lane & 15;
  const unsigned hmask = 0xFFFFu << (lane & 16);
  const int64_t total = (int64_t)L.B * L.Hk * L.N;
  const int64_t step = (int64_t)gridDim.x * (blockDim.x >> 4);
  for (int64_t i = (int64_t)blockIdx.x * (blockDim.x >> 4) + (threadIdx.x >> 4); i < total;
       i += step) {
    const int t = (int)(i % L.N);
    const int64_t bh = i / L.N;
    const int h = (int)(bh % L.Hk);
    const int b = (int)(bh / L.Hk);
    if (t >= L.len(b)) continue;  // uniform across the half-warp
    const int64_t row = L.row(b, h, t);
    quantize_row<BITS>(ld_stream16(K + row * kHeadDim + l16 * 8), row, lane, hmask, codes,
                       scales, zeros);
  }
}

// Incremental decode append: for every sequence b with len_b >= 1 and every
// KV head, quantise the newest token t = len_b - 1 and fold it into the
// metadata of its page (a page starting at t holds only t).  With the cache
// current for the lengths minus one, the result equals a rebuild for the new
// lengths bit for bit: quantisation is per row, and exact fp16 min / max of
// a page's valid rows may be taken one row at a time.
template <int BITS>
__global__ void __launch_bounds__(256)
k_append_keys(Layout L, const __half* __restrict__ K, uint8_t* __restrict__ codes,
              __half* __restrict__ scales, __half* __restrict__ zeros, __half* __restrict__ meta) {
  const int lane = threadIdx.x & 31;
  const int l16 = lane & 15;
  const unsigned hmask = 0xFFFFu << (lane & 16);
  const int64_t total = (int64_t)L.B * L.Hk;
  const int64_t step = (int64_t)gridDim.x * (blockDim.x >> 4);
  griddep_wait();
  for (int64_t i = (int64_t)blockIdx.x * (blockDim.x >> 4) + (threadIdx.x >> 4); i < total;
       i += step) {
    const int h = (int)(i % L.Hk);
    const int b = (int)(i / L.Hk);
    const int t = L.len(b) - 1;
    if (t < 0) continue;  // uniform across the half-warp
    const int64_t row = L.row(b, h, t);
    const uint4 raw = *reinterpret_cast<const uint4*>(K + row * kHeadDim + l16 * 8);
    if (codes) quantize_row<BITS>(raw, row, lane, hmask, codes, scales, zeros);
    if (meta) {
      __half* dst = meta + L.meta_index(b, h, t / kPage) * (2 * kHeadDim) + l16 * 8;
      const uint32_t w[4] = {raw.x, raw.y, raw.z, raw.w};
      uint32_t mn[4], mx[4];
      if (t % kPage == 0) {   // the page's first row
#pragma unroll
        for (int j = 0; j < 4; ++j) mn[j] = mx[j] = w[j];
      } else {
        const uint4 omn = *reinterpret_cast<const uint4*>(dst);
        const uint4 omx = *reinterpret_cast<const uint4*>(dst + kHeadDim);
        const uint32_t on[4] = {omn.x, omn.y, omn.z, omn.w};
        const uint32_t ox[4] = {omx.x, omx.y, omx.z, omx.w};
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          uint32_t a = 0, c = 0;
#pragma unroll
          for (int e = 0; e < 2; ++e) {
            const int kx = h_key((w[j] >> (16 * e)) & 0xFFFFu);
            const int kn = min(h_key((on[j] >> (16 * e)) & 0xFFFFu), kx);
            const int km = max(h_key((ox[j] >> (16 * e)) & 0xFFFFu), kx);
            a |= h_from_key(kn) << (16 * e);
            c |= h_from_key(km) << (16 * e);
          }
          mn[j] = a;
          mx[j] = c;
        }
      }
      *reinterpret_cast<uint4*>(dst) = make_uint4(mn[0], mn[1], mn[2], mn[3]);
      *reinterpret_cast<uint4*>(dst + kHeadDim) = make_uint4(mx[0], mx[1], mx[2], mx[3]);
    }
  }
  griddep_launch();
}

__global__ void __launch_bounds__(256)
k_page_meta(Layout L, const __half* __restrict__ K, __half* __restrict__ meta) {
  const int l16 = threadIdx.x & 15;
  const int64_t total = (int64_t)L.B * L.Hk * L.max_pages;
  const int64_t step = (int64_t)gridDim.x * (blockDim.x >> 4);
  for (int64_t i = (int64_t)blockIdx.x * (blockDim.x >> 4) + (threadIdx.x >> 4); i < total;
       i += step) {
    const int pg = (int)(i % L.max_pages);
    const int64_t bh = i / L.max_pages;
    const int h = (int)(bh % L.Hk);
    const int b = (int)(bh / L.Hk);
    const int n = min(kPage, L.len(b) - pg * kPage);
    if (n <= 0) continue;
    const int64_t row0 = L.page_row(b, h, pg);
    const __half* src = K + row0 * kHeadDim + l16 * 8;
    uint4 raw[kPage];
#pragma unroll
    for (int r = 0; r < kPage; ++r)
      if (r < n) raw[r] = ld_stream16(src + (int64_t)r * kHeadDim);
    int kmin[8], kmax[8];
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      kmin[j] = 0x7FFFFFFF;
      kmax[j] = -0x7FFFFFFF - 1;
    }
#pragma unroll
    for (int r = 0; r < kPage; ++r) {
      if (r < n) {
        const uint32_t w[4] = {raw[r].x, raw[r].y, raw[r].z, raw[r].w};
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          const int kk = h_key((w[j >> 1] >> (16 * (j & 1))) & 0xFFFFu);
          kmin[j] = min(kmin[j], kk);
          kmax[j] = max(kmax[j], kk);
        }
      }
    }
    uint32_t mn[4], mx[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      mn[j] = h_from_key(kmin[2 * j]) | (h_from_key(kmin[2 * j + 1]) << 16);
      mx[j] = h_from_key(kmax[2 * j]) | (h_from_key(kmax[2 * j + 1]) << 16);
    }
    __half* dst = meta + L.meta_index(b, h, pg) * (2 * kHeadDim) + l16 * 8;
    *reinterpret_cast<uint4*>(dst) = make_uint4(mn[0], mn[1], mn[2], mn[3]);
    *reinterpret_cast<uint4*>(dst + kHeadDim) = make_uint4(mx[0], mx[1], mx[2], mx[3]);
  }
}

void launch_quantize_keys(const Layout& L, const __half* K, uint8_t* codes, __half* scales,
                          __half* zeros, cudaStream_t st, int num_sms) {
  const int64_t rows = (int64_t)L.B * L.Hk * L.N;
  const int64_t want = (rows + 15) / 16;
  const int64_t cap_blocks = (int64_t)num_sms * 8;
  const int blocks = (int)(want < 1 ? 1 : (want < cap_blocks ? want : cap_blocks));
  if (L.kbits == 2)
    k_quantize_keys<2><<<blocks, 256, 0, st>>>(L, K, codes, scales, zeros);
  else
    k_quantize_keys<4><<<blocks, 256, 0, st>>>(L, K, codes, scales, zeros);
}

cudaError_t launch_append_keys(const Layout& L, const __half* K, uint8_t* codes, __half* scales,
                               __half* zeros, __half* meta, cudaStream_t st, int num_sms,
                               bool pdl) {
  const int64_t units = (int64_t)L.B * L.Hk;
  const int64_t want = (units + 15) / 16;
  const int64_t cap_blocks = (int64_t)num_sms * 8;
  const int blocks = (int)(want < 1 ? 1 : (want < cap_blocks ? want : cap_blocks));
  return launch_k(L.kbits == 2 ? k_append_keys<2> : k_append_keys<4>, dim3(blocks), dim3(256), 0,
                  st, pdl, L, K, codes, scales, zeros, meta);
}

void launch_page_meta(const Layout& L, const __half* K, __half* meta, cudaStream_t st,
                      int num_sms) {
  const int64_t pages = (int64_t)L.B * L.Hk * L.max_pages;
  const int64_t want = (pages + 15) / 16;
  const int64_t cap_blocks = (int64_t)num_sms * 8;
  const int blocks = (int)(want < 1 ? 1 : (want < cap_blocks ? want : cap_blocks));
  k_page_meta<<<blocks, 256, 0, st>>>(L, K, meta);
}

}  // namespace tw
