// Token-level label-channel base selector: a synthetic stand-in for Double
// Sparsity, the other base selector Twilight builds on ("Twilight: Adaptive
// Attention Sparsity with Hierarchical Top-p Pruning", atlas.scime.ai summary,
// "Builds on" and "Key results"; the pages give no mechanism, so this follows
// Double Sparsity's published idea).  Per KV head, r label channels (chosen by
// the caller; offline calibration on trained weights in the real method) are
// copied out of every key into a small label cache; at decode a token's score
// is q . k over those channels only, and the best min(budget, len) tokens of
// each (sequence, KV head) become the candidates that Twilight's top-p pruner
// then works on.
//
// The pruner itself is not re-implemented for token candidates: the candidate
// tokens' quantised key rows are gathered into a contiguous cache of B * Hk
// one-head "sequences" of up to cand_stride rows, on which the page-free
// estimate and top-p kernels run unchanged (the query tensor [B][Hq][128] is
// already [B * Hk][G][128] for that cache, and its selection sets have the
// same indices), and the kept positions are mapped back to token ids.
#include "tw_common.cuh"
#include "tw_label.h"
#include "tw_kernels.h"

namespace tw {

__device__ __forceinline__ int clamp_channel(int c) { return c < 0 ? 0 : (c > 127 ? 127 : c); }

// One warp per token row, lane j < r copies channel channels[h][j].
__global__ void __launch_bounds__(256)
k_label_cache(Layout L, const __half* __restrict__ K, const int32_t* __restrict__ channels, int r,
              __half* __restrict__ labels) {
  const int lane = threadIdx.x & 31;
  const int64_t total = (int64_t)L.B * L.Hk * L.N;
  const int64_t step = (int64_t)gridDim.x * (blockDim.x >> 5);
  for (int64_t i = (int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5); i < total;
       i += step) {
    const int t = (int)(i % L.N);
    const int64_t bh = i / L.N;
    const int h = (int)(bh % L.Hk);
    const int b = (int)(bh / L.Hk);
    if (t >= L.len(b)) continue;
    const int64_t row = L.row(b, h, t);
    if (lane < r)
      labels[row * r + lane] = K[row * kHeadDim + clamp_channel(channels[h * r + lane])];
  }
}

// Block (x = 256 tokens, y = unit u = b * Hk + h).  For each query head g of
// the group, s_g = sum over j = 0 .. r-1, in that order, of q_g[c_j] * label_j
// (products exact in fp32, each sum rounded); the score is s_0 + s_1 + ...
// added in head order.
__global__ void __launch_bounds__(256)
k_label_scores(Layout L, const __half* __restrict__ q, int Hq, const __half* __restrict__ labels,
               const int32_t* __restrict__ channels, int r, float* __restrict__ scores) {
  __shared__ float qs[kMaxLabelGroup][kMaxLabelChannels];
  const int u = blockIdx.y, b = u / L.Hk, h = u % L.Hk;
  const int G = Hq / L.Hk;
  for (int i = threadIdx.x; i < G * r; i += blockDim.x) {
    const int g = i / r, j = i % r;
    qs[g][j] = __half2float(
        q[((int64_t)b * Hq + h * G + g) * kHeadDim + clamp_channel(channels[h * r + j])]);
  }
  __syncthreads();
  const int t = blockIdx.x * blockDim.x + threadIdx.x;
  if (t >= L.len(b)) return;
  const __half* lr = labels + L.row(b, h, t) * r;
  float lv[kMaxLabelChannels];
#pragma unroll
  for (int j = 0; j < kMaxLabelChannels; ++j) lv[j] = j < r ? __half2float(lr[j]) : 0.f;
  float total = 0.f;
  for (int g = 0; g < G; ++g) {
    float s = 0.f;
#pragma unroll
    for (int j = 0; j < kMaxLabelChannels; ++j)
      if (j < r) s = __fadd_rn(s, __fmul_rn(qs[g][j], lv[j]));
    total = g == 0 ? s : __fadd_rn(total, s);
  }
  scores[(int64_t)u * L.N + t] = total;
}

constexpr int kTkThreads = 512;
constexpr int kTkWarps = kTkThreads / 32;
constexpr int kTkPer = 4;                      // consecutive tokens per thread in a compaction round
constexpr int kTkHistBins = 1 << 12;

// Exclusive scan of v over the block (thread order); *total gets the sum.
__device__ __forceinline__ uint32_t tk_excl_scan(uint32_t v, uint32_t* sh, uint32_t* total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  uint32_t incl = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const uint32_t x = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += x;
  }
  if (lane == 31) sh[warp] = incl;
  __syncthreads();
  if (warp == 0) {
    const uint32_t x = lane < kTkWarps ? sh[lane] : 0u;
    uint32_t xi = x;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const uint32_t y = __shfl_up_sync(0xffffffffu, xi, o);
      if (lane >= o) xi += y;
    }
    if (lane < kTkWarps) sh[lane] = xi - x;
    if (lane == 31) sh[kTkWarps] = xi;
  }
  __syncthreads();
  const uint32_t r = sh[warp] + incl - v;
  *total = sh[kTkWarps];
  __syncthreads();   // sh is reused by the next call
  return r;
}

// One block per unit: the K = min(budget, len) largest scores (keys ordered
// like the floats, -0 folded onto +0), ties to the lower token index, written
// as ascending token ids.  The K-th largest key is found digit by digit
// (12, 10, 10 bits) from histograms over the unit's scores; the tokens are
// then compacted in index order, 2048 per round.
__global__ void __launch_bounds__(kTkThreads)
k_token_topk(Layout L, const float* __restrict__ scores, int budget, int32_t* __restrict__ cand,
             int cand_stride, int32_t* __restrict__ ncand) {
  __shared__ uint32_t hist[kTkHistBins];
  __shared__ uint32_t scan_sh[kTkWarps + 1];
  __shared__ uint32_t sel_digit, sel_above;
  const int u = blockIdx.x, b = u / L.Hk, tid = threadIdx.x;
  const int len = L.len(b);
  const int K = min(budget, len);
  const float* sc = scores + (int64_t)u * L.N;
  int32_t* out = cand + (int64_t)u * cand_stride;
  if (tid == 0) ncand[u] = K;
  if (K <= 0) return;
  if (K == len) {   // every token
    for (int t = tid; t < len; t += kTkThreads) out[t] = t;
    return;
  }
  uint32_t prefix = 0, pmask = 0;
  uint32_t need = (uint32_t)K;   // keys still to take among those matching prefix, from the top
  const int shifts[3] = {20, 10, 0}, widths[3] = {12, 10, 10};
  for (int d = 0; d < 3; ++d) {
    const int sh = shifts[d], nb = 1 << widths[d];
    const uint32_t dmask = (uint32_t)nb - 1u;
    for (int i = tid; i < nb; i += kTkThreads) hist[i] = 0u;
    __syncthreads();
    for (int t = tid; t < len; t += kTkThreads) {
      const uint32_t key = f_key(sc[t]);
      if ((key & pmask) == prefix) atomicAdd(&hist[(key >> sh) & dmask], 1u);
    }
    __syncthreads();
    // thread j owns bins [nb - (j + 1) * per, nb - j * per), highest first
    const int per = nb / kTkThreads;
    const int top = nb - tid * per;
    uint32_t mine = 0;
    for (int k = 1; k <= per; ++k) mine += hist[top - k];
    uint32_t tot;
    const uint32_t above = tk_excl_scan(mine, scan_sh, &tot);
    if (above < need && need <= above + mine) {
      uint32_t acc = above;
      for (int k = 1; k <= per; ++k) {
        const uint32_t c = hist[top - k];
        if (acc + c >= need) {
          sel_digit = (uint32_t)(top - k);
          sel_above = acc;
          break;
        }
        acc += c;
      }
    }
    __syncthreads();
    prefix |= sel_digit << sh;
    pmask |= dmask << sh;
    need -= sel_above;
    __syncthreads();   // sel_* are rewritten by the next digit
  }
  // prefix is now the K-th largest key T; take every key > T and the first
  // `need` keys == T in token order
  const uint32_t T = prefix;
  uint32_t run_gt = 0, run_eq = 0;
  for (int base = 0; base < len; base += kTkThreads * kTkPer) {
    const int t0 = base + tid * kTkPer;
    uint32_t fl_gt = 0, fl_eq = 0;
#pragma unroll
    for (int k = 0; k < kTkPer; ++k) {
      if (t0 + k < len) {
        const uint32_t key = f_key(sc[t0 + k]);
        fl_gt |= (key > T ? 1u : 0u) << k;
        fl_eq |= (key == T ? 1u : 0u) << k;
      }
    }
    uint32_t tot_gt, tot_eq;
    const uint32_t ex_gt = tk_excl_scan((uint32_t)__popc(fl_gt), scan_sh, &tot_gt);
    const uint32_t ex_eq = tk_excl_scan((uint32_t)__popc(fl_eq), scan_sh, &tot_eq);
    uint32_t g = run_gt + ex_gt, e = run_eq + ex_eq;
#pragma unroll
    for (int k = 0; k < kTkPer; ++k) {
      if ((fl_gt >> k) & 1u) {
        out[g + min(e, need)] = t0 + k;
        ++g;
      } else if ((fl_eq >> k) & 1u) {
        if (e < need) out[g + e] = t0 + k;
        ++e;
      }
    }
    run_gt += tot_gt;
    run_eq += tot_eq;
  }
}

// One thread per (unit, candidate): copy the candidate token's code row,
// scales and zeros to row u * cand_stride + i of the contiguous cache.  A
// token id outside [0, len) reads row min(max(id, 0), len - 1) instead.
template <int ROWB>
__global__ void __launch_bounds__(256)
k_gather_keys(Layout L, const int32_t* __restrict__ cand, int cand_stride,
              const int32_t* __restrict__ ncand, const uint8_t* __restrict__ codes,
              const __half* __restrict__ scales, const __half* __restrict__ zeros,
              uint8_t* __restrict__ vcodes, __half* __restrict__ vscales,
              __half* __restrict__ vzeros) {
  const int64_t total = (int64_t)L.B * L.Hk * cand_stride;
  const int64_t step = (int64_t)gridDim.x * blockDim.x;
  for (int64_t x = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; x < total; x += step) {
    const int i = (int)(x % cand_stride);
    const int u = (int)(x / cand_stride);
    const int b = u / L.Hk, h = u % L.Hk;
    const int len = L.len(b);
    if (len <= 0 || i >= min(ncand[u], cand_stride)) continue;
    const int t = min(max(cand[x], 0), len - 1);
    const int64_t src = L.row(b, h, t);
    const uint4* cs = reinterpret_cast<const uint4*>(codes + src * ROWB);
    uint4* cd = reinterpret_cast<uint4*>(vcodes + x * ROWB);
#pragma unroll
    for (int k = 0; k < ROWB / 16; ++k) cd[k] = cs[k];
    *reinterpret_cast<uint2*>(vscales + x * kGroups) =
        *reinterpret_cast<const uint2*>(scales + src * kGroups);
    *reinterpret_cast<uint2*>(vzeros + x * kGroups) =
        *reinterpret_cast<const uint2*>(zeros + src * kGroups);
  }
}

// Block per set: kept positions of the contiguous cache -> token ids.
__global__ void __launch_bounds__(256)
k_map_tokens(int G, int group_sets, const int32_t* __restrict__ cand, int cand_stride,
             int32_t* __restrict__ idx, int icap, const int32_t* __restrict__ count) {
  const int s = blockIdx.x;
  const int u = group_sets ? s : s / G;
  const int n = min(max(count[s], 0), icap);
  int32_t* row = idx + (int64_t)s * icap;
  const int32_t* cu = cand + (int64_t)u * cand_stride;
  for (int i = threadIdx.x; i < n; i += blockDim.x) {
    const int v = row[i];
    row[i] = cu[min(max(v, 0), cand_stride - 1)];
  }
}

static int grid_for(int64_t items, int per_block, int num_sms) {
  const int64_t want = (items + per_block - 1) / per_block;
  const int64_t cap = (int64_t)num_sms * 8;
  return (int)(want < 1 ? 1 : (want < cap ? want : cap));
}

cudaError_t launch_label_cache(const Layout& L, const __half* K, const int32_t* channels, int r,
                               __half* labels, cudaStream_t st, int num_sms) {
  k_label_cache<<<grid_for((int64_t)L.B * L.Hk * L.N, 8, num_sms), 256, 0, st>>>(L, K, channels,
                                                                                 r, labels);
  return cudaGetLastError();
}

cudaError_t launch_label_scores(const Layout& L, const __half* q, int Hq, const __half* labels,
                                const int32_t* channels, int r, float* scores, cudaStream_t st) {
  const dim3 grid((unsigned)((L.N + 255) / 256), (unsigned)(L.B * L.Hk));
  if (grid.x == 0 || grid.y == 0) return cudaSuccess;
  k_label_scores<<<grid, 256, 0, st>>>(L, q, Hq, labels, channels, r, scores);
  return cudaGetLastError();
}

cudaError_t launch_token_topk(const Layout& L, const float* scores, int budget, int32_t* cand,
                              int cand_stride, int32_t* ncand, cudaStream_t st) {
  if (L.B * L.Hk == 0) return cudaSuccess;
  k_token_topk<<<L.B * L.Hk, kTkThreads, 0, st>>>(L, scores, budget, cand, cand_stride, ncand);
  return cudaGetLastError();
}

cudaError_t launch_gather_keys(const Layout& L, const int32_t* cand, int cand_stride,
                               const int32_t* ncand, const uint8_t* codes, const __half* scales,
                               const __half* zeros, uint8_t* vcodes, __half* vscales,
                               __half* vzeros, cudaStream_t st, int num_sms) {
  const int grid = grid_for((int64_t)L.B * L.Hk * cand_stride, 256, num_sms);
  if (L.kbits == 2)
    k_gather_keys<32><<<grid, 256, 0, st>>>(L, cand, cand_stride, ncand, codes, scales, zeros,
                                            vcodes, vscales, vzeros);
  else
    k_gather_keys<64><<<grid, 256, 0, st>>>(L, cand, cand_stride, ncand, codes, scales, zeros,
                                            vcodes, vscales, vzeros);
  return cudaGetLastError();
}

cudaError_t launch_map_tokens(int nsets, int G, int group_sets, const int32_t* cand,
                              int cand_stride, int32_t* idx, int icap, const int32_t* count,
                              cudaStream_t st) {
  if (nsets <= 0) return cudaSuccess;
  k_map_tokens<<<nsets, 256, 0, st>>>(G, group_sets, cand, cand_stride, idx, icap, count);
  return cudaGetLastError();
}

}  // namespace tw
