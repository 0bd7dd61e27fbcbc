// Twilight's top-p pruner: INT4 weight estimation with fused softmax statistics,
// then the top-p threshold search and the index compaction.
//
// Method ("Twilight: Adaptive Attention Sparsity with Hierarchical Top-p
// Pruning", atlas.scime.ai summary, "Approach"): the attention weights of the
// candidates chosen by the base selector are estimated from a 4-bit key cache,
// and top-p (nucleus) thresholding keeps the smallest set whose weight reaches
// p; under GQA the budget is per KV group ("Limitations").
//
// k_estimate  (HBM-bound): one block per (b, kv head, 256-candidate tile).  4
//   threads per candidate, one per 32-channel group: 16 B of codes + the
//   group's fp16 scale / zero, k_hat = zero + scale * code in fp32, dot with
//   every query head of the group (q staged in shared memory), xor-shuffle
//   over the 4 groups.  Writes fp32 logits [kv unit][cap][G] and the tile's
//   per-head (max, sum exp) so the next kernel needs no extra pass.
// k_topp  (on-chip): one thread-block cluster per selection set.  The set's
//   weights live in registers across the cluster (R per thread).  The
//   threshold is the largest fp32 weight value theta whose retained mass
//   sum_{w >= theta} w reaches p.  Weights are non-negative, so their fp32 bit
//   patterns order like their values and theta is found most-significant
//   digit first, 8 bits per step (4 steps instead of the 31 of a bisection),
//   with each step's per-digit masses summed over the cluster through
//   distributed shared memory.  Masses are exact integers (weights truncated
//   to multiples of 2^-40) so the sums are order independent.  Every weight
//   above theta is kept, plus the lowest-position weights equal to theta that
//   are needed to reach p; indices are compacted in ascending token order by
//   a cluster-wide prefix sum.
#include <cooperative_groups.h>

#include "tw_common.cuh"
#include "tw_kernels.h"

namespace cg = cooperative_groups;

namespace tw {

constexpr int kEstThreads = 256;
constexpr int kEstPasses = kEstTile / (kEstThreads / 4);   // 4
constexpr float kInvSqrtD = 0.08838834764831845f;          // 1 / sqrt(128)

// Candidate position c of kv unit (b, hk) -> token id, or -1 if c is not a valid token.
__device__ __forceinline__ int cand_token(const int32_t* cand, int cand_stride, int64_t ukv,
                                          int c, int C, int len) {
  if (c >= C) return -1;
  int t = c;
  if (cand) t = cand[ukv * cand_stride + (c >> 4)] * kPage + (c & 15);
  return (t >= 0 && t < len) ? t : -1;
}

template <int G>
__global__ void __launch_bounds__(kEstThreads)
k_estimate(Layout L, const __half* __restrict__ q, int Hq, const uint8_t* __restrict__ codes,
           const __half* __restrict__ scales, const __half* __restrict__ zeros,
           const int32_t* __restrict__ cand, int cand_stride, const int32_t* __restrict__ ncand,
           int cap, int cmax, float* __restrict__ logits, float2* __restrict__ stats) {
  __shared__ __align__(16) float sq[G][kGroups][36];   // padded: 4 groups hit distinct banks
  __shared__ float red[kEstThreads / 32][G];
  __shared__ float smax[G];
  const int ukv = blockIdx.y;
  const int b = ukv / L.Hk, hk = ukv % L.Hk;
  const int len = L.len(b);
  const int C = min(cand ? ncand[ukv] * kPage : len, cmax);
  const int tile = blockIdx.x;
  const int c0 = tile * kEstTile;
  if (c0 >= C) return;
  const int tid = threadIdx.x;
  for (int i = tid; i < G * kHeadDim; i += kEstThreads) {
    const int h = i / kHeadDim, d = i % kHeadDim;
    sq[h][d >> 5][d & 31] = __half2float(q[((int64_t)b * Hq + hk * G + h) * kHeadDim + d]);
  }
  const int slot = tid >> 2, g = tid & 3;
  int tok[kEstPasses];
  uint4 cw[kEstPasses];
  float scl[kEstPasses], zer[kEstPasses];
#pragma unroll
  for (int k = 0; k < kEstPasses; ++k) {
    const int c = c0 + k * (kEstThreads / 4) + slot;
    tok[k] = cand_token(cand, cand_stride, ukv, c, C, len);
    cw[k] = make_uint4(0u, 0u, 0u, 0u);
    scl[k] = 0.f;
    zer[k] = 0.f;
    if (tok[k] >= 0) {
      const int64_t row = L.row(b, hk, tok[k]);
      cw[k] = ld_stream16(codes + row * (kHeadDim / 2) + g * 16);
      scl[k] = __half2float(scales[row * kGroups + g]);
      zer[k] = __half2float(zeros[row * kGroups + g]);
    }
  }
  __syncthreads();
  float lg[kEstPasses][G];
#pragma unroll
  for (int k = 0; k < kEstPasses; ++k) {
    const uint32_t w[4] = {cw[k].x, cw[k].y, cw[k].z, cw[k].w};
    // two accumulators per head (even / odd 8-channel chunk) for a shorter fp32 chain
    float a[G][2];
#pragma unroll
    for (int h = 0; h < G; ++h) a[h][0] = a[h][1] = 0.f;
#pragma unroll
    for (int m = 0; m < 4; ++m) {
      float kh[8];
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        // code as float without an int->float conversion: (2^23 + c) - 2^23 is exact
        const float cf = __uint_as_float(0x4B000000u | ((w[m] >> (4 * j)) & 0xFu)) - 8388608.0f;
        kh[j] = __fmaf_rn(scl[k], cf, zer[k]);
      }
#pragma unroll
      for (int h = 0; h < G; ++h) {
        const float4 q0 = *reinterpret_cast<const float4*>(&sq[h][g][8 * m]);
        const float4 q1 = *reinterpret_cast<const float4*>(&sq[h][g][8 * m + 4]);
        float t = a[h][m & 1];
        t = __fmaf_rn(q0.x, kh[0], t);
        t = __fmaf_rn(q0.y, kh[1], t);
        t = __fmaf_rn(q0.z, kh[2], t);
        t = __fmaf_rn(q0.w, kh[3], t);
        t = __fmaf_rn(q1.x, kh[4], t);
        t = __fmaf_rn(q1.y, kh[5], t);
        t = __fmaf_rn(q1.z, kh[6], t);
        t = __fmaf_rn(q1.w, kh[7], t);
        a[h][m & 1] = t;
      }
    }
#pragma unroll
    for (int h = 0; h < G; ++h) {
      float s = a[h][0] + a[h][1];
      s += __shfl_xor_sync(0xffffffffu, s, 1);
      s += __shfl_xor_sync(0xffffffffu, s, 2);
      lg[k][h] = tok[k] >= 0 ? s * kInvSqrtD : -INFINITY;
    }
  }
  // logits: lane g of a quad writes heads g, g+4, ...
#pragma unroll
  for (int k = 0; k < kEstPasses; ++k) {
    const int c = c0 + k * (kEstThreads / 4) + slot;
    if (c < C) {
#pragma unroll
      for (int h = 0; h < G; ++h)
        if ((h & 3) == g) logits[((int64_t)ukv * cap + c) * G + h] = lg[k][h];
    }
  }
  // tile statistics per head: max, then sum exp(l - max)
  const int lane = tid & 31, warp = tid >> 5;
#pragma unroll
  for (int h = 0; h < G; ++h) {
    float m = -INFINITY;
#pragma unroll
    for (int k = 0; k < kEstPasses; ++k) m = fmaxf(m, lg[k][h]);
    m = warp_max(m);
    if (lane == 0) red[warp][h] = m;
  }
  __syncthreads();
  if (tid < G) {
    float m = -INFINITY;
    for (int w = 0; w < kEstThreads / 32; ++w) m = fmaxf(m, red[w][tid]);
    smax[tid] = m;
  }
  __syncthreads();
#pragma unroll
  for (int h = 0; h < G; ++h) {
    const float m = smax[h];
    float z = 0.f;
    if (g == 0 && m != -INFINITY) {
#pragma unroll
      for (int k = 0; k < kEstPasses; ++k)
        if (tok[k] >= 0) z += expf(lg[k][h] - m);
    }
    z = warp_sum(z);
    if (lane == 0) red[warp][h] = z;
  }
  __syncthreads();
  if (tid < G) {
    float z = 0.f;
    for (int w = 0; w < kEstThreads / 32; ++w) z += red[w][tid];
    stats[((int64_t)ukv * (cap / kEstTile) + tile) * G + tid] = make_float2(smax[tid], z);
  }
}

// ---------------------------------------------------------------------------
constexpr int kToppThreads = 512;
constexpr int kToppWarps = kToppThreads / 32;
constexpr double kMassEps = 1e-12;
constexpr float kMassScale = 1099511627776.0f;   // 2^40

__device__ __forceinline__ unsigned long long mass_of(float w) {
  return __float2ull_rz(w * kMassScale);
}

// Block-wide exclusive scan of an unsigned value in thread order; returns the
// exclusive prefix and writes the block total to *total.  Uses sh[0..kToppWarps].
__device__ __forceinline__ unsigned block_excl_scan(unsigned v, unsigned* sh, unsigned* total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  unsigned incl = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const unsigned t = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += t;
  }
  if (lane == 31) sh[warp] = incl;
  __syncthreads();
  if (warp == 0) {
    const unsigned x = lane < kToppWarps ? sh[lane] : 0u;
    unsigned xi = x;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const unsigned t = __shfl_up_sync(0xffffffffu, xi, o);
      if (lane >= o) xi += t;
    }
    if (lane < kToppWarps) sh[lane] = xi - x;
    if (lane == 31) sh[kToppWarps] = xi;
  }
  __syncthreads();
  const unsigned r = sh[warp] + incl - v;
  *total = sh[kToppWarps];
  __syncthreads();
  return r;
}

// Cluster-wide exclusive prefix of per-block totals: returns the sum of the
// totals of lower-ranked blocks and writes the cluster total to *all.
// `slot` is this block's shared variable holding its total.
__device__ __forceinline__ unsigned cluster_prefix(cg::cluster_group& cl, unsigned* slot,
                                                   unsigned mine, unsigned* all) {
  if (threadIdx.x == 0) *slot = mine;
  cl.sync();
  const unsigned rank = cl.block_rank(), n = cl.num_blocks();
  unsigned before = 0, tot = 0;
  for (unsigned r = 0; r < n; ++r) {
    const unsigned v = *cl.map_shared_rank(slot, r);
    if (r < rank) before += v;
    tot += v;
  }
  *all = tot;
  return before;
}

// NH: heads averaged into one set (1 for per-head sets, G for group sets).
template <int NH, int R>
__global__ void __launch_bounds__(kToppThreads)
k_topp(Layout L, int Hq, int G, int group_sets, const int32_t* __restrict__ cand,
       int cand_stride, const int32_t* __restrict__ ncand, int lcap, int cmax,
       const float* __restrict__ logits, const float2* __restrict__ stats, double p,
       int32_t* __restrict__ idx, int icap, int32_t* __restrict__ count) {
  cg::cluster_group cl = cg::this_cluster();
  __shared__ unsigned long long hist[2][256];
  __shared__ unsigned long long wsuf[8];
  __shared__ unsigned long long sh_mass;
  __shared__ unsigned long long sh_above;
  __shared__ unsigned sh_scan[kToppWarps + 1];
  __shared__ unsigned sh_eq_tot, sh_sel_tot;
  __shared__ float sh_m[NH], sh_iz[NH];
  __shared__ float red[kToppWarps][NH];
  __shared__ unsigned long long wm[kToppWarps];
  __shared__ int sh_d;

  const int CS = (int)cl.num_blocks();
  const int cr = (int)cl.block_rank();
  const int set = blockIdx.x / CS;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  int b, hk, h0;
  if (group_sets) {
    b = set / L.Hk;
    hk = set % L.Hk;
    h0 = 0;
  } else {
    b = set / Hq;
    hk = (set % Hq) / G;
    h0 = (set % Hq) % G;
  }
  const int64_t ukv = (int64_t)b * L.Hk + hk;
  const int len = L.len(b);
  const int C = min(cand ? ncand[ukv] * kPage : len, cmax);
  const int ntiles = (C + kEstTile - 1) / kEstTile;
  const int tiles_cap = lcap / kEstTile;

  // 1. merge the tile statistics into each head's max and 1 / sum exp
  float mloc[NH];
#pragma unroll
  for (int h = 0; h < NH; ++h) mloc[h] = -INFINITY;
  for (int t = tid; t < ntiles; t += kToppThreads)
#pragma unroll
    for (int h = 0; h < NH; ++h)
      mloc[h] = fmaxf(mloc[h], stats[(ukv * tiles_cap + t) * G + h0 + h].x);
#pragma unroll
  for (int h = 0; h < NH; ++h) {
    const float m = warp_max(mloc[h]);
    if (lane == 0) red[warp][h] = m;
  }
  __syncthreads();
  if (tid < NH) {
    float m = -INFINITY;
    for (int w = 0; w < kToppWarps; ++w) m = fmaxf(m, red[w][tid]);
    sh_m[tid] = m;
  }
  __syncthreads();
  float zloc[NH];
#pragma unroll
  for (int h = 0; h < NH; ++h) zloc[h] = 0.f;
  for (int t = tid; t < ntiles; t += kToppThreads)
#pragma unroll
    for (int h = 0; h < NH; ++h) {
      const float2 s = stats[(ukv * tiles_cap + t) * G + h0 + h];
      if (s.x != -INFINITY) zloc[h] += s.y * expf(s.x - sh_m[h]);
    }
#pragma unroll
  for (int h = 0; h < NH; ++h) {
    const float z = warp_sum(zloc[h]);
    if (lane == 0) red[warp][h] = z;
  }
  __syncthreads();
  if (tid < NH) {
    float z = 0.f;
    for (int w = 0; w < kToppWarps; ++w) z += red[w][tid];
    sh_iz[tid] = z > 0.f ? 1.0f / z : 0.f;
  }
  __syncthreads();

  // 2. this thread's R consecutive candidate positions -> weights (invalid: -1)
  const int cbase = cr * (kToppThreads * R) + tid * R;
  float w[R];
#pragma unroll
  for (int i = 0; i < R; ++i) {
    const int c = cbase + i;
    w[i] = -1.0f;
    if (c < C) {
      float acc = 0.f;
      bool ok = true;
#pragma unroll
      for (int h = 0; h < NH; ++h) {
        const float l = logits[(ukv * lcap + c) * G + h0 + h];
        ok = ok && (l != -INFINITY);
        acc += expf(l - sh_m[h]) * sh_iz[h];
      }
      if (ok) w[i] = NH == 1 ? acc : acc * (1.0f / NH);
    }
  }

  // 3. total mass over the cluster
  unsigned long long mloc64 = 0;
#pragma unroll
  for (int i = 0; i < R; ++i)
    if (w[i] >= 0.f) mloc64 += mass_of(w[i]);
  mloc64 = warp_sum(mloc64);
  if (lane == 0) wm[warp] = mloc64;
  __syncthreads();
  if (tid == 0) {
    unsigned long long s = 0;
    for (int i = 0; i < kToppWarps; ++i) s += wm[i];
    sh_mass = s;
  }
  cl.sync();
  unsigned long long total = 0;
  for (int r = 0; r < CS; ++r) total += *cl.map_shared_rank(&sh_mass, r);

  const bool keep_all = p >= 1.0;
  uint32_t theta_key = 0;
  unsigned long long r_need = 0;
  if (!keep_all && total > 0) {
    double tf = ceil((p - kMassEps) * (double)total);
    unsigned long long T = tf < 1.0 ? 1ull : (unsigned long long)tf;
    if (T > total) T = total;
    uint32_t prefix = 0, pmask = 0;
    unsigned long long A = 0;   // mass strictly above the current prefix range
    for (int round = 0; round < 4; ++round) {
      const int shift = 24 - 8 * round;
      unsigned long long* hb = hist[round & 1];
      if (tid < 256) hb[tid] = 0;
      __syncthreads();
#pragma unroll
      for (int i = 0; i < R; ++i) {
        if (w[i] >= 0.f) {
          const uint32_t key = __float_as_uint(w[i]);
          if ((key & pmask) == prefix) atomicAdd(&hb[(key >> shift) & 255], mass_of(w[i]));
        }
      }
      cl.sync();
      unsigned long long suf = 0;
      if (tid < 256) {
        for (int r = 0; r < CS; ++r) suf += cl.map_shared_rank(hb, r)[tid];
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
          const unsigned long long t = __shfl_down_sync(0xffffffffu, suf, o);
          if (lane + o < 32) suf += t;
        }
        if (lane == 0) wsuf[warp] = suf;
      }
      __syncthreads();
      if (tid < 256)
        for (int ww = warp + 1; ww < 8; ++ww) suf += wsuf[ww];
      const int cnt = __syncthreads_count(tid < 256 && A + suf >= T);
      const int d = cnt - 1;
      if (tid == d + 1) sh_above = suf;
      if (tid == 0) sh_d = d;
      __syncthreads();
      A += (d == 255) ? 0ull : sh_above;
      prefix |= (uint32_t)sh_d << shift;
      pmask |= 255u << shift;
      __syncthreads();
    }
    theta_key = prefix;
    unsigned long long Ft = mass_of(__uint_as_float(theta_key));
    if (Ft == 0) Ft = 1;
    r_need = (T - A + Ft - 1) / Ft;
  }

  // 4. compaction in ascending position order over the cluster
  unsigned n_gt = 0, n_eq = 0;
#pragma unroll
  for (int i = 0; i < R; ++i) {
    if (w[i] < 0.f) continue;
    const uint32_t key = __float_as_uint(w[i]);
    if (keep_all || key > theta_key) ++n_gt;
    else if (key == theta_key && total > 0) ++n_eq;
  }
  unsigned eq_blk_total, eq_all;
  const unsigned eq_in_blk = block_excl_scan(n_eq, sh_scan, &eq_blk_total);
  const unsigned eq_before = cluster_prefix(cl, &sh_eq_tot, eq_blk_total, &eq_all) + eq_in_blk;
  unsigned take_eq = 0;
  if ((unsigned long long)eq_before < r_need)
    take_eq = (unsigned)((r_need - eq_before) < n_eq ? (r_need - eq_before) : n_eq);
  const unsigned n_sel = n_gt + take_eq;
  unsigned sel_blk_total, sel_all;
  const unsigned sel_in_blk = block_excl_scan(n_sel, sh_scan, &sel_blk_total);
  unsigned pos = cluster_prefix(cl, &sh_sel_tot, sel_blk_total, &sel_all) + sel_in_blk;
  int32_t* out = idx + (int64_t)set * icap;
  unsigned eq_taken = 0;
#pragma unroll
  for (int i = 0; i < R; ++i) {
    if (w[i] < 0.f) continue;
    const uint32_t key = __float_as_uint(w[i]);
    bool sel = keep_all || key > theta_key;
    if (!sel && key == theta_key && total > 0 && eq_taken < take_eq) {
      sel = true;
      ++eq_taken;
    }
    if (sel) out[pos++] = cand_token(cand, cand_stride, ukv, cbase + i, C, len);
  }
  if (cr == 0 && tid == 0) count[set] = (int32_t)sel_all;
  cl.sync();   // keep this block's shared memory alive until every peer has read it
}

// ---------------------------------------------------------------------------
void launch_estimate(const Layout& L, const __half* q, int Hq, const uint8_t* codes,
                     const __half* scales, const __half* zeros, const int32_t* cand,
                     int cand_stride, const int32_t* ncand, int cap, int cmax, float* logits,
                     float2* stats, cudaStream_t st) {
  const int G = Hq / L.Hk;
  dim3 grid(cap / kEstTile, L.B * L.Hk);
  switch (G) {
#define TW_EST(GG)                                                                        \
  case GG:                                                                                \
    k_estimate<GG><<<grid, kEstThreads, 0, st>>>(L, q, Hq, codes, scales, zeros, cand,     \
                                                 cand_stride, ncand, cap, cmax, logits,   \
                                                 stats);                                  \
    break;
    TW_EST(1) TW_EST(2) TW_EST(4) TW_EST(8)
#undef TW_EST
  }
}

template <int NH, int R>
static cudaError_t launch_topp_t(int sets, int CS, const Layout& L, int Hq, int G, int group_sets,
                                 const int32_t* cand, int cand_stride, const int32_t* ncand,
                                 int lcap, int cmax, const float* logits, const float2* stats,
                                 double p, int32_t* idx, int icap, int32_t* count,
                                 cudaStream_t st) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(sets * CS);
  cfg.blockDim = dim3(kToppThreads);
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = CS;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, k_topp<NH, R>, L, Hq, G, group_sets, cand, cand_stride, ncand,
                            lcap, cmax, logits, stats, p, idx, icap, count);
}

int topp_cluster_shape(int cmax, int* R, int* CS) {
  static const int Rs[4] = {4, 8, 16, 32};
  for (int i = 0; i < 4; ++i) {
    const int per_block = kToppThreads * Rs[i];
    const int cs = (cmax + per_block - 1) / per_block;
    if (cs <= 8) {
      *R = Rs[i];
      *CS = cs < 1 ? 1 : cs;
      return 0;
    }
  }
  return -1;
}

cudaError_t launch_topp(const Layout& L, int Hq, int group_sets, const int32_t* cand,
                        int cand_stride, const int32_t* ncand, int lcap, int cmax,
                        const float* logits, const float2* stats, double p, int32_t* idx,
                        int icap, int32_t* count, cudaStream_t st) {
  const int G = Hq / L.Hk;
  const int NH = group_sets ? G : 1;
  const int sets = group_sets ? L.B * L.Hk : L.B * Hq;
  int R = 0, CS = 0;
  if (topp_cluster_shape(cmax, &R, &CS) != 0) return cudaErrorInvalidValue;
#define TW_TOPP(NN, RR)                                                                        \
  if (NH == NN && R == RR)                                                                     \
    return launch_topp_t<NN, RR>(sets, CS, L, Hq, G, group_sets, cand, cand_stride, ncand,      \
                                 lcap, cmax, logits, stats, p, idx, icap, count, st);
#define TW_TOPP_R(NN) TW_TOPP(NN, 4) TW_TOPP(NN, 8) TW_TOPP(NN, 16) TW_TOPP(NN, 32)
  TW_TOPP_R(1) TW_TOPP_R(2) TW_TOPP_R(4) TW_TOPP_R(8)
#undef TW_TOPP_R
#undef TW_TOPP
  return cudaErrorInvalidValue;
}

}  // namespace tw
