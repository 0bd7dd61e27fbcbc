// Twilight's top-p threshold search and index compaction.
//
// Method ("Twilight: Adaptive Attention Sparsity with Hierarchical Top-p
// Pruning", atlas.scime.ai summary, "Approach"): keep the smallest set of
// candidates whose estimated attention weight reaches p (nucleus selection),
// found by a search over the threshold; under GQA one set per KV group with the
// group's averaged weights ("Limitations").
//
// One CTA per selection set (or a thread-block cluster of up to 8 CTAs when a
// set has more than 8192 candidates).  The set's weights stay in registers, R
// consecutive candidates per thread:
//   w = 2^(l - m) / Z               (per-head sets)
//   w = mean_h 2^(l_h - m_h) / Z_h  (group sets)
// with logits l in log2 units (the estimate kernel folds log2(e) into its
// scale) and m, Z merged from that kernel's per-32-candidate statistics.
// The threshold theta is the largest weight value whose retained mass
// sum_{w >= theta} w reaches p.  Weights lie in [0, 1], so their fp32 bit
// patterns order like their values and use 30 bits; theta is found most
// significant digit first in 4 steps (8 + 8 + 8 + 6 bits) instead of the 30 of
// a plain bisection.  Each step builds a histogram of masses per digit among
// the weights that match the digits found so far.  Masses are exact integers
// (each weight truncated to a multiple of 2^-40), so sums are independent of
// order; they are accumulated with native 32-bit shared-memory atomics on a low
// and a high word with an explicit carry.  The histogram is replicated 8 ways
// (by lane) because the weights of a set share few exponents and the first step
// would otherwise serialise on a few shared-memory addresses.  Across a cluster the per-CTA histograms are summed
// through distributed shared memory.  Every weight above theta is kept, plus
// the lowest-position weights equal to theta needed to reach p; the kept token
// ids are compacted in ascending order by one block scan (and one exchange of
// per-CTA totals in a cluster).  Each round costs two block barriers: the
// replicated histogram is summed, scanned and its digit chosen by one warp
// while the other warps clear the next round's buffer.
#include <cooperative_groups.h>

#include "tw_common.cuh"
#include "tw_kernels.h"

namespace cg = cooperative_groups;

namespace tw {

constexpr int kToppThreads = 512;
constexpr int kToppWarps = kToppThreads / 32;
constexpr int kHistReps = 8;
constexpr double kMassEps = 1e-12;               // exact ties at p resolve as in real arithmetic
constexpr float kMassScale = 1099511627776.0f;   // 2^40

__device__ __forceinline__ unsigned long long mass_of(float w) {
  return __float2ull_rz(w * kMassScale);
}

__device__ __forceinline__ int digit_shift(int round) { return round < 3 ? 22 - 8 * round : 0; }
__device__ __forceinline__ uint32_t digit_mask(int round) { return round < 3 ? 255u : 63u; }

// Block-wide exclusive scan of an unsigned value in thread order; writes the
// block total to *total.  Uses sh[0..kToppWarps].
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


// NH: heads averaged into one set (1 for per-head sets, G for group sets).
template <int NH, int R, bool CLUSTER>
__global__ void __launch_bounds__(kToppThreads)
k_topp(Layout L, int Hq, int G, int group_sets, const int32_t* __restrict__ cand,
       int cand_stride, const int32_t* __restrict__ ncand, int lcap, int cmax,
       const float* __restrict__ logits, const float2* __restrict__ stats, double p,
       int32_t* __restrict__ idx, int icap, int32_t* __restrict__ count,
       int32_t* __restrict__ done) {
  constexpr int NPG = (R + kPage - 1) / kPage;   // candidate pages a thread's R positions span
  __shared__ uint32_t hlo[2][kHistReps][256], hhi[2][kHistReps][256];   // double-buffered
  __shared__ unsigned long long hloc[2][256];                           // per-CTA totals (cluster)
  __shared__ unsigned long long sh_total, sh_above;
  __shared__ int sh_d;
  __shared__ unsigned sh_scan[kToppWarps + 1];
  __shared__ unsigned sh_blk[2];
  __shared__ unsigned sh_pre[4];
  __shared__ float sh_m[NH], sh_iz[NH];
  __shared__ float red[kToppWarps][NH];

  int CS = 1, cr = 0;
  if (CLUSTER) {
    cg::cluster_group cl = cg::this_cluster();
    CS = (int)cl.num_blocks();
    cr = (int)cl.block_rank();
  }
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
  const int cbase = cr * (kToppThreads * R) + tid * R;   // this thread's R consecutive candidates
  griddep_wait();
  // Loads that do not depend on the candidate count go out first: the page ids
  // of this thread's candidates and their logits (masked by the count below).
  int pgid[NPG];
#pragma unroll
  for (int k = 0; k < NPG; ++k) {
    const int pgl = (cbase >> 4) + k;
    pgid[k] = cand ? (pgl < cand_stride ? cand[ukv * cand_stride + pgl] : -1) : pgl;
  }
  // small sets of logits are loaded now, into registers; large ones when used
  constexpr bool kPre = NH * R <= 64;
  float lv[kPre ? R : 1][kPre ? NH : 1];
  if (kPre) {
#pragma unroll
    for (int i = 0; i < R; ++i)
#pragma unroll
      for (int h = 0; h < NH; ++h)
        lv[kPre ? i : 0][kPre ? h : 0] =
            (cbase + i < lcap) ? logits[(ukv * lcap + cbase + i) * G + h0 + h] : -INFINITY;
  }
  const int len = L.len(b);
  const int C = min(cand ? ncand[ukv] * kPage : len, cmax);
  const int nspans = (C + kStatSpan - 1) / kStatSpan;
  const float2* st = stats + ukv * (lcap / kStatSpan) * G + h0;
  {   // round 0's histogram starts at zero
    uint32_t* a = &hlo[0][0][0];
    uint32_t* c = &hhi[0][0][0];
    for (int i = tid; i < kHistReps * 256; i += kToppThreads) a[i] = c[i] = 0u;
  }

  // 1. merge the statistics records into each head's max and 1 / sum 2^(l - max)
  float mloc[NH];
#pragma unroll
  for (int h = 0; h < NH; ++h) mloc[h] = -INFINITY;
  for (int t = tid; t < nspans; t += kToppThreads)
#pragma unroll
    for (int h = 0; h < NH; ++h) mloc[h] = fmaxf(mloc[h], st[(int64_t)t * G + h].x);
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
  for (int t = tid; t < nspans; t += kToppThreads)
#pragma unroll
    for (int h = 0; h < NH; ++h) {
      const float2 s2 = st[(int64_t)t * G + h];
      if (s2.x != -INFINITY) zloc[h] += s2.y * exp2f(s2.x - sh_m[h]);
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

  // 2. weights (-1 marks an invalid slot)
  float w[R];
#pragma unroll
  for (int i = 0; i < R; ++i) {
    w[i] = -1.0f;
    if (cbase + i < C) {
      float acc = 0.f;
      bool ok = true;
#pragma unroll
      for (int h = 0; h < NH; ++h) {
        const float l = kPre ? lv[kPre ? i : 0][kPre ? h : 0]
                             : logits[(ukv * lcap + cbase + i) * G + h0 + h];
        ok = ok && (l != -INFINITY);
        acc += exp2f(l - sh_m[h]) * sh_iz[h];
      }
      if (ok) w[i] = NH == 1 ? acc : acc * (1.0f / NH);
    }
  }

  // 3. digit-by-digit search of theta over the cluster
  const bool keep_all = p >= 1.0;
  uint32_t theta = 0;
  unsigned long long r_need = 0, total = 0;
  bool have = false;
  if (!keep_all) {
    uint32_t prefix = 0, pmask = 0;
    unsigned long long A = 0, T = 0;   // A: mass strictly above the current prefix range
    const int rep = lane & (kHistReps - 1);
    for (int round = 0; round < 4; ++round) {
      const int buf = round & 1;
      const int shift = digit_shift(round);
      const uint32_t dm = digit_mask(round);
#pragma unroll
      for (int i = 0; i < R; ++i) {
        if (w[i] >= 0.f) {
          const uint32_t key = __float_as_uint(w[i]);
          if ((key & pmask) == prefix) {
            // exact 64-bit mass sum from native 32-bit atomics: low word, then
            // the high word plus the carry out of the low word
            const unsigned long long F = mass_of(w[i]);
            const uint32_t dg = (key >> shift) & dm;
            const uint32_t lo = (uint32_t)F;
            const uint32_t old = atomicAdd(&hlo[buf][rep][dg], lo);
            const uint32_t up = (uint32_t)(F >> 32) + (old + lo < old ? 1u : 0u);
            if (up) atomicAdd(&hhi[buf][rep][dg], up);
          }
        }
      }
      {   // the other buffer is not read in this round: clear it for the next one
        uint32_t* a = &hlo[buf ^ 1][0][0];
        uint32_t* c = &hhi[buf ^ 1][0][0];
        for (int i = tid; i < kHistReps * 256; i += kToppThreads) a[i] = c[i] = 0u;
      }
      __syncthreads();
      // warp 0: per-digit mass over the CTA (and cluster), suffix sums, the digit
      unsigned long long v[8];
      if (warp == 0) {
#pragma unroll
        for (int k = 0; k < 8; ++k) {
          const int j = 8 * lane + k;
          unsigned long long x = 0;
#pragma unroll
          for (int r = 0; r < kHistReps; ++r)
            x += ((unsigned long long)hhi[buf][r][j] << 32) | hlo[buf][r][j];
          v[k] = x;
          if (CLUSTER) hloc[buf][j] = x;
        }
      }
      if (CLUSTER) {
        cg::cluster_group cl = cg::this_cluster();
        cl.sync();
        if (warp == 0) {
#pragma unroll
          for (int k = 0; k < 8; ++k) {
            unsigned long long x = 0;
            for (int r = 0; r < CS; ++r) x += cl.map_shared_rank(&hloc[buf][0], r)[8 * lane + k];
            v[k] = x;
          }
        }
      }
      if (warp == 0) {
        unsigned long long sl[8];   // suffix within this lane's 8 digits
        sl[7] = v[7];
#pragma unroll
        for (int k = 6; k >= 0; --k) sl[k] = v[k] + sl[k + 1];
        unsigned long long incl = sl[0];   // suffix over lanes >= this one
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
          const unsigned long long t = __shfl_down_sync(0xffffffffu, incl, o);
          if (lane + o < 32) incl += t;
        }
        const unsigned long long after = incl - sl[0];   // mass of digits above this lane's
        if (round == 0) {
          total = __shfl_sync(0xffffffffu, incl, 0);
          const double tf = ceil((p - kMassEps) * (double)total);
          T = tf < 1.0 ? 1ull : (unsigned long long)tf;
          if (T > total) T = total;
        }
        int cnt = 0;
#pragma unroll
        for (int k = 0; k < 8; ++k) cnt += (A + sl[k] + after >= T) ? 1 : 0;
        cnt = warp_sum(cnt);
        const int d = cnt - 1;   // largest digit whose suffix mass reaches T
        const int dn = d + 1;
        unsigned long long ab = 0;
        if (dn < 256 && lane == (dn >> 3)) {
#pragma unroll
          for (int k = 0; k < 8; ++k)
            if (k == (dn & 7)) ab = sl[k] + after;
        }
        ab = __shfl_sync(0xffffffffu, ab, dn < 256 ? (dn >> 3) : 0);
        if (lane == 0) {
          sh_d = d;
          sh_above = dn < 256 ? ab : 0ull;
          if (round == 0) sh_total = total;
        }
      }
      __syncthreads();
      if (round == 0) {
        total = sh_total;
        if (total == 0) break;   // no valid candidate (uniform over the cluster)
        const double tf = ceil((p - kMassEps) * (double)total);
        T = tf < 1.0 ? 1ull : (unsigned long long)tf;
        if (T > total) T = total;
        have = true;
      }
      A += sh_above;
      prefix |= (uint32_t)sh_d << shift;
      pmask |= dm << shift;
    }
    if (have) {
      theta = prefix;
      unsigned long long Ft = mass_of(__uint_as_float(theta));
      if (Ft == 0) Ft = 1;
      r_need = (T - A + Ft - 1) / Ft;
    }
  }

  // 4. compaction in ascending position order
  unsigned n_gt = 0, n_eq = 0;
#pragma unroll
  for (int i = 0; i < R; ++i) {
    if (w[i] < 0.f) continue;
    const uint32_t key = __float_as_uint(w[i]);
    if (keep_all || (have && key > theta)) ++n_gt;
    else if (have && key == theta) ++n_eq;
  }
  unsigned blk_total;
  const unsigned ex = block_excl_scan((n_gt << 16) | n_eq, sh_scan, &blk_total);
  unsigned gt_before = 0, eq_before = 0, gt_all = blk_total >> 16, eq_all = blk_total & 0xFFFFu;
  if (CLUSTER) {
    cg::cluster_group cl = cg::this_cluster();
    if (tid == 0) {
      sh_blk[0] = blk_total >> 16;
      sh_blk[1] = blk_total & 0xFFFFu;
    }
    cl.sync();
    if (warp == 0) {
      unsigned g = 0, e = 0, gb = 0, eb = 0;
      if (lane < CS) {
        const unsigned* rb = cl.map_shared_rank(&sh_blk[0], lane);
        g = rb[0];
        e = rb[1];
        if (lane < cr) {
          gb = g;
          eb = e;
        }
      }
      g = warp_sum(g);
      e = warp_sum(e);
      gb = warp_sum(gb);
      eb = warp_sum(eb);
      if (lane == 0) {
        sh_pre[0] = gb;
        sh_pre[1] = eb;
        sh_pre[2] = g;
        sh_pre[3] = e;
      }
    }
    __syncthreads();
    gt_before = sh_pre[0];
    eq_before = sh_pre[1];
    gt_all = sh_pre[2];
    eq_all = sh_pre[3];
  }
  const unsigned long long ties_before = (unsigned long long)eq_before + (ex & 0xFFFFu);
  unsigned take = 0;
  if (ties_before < r_need) take = (unsigned)min((unsigned long long)n_eq, r_need - ties_before);
  unsigned pos = gt_before + (ex >> 16) + (unsigned)min(r_need, ties_before);
  int32_t* out = idx + (int64_t)set * icap;
  unsigned taken = 0;
#pragma unroll
  for (int i = 0; i < R; ++i) {
    if (w[i] < 0.f) continue;
    const uint32_t key = __float_as_uint(w[i]);
    bool sel = keep_all || (have && key > theta);
    if (!sel && have && key == theta && taken < take) {
      sel = true;
      ++taken;
    }
    if (sel) {
      const int c = cbase + i;
      out[pos++] = cand ? pgid[(c >> 4) - (cbase >> 4)] * kPage + (c & 15) : c;
    }
  }
  if (cr == 0 && tid == 0) {
    count[set] = (int32_t)(gt_all + (unsigned)min(r_need, (unsigned long long)eq_all));
    if (done) done[set] = 0;   // the attention kernel's per-set completion counter
  }
  griddep_launch();
  if (CLUSTER) cg::this_cluster().sync();   // peers may still read this block's shared memory
}

// ---------------------------------------------------------------------------
int topp_shape(int cmax, int* R, int* CS) {
  if (cmax <= kToppThreads * 16) {
    *CS = 1;
    *R = cmax <= kToppThreads * 4 ? 4 : (cmax <= kToppThreads * 8 ? 8 : 16);
    return 0;
  }
  for (int r = 16; r <= 32; r *= 2) {
    const int cs = (cmax + kToppThreads * r - 1) / (kToppThreads * r);
    if (cs <= 8) {
      *R = r;
      *CS = cs;
      return 0;
    }
  }
  return -1;
}

template <int NH, int R>
static cudaError_t launch_topp_t(int sets, int CS, const Layout& L, int Hq, int G, int group_sets,
                                 const int32_t* cand, int cand_stride, const int32_t* ncand,
                                 int lcap, int cmax, const float* logits, const float2* stats,
                                 double p, int32_t* idx, int icap, int32_t* count,
                                 int32_t* done, cudaStream_t st, bool pdl) {
  if (CS == 1)
    return launch_k(k_topp<NH, R, false>, dim3(sets), dim3(kToppThreads), 0, st, pdl, L, Hq, G,
                    group_sets, cand, cand_stride, ncand, lcap, cmax, logits, stats, p, idx, icap,
                    count, done);
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(sets * CS);
  cfg.blockDim = dim3(kToppThreads);
  cfg.stream = st;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = CS;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = pdl ? 2 : 1;
  return cudaLaunchKernelEx(&cfg, k_topp<NH, R, true>, L, Hq, G, group_sets, cand, cand_stride,
                            ncand, lcap, cmax, logits, stats, p, idx, icap, count, done);
}

cudaError_t launch_topp(const Layout& L, int Hq, int group_sets, const int32_t* cand,
                        int cand_stride, const int32_t* ncand, int lcap, int cmax,
                        const float* logits, const float2* stats, double p, int32_t* idx,
                        int icap, int32_t* count, int32_t* done, cudaStream_t st, bool pdl) {
  const int G = Hq / L.Hk;
  const int NH = group_sets ? G : 1;
  const int sets = group_sets ? L.B * L.Hk : L.B * Hq;
  int R = 0, CS = 0;
  if (topp_shape(cmax, &R, &CS) != 0) return cudaErrorInvalidValue;
#define TW_TOPP(NN, RR)                                                                       \
  if (NH == NN && R == RR)                                                                    \
    return launch_topp_t<NN, RR>(sets, CS, L, Hq, G, group_sets, cand, cand_stride, ncand,    \
                                 lcap, cmax, logits, stats, p, idx, icap, count, done, st, pdl);
#define TW_TOPP_R(NN) TW_TOPP(NN, 4) TW_TOPP(NN, 8) TW_TOPP(NN, 16) TW_TOPP(NN, 32)
  TW_TOPP_R(1) TW_TOPP_R(2) TW_TOPP_R(4) TW_TOPP_R(8)
#undef TW_TOPP_R
#undef TW_TOPP
  return cudaErrorInvalidValue;
}

}  // namespace tw
