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
//
// The threshold theta is the largest weight value whose retained mass
// sum_{w >= theta} w reaches p.  Weights lie in [0, 1], so their fp32 bit
// patterns order like their values and use 30 bits.  theta is found most
// significant digit first in 3 steps of 12 + 9 + 9 bits instead of the 30
// steps of a plain bisection.  Each step builds a histogram of masses per
// digit over the weights that match the digits found so far; one block-wide
// suffix scan (each thread owns 8 or 1 consecutive digits) then finds the
// digit where the retained mass crosses p.  The 12-bit first digit splits each
// binade of weight values 32 ways, so its shared-memory atomics rarely collide.
// Masses are exact integers (each weight truncated to a multiple of 2^-40), so
// sums are independent of order; they use native 32-bit atomics on a low and a
// high word with an explicit carry.  In a cluster every CTA sums all CTAs'
// histograms through distributed shared memory and reaches the same digit.
// Every weight above theta is kept, plus the lowest-position weights equal to
// theta needed to reach p; the kept token ids are compacted in ascending order
// by one block scan (and one exchange of per-CTA totals in a cluster).  When
// asked, the kernel also writes each kept token's physical K/V row (its page's
// first row, from the selector's row list, plus the offset in the page), so
// the attention kernel gathers rows without walking the page table.
#include <cooperative_groups.h>

#include "tw_common.cuh"
#include "tw_kernels.h"

namespace cg = cooperative_groups;

namespace tw {

constexpr int kToppThreads = 512;
constexpr int kToppWarps = kToppThreads / 32;
constexpr int kBins = 4096;                      // first digit: 12 bits
constexpr int kBinsPerThread = kBins / kToppThreads;
static_assert(kBinsPerThread == 8, "the first round reads two uint4 of bins per thread");
constexpr double kMassEps = 1e-12;               // exact ties at p resolve as in real arithmetic
constexpr float kMassScale = 1099511627776.0f;   // 2^40

__device__ __forceinline__ unsigned long long mass_of(float w) {
  return __float2ull_rz(w * kMassScale);
}

// Digits of the 30-bit weight key: bits 29..18, 17..9, 8..0.
__device__ __forceinline__ int digit_shift(int round) { return round == 0 ? 18 : (round == 1 ? 9 : 0); }
__device__ __forceinline__ uint32_t digit_mask(int round) { return round == 0 ? 0xFFFu : 0x1FFu; }

__device__ __forceinline__ unsigned long long join64(uint32_t hi, uint32_t lo) {
  return ((unsigned long long)hi << 32) | lo;
}

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

// State of the threshold search: the digits fixed so far (prefix under pmask),
// the mass A of the weights above that prefix range and the target mass T.
struct Search {
  uint32_t prefix, pmask;
  unsigned long long A, T;
};

// One digit of the search within one CTA: histogram the masses of the weights
// inside the current prefix range by the digit (key >> shift) & dm, scan the
// digits from the top, and fix the digit where the retained mass crosses T.
// Each thread owns BPT consecutive digits (BPT * 512 digits in all).  The
// first step (BPT == 8) also sets T from the total mass, and returns false if
// that is zero.  Leaves the histogram zeroed.
template <int R, int BPT>
__device__ __forceinline__ bool digit_step(const float (&w)[R], int shift, uint32_t dm, double p,
                                           uint32_t* hlo, uint32_t* hhi,
                                           unsigned long long* wsuf, int* sh_d,
                                           unsigned long long* sh_above, Search& s) {
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
#pragma unroll
  for (int i = 0; i < R; ++i) {
    if (w[i] >= 0.f) {
      const uint32_t key = __float_as_uint(w[i]);
      if ((key & s.pmask) == s.prefix) {
        // exact 64-bit mass sum from native 32-bit atomics: low word, then the
        // high word plus the carry out of the low word
        const unsigned long long F = mass_of(w[i]);
        const uint32_t dg = (key >> shift) & dm;
        const uint32_t lo = (uint32_t)F;
        const uint32_t old = atomicAdd(&hlo[dg], lo);
        const uint32_t up = (uint32_t)(F >> 32) + (old + lo < old ? 1u : 0u);
        if (up) atomicAdd(&hhi[dg], up);
      }
    }
  }
  __syncthreads();
  unsigned long long sl[BPT];   // suffix sums within this thread's digits
  if (BPT == 8) {
    const uint4 l0 = reinterpret_cast<const uint4*>(hlo)[2 * tid];
    const uint4 l1 = reinterpret_cast<const uint4*>(hlo)[2 * tid + 1];
    const uint4 u0 = reinterpret_cast<const uint4*>(hhi)[2 * tid];
    const uint4 u1 = reinterpret_cast<const uint4*>(hhi)[2 * tid + 1];
    const uint32_t lv[8] = {l0.x, l0.y, l0.z, l0.w, l1.x, l1.y, l1.z, l1.w};
    const uint32_t uv[8] = {u0.x, u0.y, u0.z, u0.w, u1.x, u1.y, u1.z, u1.w};
#pragma unroll
    for (int k = 0; k < BPT; ++k) sl[k] = join64(uv[k], lv[k]);
  } else {
#pragma unroll
    for (int k = 0; k < BPT; ++k) sl[k] = join64(hhi[BPT * tid + k], hlo[BPT * tid + k]);
  }
#pragma unroll
  for (int k = BPT - 2; k >= 0; --k) sl[k] += sl[k + 1];
  // suffix over this warp's higher lanes, then over the later warps
  unsigned long long incl = sl[0];
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const unsigned long long t = __shfl_down_sync(0xffffffffu, incl, o);
    if (lane + o < 32) incl += t;
  }
  if (lane == 0) wsuf[warp] = incl;
  __syncthreads();
  unsigned long long after = incl - sl[0];
  unsigned long long grand = 0;
#pragma unroll
  for (int w2 = 0; w2 < kToppWarps; ++w2) {
    const unsigned long long x = wsuf[w2];
    grand += x;
    if (w2 > warp) after += x;
  }
  if (BPT == 8) {
    if (grand == 0) return false;   // no valid candidate
    const double tf = ceil((p - kMassEps) * (double)grand);
    unsigned long long T = tf < 1.0 ? 1ull : (unsigned long long)tf;
    s.T = T > grand ? grand : T;
  }
  // the digit d with A + suffix(d) >= T > A + suffix(d + 1); exactly one thread
  // holds it, since A < T <= A + suffix(0)
#pragma unroll
  for (int k = 0; k < BPT; ++k) {
    const unsigned long long here = s.A + sl[k] + after;
    const unsigned long long next = s.A + (k + 1 < BPT ? sl[k + 1] : 0ull) + after;
    if (here >= s.T && next < s.T) {
      *sh_d = BPT * tid + k;
      *sh_above = next - s.A;
    }
  }
  // clear this thread's own digits (all readers are done) for the next step
  if (BPT == 8) {
    const uint4 z = make_uint4(0u, 0u, 0u, 0u);
    reinterpret_cast<uint4*>(hlo)[2 * tid] = z;
    reinterpret_cast<uint4*>(hlo)[2 * tid + 1] = z;
    reinterpret_cast<uint4*>(hhi)[2 * tid] = z;
    reinterpret_cast<uint4*>(hhi)[2 * tid + 1] = z;
  } else {
#pragma unroll
    for (int k = 0; k < BPT; ++k) hlo[BPT * tid + k] = hhi[BPT * tid + k] = 0u;
  }
  __syncthreads();
  // sh_d, sh_above and wsuf are next written after the next step's first barrier
  s.A += *sh_above;
  s.prefix |= (uint32_t)*sh_d << shift;
  s.pmask |= dm << shift;
  return true;
}

// Cluster form of digit_step: CTA r of the cluster sums slice r of the digits
// ([r NB / CS, (r + 1) NB / CS)) over every CTA's histogram through
// distributed shared memory (a reduce-scatter, so each histogram word crosses
// the cluster once), the slice totals are exchanged, and the one thread whose
// digit holds the crossing writes it into every CTA's shared memory.  Three
// cluster barriers per step; leaves this CTA's histogram zeroed.
template <int R, int NB>
__device__ __forceinline__ bool digit_step_cluster(const float (&w)[R], int shift, uint32_t dm,
                                                   double p, int CS, int cr, uint32_t* hlo,
                                                   uint32_t* hhi, unsigned long long* wsuf,
                                                   unsigned long long* slice_tot, int* sh_d,
                                                   unsigned long long* sh_above, Search& s) {
  cg::cluster_group cl = cg::this_cluster();
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
#pragma unroll
  for (int i = 0; i < R; ++i) {
    if (w[i] >= 0.f) {
      const uint32_t key = __float_as_uint(w[i]);
      if ((key & s.pmask) == s.prefix) {
        const unsigned long long F = mass_of(w[i]);
        const uint32_t dg = (key >> shift) & dm;
        const uint32_t lo = (uint32_t)F;
        const uint32_t old = atomicAdd(&hlo[dg], lo);
        const uint32_t up = (uint32_t)(F >> 32) + (old + lo < old ? 1u : 0u);
        if (up) atomicAdd(&hhi[dg], up);
      }
    }
  }
  cl.sync();   // every CTA's histogram is complete
  const int SB = NB / CS;                                       // digits per slice
  const int bpt = SB > kToppThreads ? SB / kToppThreads : 1;    // digits per thread (<= 8)
  const int first = cr * SB + tid * bpt;                        // this thread's first digit
  const bool holder = tid * bpt < SB;
  unsigned long long sl[8];
#pragma unroll
  for (int k = 0; k < 8; ++k) sl[k] = 0;
  if (holder) {
    // every peer's words are requested before any is added, so the remote
    // loads overlap instead of costing one round trip per peer
    for (int k0 = 0; k0 < bpt; k0 += 2) {
      uint32_t lv[8][2], hv[8][2];
#pragma unroll
      for (int r = 0; r < 8; ++r)
#pragma unroll
        for (int k = 0; k < 2; ++k) {
          lv[r][k] = hv[r][k] = 0u;
          if (r < CS && k0 + k < bpt) {
            lv[r][k] = cl.map_shared_rank(hlo, r)[first + k0 + k];
            hv[r][k] = cl.map_shared_rank(hhi, r)[first + k0 + k];
          }
        }
#pragma unroll
      for (int k = 0; k < 8; ++k)
        if (k >= k0 && k < k0 + 2)
#pragma unroll
          for (int r = 0; r < 8; ++r)
            sl[k] += ((unsigned long long)hv[r][k - k0] << 32) | lv[r][k - k0];
    }
  }
#pragma unroll
  for (int k = 6; k >= 0; --k)
    if (k + 1 < bpt) sl[k] += sl[k + 1];
  unsigned long long incl = sl[0];
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const unsigned long long t = __shfl_down_sync(0xffffffffu, incl, o);
    if (lane + o < 32) incl += t;
  }
  if (lane == 0) wsuf[warp] = incl;
  __syncthreads();
  unsigned long long after = incl - sl[0];   // within the slice, digits above this thread's
  unsigned long long slice = 0;
#pragma unroll
  for (int w2 = 0; w2 < kToppWarps; ++w2) {
    const unsigned long long x = wsuf[w2];
    slice += x;
    if (w2 > warp) after += x;
  }
  if (tid == 0) *slice_tot = slice;
  cl.sync();   // slice totals published; nobody reads this CTA's histogram any more
  for (int i = tid; i < NB; i += kToppThreads) hlo[i] = hhi[i] = 0u;
  unsigned long long tots[8];   // every slice's mass, requested together
#pragma unroll
  for (int r = 0; r < 8; ++r) tots[r] = r < CS ? *cl.map_shared_rank(slice_tot, r) : 0ull;
  unsigned long long total = 0, higher = 0;   // all slices; slices of larger digits
#pragma unroll
  for (int r = 0; r < 8; ++r) {
    total += tots[r];
    if (r > cr) higher += tots[r];
  }
  if (NB == kBins) {   // first step: the target mass (the same in every CTA)
    if (total == 0) return false;
    const double tf = ceil((p - kMassEps) * (double)total);
    unsigned long long T = tf < 1.0 ? 1ull : (unsigned long long)tf;
    s.T = T > total ? total : T;
  }
  if (holder) {
#pragma unroll
    for (int k = 0; k < 8; ++k) {
      if (k < bpt) {
        const unsigned long long here = s.A + higher + sl[k] + after;
        const unsigned long long next =
            s.A + higher + (k + 1 < bpt ? sl[k + 1] : 0ull) + after;
        if (here >= s.T && next < s.T)
          for (int r = 0; r < CS; ++r) {
            *cl.map_shared_rank(sh_d, r) = first + k;
            *cl.map_shared_rank(sh_above, r) = next - s.A;
          }
      }
    }
  }
  cl.sync();   // the digit is in every CTA's shared memory
  s.A += *sh_above;
  s.prefix |= (uint32_t)*sh_d << shift;
  s.pmask |= dm << shift;
  return true;
}

// Shared memory of k_topp<NH, R>: the mass histogram (reused after the
// search to stage the outputs), then, for mid-sized logit runs, a staging
// area the logits are copied into while the statistics are merged.
// kMode: 0 = logits to registers at entry, 1 = to shared memory at entry,
// 2 = loaded once the statistics are known.
template <int NH, int R>
struct ToppShape {
  static constexpr int kMode = NH * R <= 16 ? 0 : (NH * R <= 64 ? 1 : 2);
  static constexpr size_t kHistBytes =
      2 * kBins * 4 > kToppThreads * R * 4 ? 2 * kBins * 4 : (size_t)kToppThreads * R * 4;
  static constexpr size_t kBytes = kHistBytes + (kMode == 1 ? (size_t)kToppThreads * NH * R * 4 : 0);
};

__device__ __forceinline__ void cp_async16(void* smem, const void* gmem) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(
                   (unsigned)__cvta_generic_to_shared(smem)),
               "l"(gmem)
               : "memory");
}
__device__ __forceinline__ void cp_async_commit() {
  asm volatile("cp.async.commit_group;" ::: "memory");
}
template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

// NH: heads averaged into one set (1 for per-head sets, G for group sets).
template <int NH, int R, bool CLUSTER>
__global__ void __launch_bounds__(kToppThreads)
k_topp(Layout L, int Hq, int G, int group_sets, const int32_t* __restrict__ cand,
       int cand_stride, const int32_t* __restrict__ ncand, const uint32_t* __restrict__ row0,
       int lcap, int cmax, const float* __restrict__ logits, const float2* __restrict__ stats,
       double p, int32_t* __restrict__ idx, uint32_t* __restrict__ rows, int icap,
       int32_t* __restrict__ count, int32_t* __restrict__ done) {
  constexpr int NPG = (R + kPage - 1) / kPage;   // candidate pages a thread's R positions span
  using SH = ToppShape<NH, R>;
  extern __shared__ __align__(16) unsigned char topp_smem_raw[];
  uint32_t* hlo = reinterpret_cast<uint32_t*>(topp_smem_raw);   // mass histogram, low words
  uint32_t* hhi = hlo + kBins;                                   // and high words
  uint32_t* obuf = hlo;   // after the search: this CTA's output, staged for coalesced stores
  float4* lstage = reinterpret_cast<float4*>(topp_smem_raw + SH::kHistBytes);   // [NH][R/4][512]
  __shared__ unsigned long long wsuf[kToppWarps];   // per-warp suffix mass of its digits
  __shared__ unsigned long long sh_above;
  __shared__ int sh_d;
  __shared__ unsigned sh_scan[kToppWarps + 1];
  __shared__ unsigned sh_blk[2];
  __shared__ unsigned sh_pre[4];
  __shared__ float redm[kToppWarps][NH], redz[kToppWarps][NH];
  __shared__ unsigned long long slice_tot;       // cluster: this CTA's digit-slice mass
  __shared__ float2 mz_own[NH];                  // cluster: this CTA's (max, sum) per head
  __shared__ float2 mz_all[8][NH];               // cluster: every CTA's (max, sum) per head

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
  const int spans_cap = lcap / kStatSpan;
  const float2* st = stats + ukv * spans_cap * G + h0;
  {   // the first round's histogram starts at zero
    const uint4 z = make_uint4(0u, 0u, 0u, 0u);
    reinterpret_cast<uint4*>(hlo)[2 * tid] = z;
    reinterpret_cast<uint4*>(hlo)[2 * tid + 1] = z;
    reinterpret_cast<uint4*>(hhi)[2 * tid] = z;
    reinterpret_cast<uint4*>(hhi)[2 * tid + 1] = z;
  }
  griddep_wait();
  // Every load goes out before any result is needed: the candidate count, the
  // page ids of this thread's candidates, their logits and the first
  // statistics records (all masked by the count once it arrives).
  const int len = L.len(b);
  const int ncnt = cand ? ncand[ukv] : 0;
  int pgid[NPG];
  uint32_t pr0[NPG];   // first physical row of each page (for the attention kernel)
#pragma unroll
  for (int k = 0; k < NPG; ++k) {
    const int pgl = (cbase >> 4) + k;
    pgid[k] = cand ? (pgl < cand_stride ? cand[ukv * cand_stride + pgl] : -1) : pgl;
    pr0[k] = (!rows || pgl >= L.max_pages) ? 0u
             : row0                       ? row0[ukv * L.max_pages + pgl]
                                          : (uint32_t)L.page_row(b, hk, pgl);   // no candidate list
  }
  // logits [unit][G][lcap]: per head, this thread's R candidates are one
  // contiguous run of R / 4 float4 (R and lcap are multiples of 4)
  auto lrun = [&](int h) {
    return reinterpret_cast<const float4*>(logits + (ukv * G + h0 + h) * lcap + cbase);
  };
  const float4 kNone = make_float4(-INFINITY, -INFINITY, -INFINITY, -INFINITY);
  float4 lv[SH::kMode == 0 ? NH : 1][SH::kMode == 0 ? R / 4 : 1];
  if (SH::kMode == 0) {   // few: straight to registers
#pragma unroll
    for (int h = 0; h < NH; ++h)
#pragma unroll
      for (int j = 0; j < R / 4; ++j)
        lv[SH::kMode == 0 ? h : 0][SH::kMode == 0 ? j : 0] =
            cbase + 4 * j < lcap ? lrun(h)[j] : kNone;
  } else if (SH::kMode == 1) {   // more: to shared memory by cp.async, read after the statistics
#pragma unroll
    for (int h = 0; h < NH; ++h)
#pragma unroll
      for (int j = 0; j < R / 4; ++j) {
        float4* dst = &lstage[(h * (R / 4) + j) * kToppThreads + tid];
        if (cbase + 4 * j < lcap) cp_async16(dst, lrun(h) + j);
        else *dst = kNone;
      }
    cp_async_commit();
  }
  // statistics records of this CTA's candidates: one 32-candidate span per
  // thread (a CTA holds at most 512 * 32 candidates = 512 spans)
  const int sp = cr * (kToppThreads * R / kStatSpan) + tid;
  float2 sv[NH];
#pragma unroll
  for (int h = 0; h < NH; ++h)
    sv[h] = (tid < kToppThreads * R / kStatSpan && sp < spans_cap) ? st[(int64_t)sp * G + h]
                                                                    : make_float2(-INFINITY, 0.f);
  const int C = min(cand ? ncnt * kPage : len, cmax);
  const int nspans = (C + kStatSpan - 1) / kStatSpan;
  const bool mine = tid < kToppThreads * R / kStatSpan && sp < nspans;

  // 1. merge the statistics records into each head's max and 1 / sum 2^(l - max)
#pragma unroll
  for (int h = 0; h < NH; ++h) {
    const float m = warp_max(mine ? sv[h].x : -INFINITY);
    if (lane == 0) redm[warp][h] = m;
  }
  __syncthreads();
  float M[NH];
#pragma unroll
  for (int h = 0; h < NH; ++h) {
    M[h] = redm[0][h];
#pragma unroll
    for (int w2 = 1; w2 < kToppWarps; ++w2) M[h] = fmaxf(M[h], redm[w2][h]);
  }
#pragma unroll
  for (int h = 0; h < NH; ++h) {
    const float z =
        warp_sum((mine && sv[h].x != -INFINITY) ? sv[h].y * exp2f(sv[h].x - M[h]) : 0.f);
    if (lane == 0) redz[warp][h] = z;
  }
  __syncthreads();
  float Z[NH];
#pragma unroll
  for (int h = 0; h < NH; ++h) {
    Z[h] = 0.f;
#pragma unroll
    for (int w2 = 0; w2 < kToppWarps; ++w2) Z[h] += redz[w2][h];
  }
  if (CLUSTER) {   // combine the CTAs' (max, sum) pairs
    cg::cluster_group cl = cg::this_cluster();
    if (tid < NH) mz_own[tid] = make_float2(M[tid], Z[tid]);
    cl.sync();
    if (tid < CS * NH) mz_all[tid / NH][tid % NH] = *cl.map_shared_rank(&mz_own[tid % NH], tid / NH);
    cl.sync();   // also: no CTA reads mz_own again
#pragma unroll
    for (int h = 0; h < NH; ++h) {
      float m = -INFINITY;
      for (int r = 0; r < CS; ++r) m = fmaxf(m, mz_all[r][h].x);
      float z = 0.f;
      for (int r = 0; r < CS; ++r)
        if (mz_all[r][h].x != -INFINITY) z += mz_all[r][h].y * exp2f(mz_all[r][h].x - m);
      M[h] = m;
      Z[h] = z;
    }
  }
  float iz[NH];
#pragma unroll
  for (int h = 0; h < NH; ++h) iz[h] = Z[h] > 0.f ? 1.0f / Z[h] : 0.f;

  // 2. weights (-1 marks an invalid slot)
  if (SH::kMode == 1) {
    cp_async_wait<0>();   // each thread reads back only its own staged logits
  }
  float w[R];
#pragma unroll
  for (int i = 0; i < R; ++i) w[i] = 0.f;
  bool okw[R];
#pragma unroll
  for (int i = 0; i < R; ++i) okw[i] = cbase + i < C;
#pragma unroll
  for (int h = 0; h < NH; ++h) {
#pragma unroll
    for (int j = 0; j < R / 4; ++j) {
      float4 l4;
      if (SH::kMode == 0) l4 = lv[SH::kMode == 0 ? h : 0][SH::kMode == 0 ? j : 0];
      else if (SH::kMode == 1) l4 = lstage[(h * (R / 4) + j) * kToppThreads + tid];
      else l4 = cbase + 4 * j < lcap ? lrun(h)[j] : kNone;
      const float l[4] = {l4.x, l4.y, l4.z, l4.w};
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        okw[4 * j + e] = okw[4 * j + e] && (l[e] != -INFINITY);
        w[4 * j + e] += exp2f(l[e] - M[h]) * iz[h];
      }
    }
  }
#pragma unroll
  for (int i = 0; i < R; ++i) w[i] = okw[i] ? (NH == 1 ? w[i] : w[i] * (1.0f / NH)) : -1.0f;

  // 3. digit-by-digit search of theta over the cluster
  const bool keep_all = p >= 1.0;
  uint32_t theta = 0;
  unsigned long long r_need = 0;
  bool have = false;
  if (!keep_all) {
    Search s{0u, 0u, 0ull, 0ull};
    if (CLUSTER) {
      have = digit_step_cluster<R, kBins>(w, 18, 0xFFFu, p, CS, cr, hlo, hhi, wsuf, &slice_tot,
                                          &sh_d, &sh_above, s);
      if (have) {
        digit_step_cluster<R, 512>(w, 9, 0x1FFu, p, CS, cr, hlo, hhi, wsuf, &slice_tot, &sh_d,
                                   &sh_above, s);
        digit_step_cluster<R, 512>(w, 0, 0x1FFu, p, CS, cr, hlo, hhi, wsuf, &slice_tot, &sh_d,
                                   &sh_above, s);
      }
    } else {
      have = digit_step<R, kBinsPerThread>(w, 18, 0xFFFu, p, hlo, hhi, wsuf, &sh_d, &sh_above, s);
      if (have) {
        digit_step<R, 1>(w, 9, 0x1FFu, p, hlo, hhi, wsuf, &sh_d, &sh_above, s);
        digit_step<R, 1>(w, 0, 0x1FFu, p, hlo, hhi, wsuf, &sh_d, &sh_above, s);
      }
    }
    if (have) {
      theta = s.prefix;
      unsigned long long Ft = mass_of(__uint_as_float(theta));
      if (Ft == 0) Ft = 1;
      r_need = (s.T - s.A + Ft - 1) / Ft;
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
  // this CTA's outputs are one contiguous run [first, first + n_out) of the
  // set's list; they are staged in shared memory and written coalesced
  const unsigned first = gt_before + (unsigned)min(r_need, (unsigned long long)eq_before);
  const unsigned eq_blk = blk_total & 0xFFFFu;
  const unsigned n_out =
      (blk_total >> 16) +
      (r_need > eq_before ? (unsigned)min((unsigned long long)eq_blk, r_need - eq_before) : 0u);
  const unsigned lpos0 = (ex >> 16) + (unsigned)min(r_need, ties_before) -
                         (unsigned)min(r_need, (unsigned long long)eq_before);
  unsigned sel_mask = 0;   // bit i: candidate cbase + i is kept
  {
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
      if (sel) sel_mask |= 1u << i;
    }
  }
  int32_t* out = idx + (int64_t)set * icap + first;
  for (int pass = 0; pass < (rows ? 2 : 1); ++pass) {
    unsigned lp = lpos0;
#pragma unroll
    for (int i = 0; i < R; ++i) {
      if (sel_mask & (1u << i)) {
        const int c = cbase + i;
        const int k = (c >> 4) - (cbase >> 4);
        obuf[lp++] = pass == 0 ? (uint32_t)(cand ? pgid[k] * kPage + (c & 15) : c)
                               : pr0[k] + (uint32_t)(c & 15);
      }
    }
    __syncthreads();
    uint32_t* dst = pass == 0 ? reinterpret_cast<uint32_t*>(out) : rows + (int64_t)set * icap + first;
    for (unsigned i = tid; i < n_out; i += kToppThreads) dst[i] = obuf[i];
    __syncthreads();   // obuf is rewritten by the next pass
  }
  if (cr == 0 && tid == 0) {
    count[set] = (int32_t)(gt_all + (unsigned)min(r_need, (unsigned long long)eq_all));
    if (done) done[set] = 0;   // the attention kernel's per-set completion counter
  }
  griddep_launch();
  if (CLUSTER) cg::this_cluster().sync();   // peers may still read this block's shared memory
}

// ---------------------------------------------------------------------------
int topp_shape(int cmax, int sets, int* R, int* CS) {
  if (cmax <= kToppThreads * 16) {
    *CS = 1;
    *R = cmax <= kToppThreads * 4 ? 4 : (cmax <= kToppThreads * 8 ? 8 : 16);
    return 0;
  }
  // clusters of 2, 4 or 8 CTAs (a power of two splits the digits into equal
  // slices for the reduce-scatter) of one CTA per SM: 16 weights per thread,
  // or 32 when that keeps every cluster of the launch resident at once
  int best_r = 0, best_cs = 0;
  for (int r = 16; r <= 32; r *= 2) {
    int cs = (cmax + kToppThreads * r - 1) / (kToppThreads * r);
    cs = cs <= 2 ? 2 : (cs <= 4 ? 4 : (cs <= 8 ? 8 : 16));
    if (cs > 8) continue;
    if (best_r == 0 || ((long long)sets * best_cs > kTargetSms && (long long)sets * cs <= kTargetSms)) {
      best_r = r;
      best_cs = cs;
    }
  }
  if (best_r == 0) return -1;
  *R = best_r;
  *CS = best_cs;
  return 0;
}

template <int NH, int R>
static cudaError_t launch_topp_t(int sets, int CS, const Layout& L, int Hq, int G, int group_sets,
                                 const int32_t* cand, int cand_stride, const int32_t* ncand,
                                 const uint32_t* row0, int lcap, int cmax, const float* logits,
                                 const float2* stats, double p, int32_t* idx, uint32_t* rows,
                                 int icap, int32_t* count, int32_t* done, cudaStream_t st,
                                 bool pdl) {
  using SH = ToppShape<NH, R>;
  static std::atomic<int> attr_set[kMaxDevices];
  const cudaError_t prepared = once_per_device(attr_set, [] {
    cudaError_t e = cudaFuncSetAttribute(k_topp<NH, R, false>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)SH::kBytes);
    if (e == cudaSuccess)
      e = cudaFuncSetAttribute(k_topp<NH, R, true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               (int)SH::kBytes);
    return e;
  });
  if (prepared != cudaSuccess) return prepared;
  if (CS == 1)
    return launch_k(k_topp<NH, R, false>, dim3(sets), dim3(kToppThreads), SH::kBytes, st, pdl, L, Hq, G,
                    group_sets, cand, cand_stride, ncand, row0, lcap, cmax, logits, stats, p, idx,
                    rows, icap, count, done);
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(sets * CS);
  cfg.blockDim = dim3(kToppThreads);
  cfg.dynamicSmemBytes = SH::kBytes;
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
                            ncand, row0, lcap, cmax, logits, stats, p, idx, rows, icap, count,
                            done);
}

cudaError_t launch_topp(const Layout& L, int Hq, int group_sets, const int32_t* cand,
                        int cand_stride, const int32_t* ncand, const uint32_t* row0, int lcap,
                        int cmax, const float* logits, const float2* stats, double p,
                        int32_t* idx, uint32_t* rows, int icap, int32_t* count, int32_t* done,
                        cudaStream_t st, bool pdl) {
  const int G = Hq / L.Hk;
  const int NH = group_sets ? G : 1;
  const int sets = group_sets ? L.B * L.Hk : L.B * Hq;
  int R = 0, CS = 0;
  if (topp_shape(cmax, sets, &R, &CS) != 0) return cudaErrorInvalidValue;
#define TW_TOPP(NN, RR)                                                                       \
  if (NH == NN && R == RR)                                                                    \
    return launch_topp_t<NN, RR>(sets, CS, L, Hq, G, group_sets, cand, cand_stride, ncand,    \
                                 row0, lcap, cmax, logits, stats, p, idx, rows, icap, count,  \
                                 done, st, pdl);
#define TW_TOPP_R(NN) TW_TOPP(NN, 4) TW_TOPP(NN, 8) TW_TOPP(NN, 16) TW_TOPP(NN, 32)
  TW_TOPP_R(1) TW_TOPP_R(2) TW_TOPP_R(4) TW_TOPP_R(8)
#undef TW_TOPP_R
#undef TW_TOPP
  return cudaErrorInvalidValue;
}

}  // namespace tw
