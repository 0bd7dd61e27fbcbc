// Twilight's selection stages for one (sequence, KV head) unit on one
// thread-block cluster: Quest page scores and top-K_p pages, then the
// quantised-key weight estimate, the top-p threshold and the compaction of the
// kept tokens.
//
// Method ("Twilight: Adaptive Attention Sparsity with Hierarchical Top-p
// Pruning", atlas.scime.ai summary): a base selector pre-selects candidates
// and top-p over the candidates' estimated attention weights prunes them
// ("Approach"); Quest, the base selector here, ranks 16-token pages by a bound
// from the page's per-channel key min / max ("Surprising findings", "Builds
// on"); the weights are estimated from the 4-bit key cache ("Approach"; the
// 2-bit cache of the quantisation ablation, table of measured effects, runs
// through the same code); under GQA the budget is group-wise ("Limitations").
//
// Work split.  A unit is processed by one cluster of CS CTAs (CS = 1..16).
//   Phase 1 (scores, top-K_p).  CTA r scores pages [r P / CS, (r+1) P / CS) of
//   the unit's P pages: their 512-byte metadata records stream through a
//   shared-memory ring filled by bulk copies.  Each page's score key is stored
//   into every CTA's key array (distributed shared memory), so after one
//   cluster barrier every CTA holds all P keys and runs the same radix select
//   on its own: the K_p best pages (ties to the lower page) and their
//   ascending order, with no further exchange.  CTA r then owns the share
//   [r K_p / CS, (r+1) K_p / CS) of the candidate list.
//   Phase 2 (estimate, top-p).  Each CTA streams its share's quantised key
//   rows (whole 16-row pages) through a second ring, computes the logits of
//   every query head of the group on the tensor cores (mma.sync, codes as the
//   A operand) into shared memory and keeps per-head (max, sum 2^(l - max)).
//   One exchange of those pairs gives every CTA the unit's softmax statistics.
//   Each thread then owns the weights of R consecutive candidates of its
//   CTA's share (in shared memory), and the threshold is found most
//   significant digit first (12 + 9 + 9 bits of the fp32 weight) over exact
//   integer masses.  The first digit's histograms are reduce-scattered over
//   the cluster through distributed shared memory; when that digit holds few
//   enough weights over the cluster, every CTA gathers them and finishes on
//   its own (a one-warp sort up to 128 weights, the remaining two digits on
//   the list up to 1024), else the remaining digits are reduced like the
//   first.  The kept tokens are compacted in ascending order with their
//   physical K/V rows for the attention kernel.
//
// The score of a page is a deterministic fp32 sum in one fixed order, so the
// selected page ids are an exact integer result: products of two fp16 values
// are exact in fp32; each lane of a half-warp sums its 8 channels left to
// right; the 16 lane sums are combined by xor-butterfly 8, 4, 2, 1 (fp32
// addition is commutative, so both butterfly partners hold the same value);
// the group's heads are added in head order.  Each channel's bound term
// max(q min, q max) equals q+ max + q- min with q+ = max(q, 0), q- = min(q, 0)
// (one of the two products is zero), so it is accumulated with two fused
// multiply-adds whose single rounding is the rounding of the sum.
//
// Streaming: each ring stage completes on its "full" mbarrier: bulk copies
// (cp.async.bulk) with their byte counts for the metadata records, or every
// thread's cp.async pieces (one arrival per thread when they have landed) for
// the quantised rows, whose scales and zeros need not start 16-byte aligned
// in a contiguous cache.  A stage is refilled after the block barrier that
// ends its use.  No copy uses cluster multicast.  Every wait is bounded
// (tw_bulk.cuh).
#include "tw_bulk.cuh"
#include "tw_common.cuh"
#include "tw_kernels.h"

namespace tw {

constexpr int kSpWarps = kSpThreads / 32;
constexpr int kMetaStagePages = 64;     // page records per score stage (32 KB); 32 or 64
static_assert(kMetaStagePages == 32 || kMetaStagePages == 64, "two or four pages per half-warp");
constexpr int kMetaRecBytes = 2 * kHeadDim * 2;          // one page's min and max rows
constexpr int kEstStagePages = 16;                       // 256 candidate tokens per stage
constexpr int kEstStageTok = kEstStagePages * kPage;
constexpr int kSpBins = 4096;                            // first digit of the searches: 12 bits
constexpr int kSpBinList = 1024;                         // a first-digit bin this small is resolved in every CTA
constexpr float kEstL2Scale = 1.4426950408889634f * 0.08838834764831845f;   // log2(e)/sqrt(128)
constexpr double kSpMassEps = 1e-12;           // exact ties at p resolve as in real arithmetic
constexpr float kSpMassScale = 1099511627776.0f;   // 2^40

template <int BITS>
struct SpKeyWidth {
  static_assert(BITS == 4 || BITS == 2, "key-cache width");
  static constexpr int kRowBytes = kHeadDim * BITS / 8;
  static constexpr int kLaneBytes = kGroup * BITS / 8;
  static constexpr float kCentre = BITS == 4 ? 8.f : 2.f;
  static constexpr int kStageBytes = kEstStageTok * (kRowBytes + 2 * kGroups * 2);
  // channel that feeds MMA k-slot pair j, element hi, at K-step s (offset in the lane's group)
  __device__ static constexpr int chan(int s, int j, int hi) {
    return BITS == 4 ? 8 * (s >> 1) + 2 * (s & 1) + j + 4 * hi
                     : 16 * (s >> 2) + 2 * (s & 3) + j + 8 * hi;
  }
};

// Fixed part of the shared memory; the phase regions follow it.
struct SpFixed {
  __align__(16) __half qs[8][kHeadDim];   // the unit's query heads
  int seq;                                // the unit's sequence
  uint64_t full1[kSpMaxStages];
  int32_t pt1[kSpMaxStages][kMetaStagePages];   // paged: pool pages of each ring stage
  uint64_t full2[kSpMaxStages];
  uint32_t pg[kSpSharePages];     // this CTA's share of the candidate list: page ids
  uint32_t r0[kSpSharePages];     // first physical row of each page
  int32_t nrow[kSpSharePages];    // valid rows of each page (0: not a page of the sequence)
  int32_t crow[kSpSharePages];    // rows of each page copied (whole page, short at the allocation end)
  float2 wstat[kSpWarps][8];      // per warp and head: (max, sum 2^(l - max))
  float2 mz_loc[8];               // this CTA's pair per head
  float2 mz_all[kSpMaxCluster][8];   // every CTA's pair per head
  unsigned long long wsuf[kSpWarps];
  unsigned long long slice_tot;
  unsigned long long sh_above;
  int sh_d;
  int sh_need;
  uint32_t sh_pref;
  int2 scan2[kSpWarps + 1];
  unsigned scan[kSpWarps + 1];
  uint32_t wmin[kSpWarps], wmax[kSpWarps];
  uint32_t kmin[kSpMaxCluster * kSpWarps], kmax[kSpMaxCluster * kSpWarps];   // per CTA and warp
  unsigned blk[2];
  unsigned pre[4];
  int lst_n;
  uint32_t res_theta;             // small-bin resolution: theta
  unsigned long long res_above;   // and the bin's mass above it
};

constexpr size_t kSpFixedBytes = (sizeof(SpFixed) + 127) / 128 * 128;

size_t sp_fixed_bytes() { return kSpFixedBytes; }

__device__ __forceinline__ void cp_async16_sm(void* smem, const void* gmem) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(smem_u32(smem)), "l"(gmem)
               : "memory");
}

__device__ __forceinline__ void cp_async8_sm(void* smem, const void* gmem) {
  asm volatile("cp.async.ca.shared.global [%0], [%1], 8;" ::"r"(smem_u32(smem)), "l"(gmem)
               : "memory");
}

// All of this thread's earlier cp.async arrive on `bar` when they complete.
__device__ __forceinline__ void cp_async_arrive_noinc(uint64_t* bar) {
  asm volatile("cp.async.mbarrier.arrive.noinc.shared::cta.b64 [%0];" ::"r"(smem_u32(bar))
               : "memory");
}

__device__ __forceinline__ void fence_proxy_async() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// Shared-memory index of element i of an array padded by one word per 32:
// a thread's run of E consecutive elements (E <= 32) is then conflict-free
// when the threads of a warp read their runs in step.
__host__ __device__ __forceinline__ int sp_pad(int i) { return i + (i >> 5); }

// Words of a padded digit histogram of kSpBins bins (the bins a thread scans
// are consecutive, so their padded words are conflict-free across a warp).
constexpr int kSpHistWords = kSpBins + kSpBins / 32;
constexpr int kSpHistBytes = kSpHistWords * 8;   // a digit histogram of 64-bit words
constexpr int kSpListWord = 1024;
constexpr int kMetaBulkLanes = 8;  // lanes per warp issuing a paged stage's record copies
static_assert(kMetaBulkLanes * kSpWarps >= kMetaStagePages, "a lane per record of a stage");
constexpr int kSpSortPerLane = 4;   // a bin list of at most 32 * this is sorted by one warp   // 64-bit word of the histogram storage where the bin lists start
constexpr int kSpLoBits = 19;
// First digit of the top-p search: bits 29..18 of the weight's fp32 pattern.
// A weight of nonzero mass is at least 2^-40, so its digit is at least
// 87 * 32; the histogram covers digits [2048, 4096) only.
constexpr int kSpShift0 = 18;
constexpr int kTopkDigitBits = 10;   // digit width of the page top-k rounds
constexpr int kSpDigit0Base = 2048;
constexpr int kSpBins0 = kSpBins - kSpDigit0Base;
constexpr int kPtAhead = 6;   // iterations between a page-table load and its store (< kSpWarps)   // low bits of a mass in a bin word's low half

__device__ __forceinline__ float sp_h(uint32_t w, int hi) {
  return __half2float(__ushort_as_half((unsigned short)((w >> (16 * hi)) & 0xFFFFu)));
}

// ---------------------------------------------------------------------------
// Block-wide scans over the 256 threads (all threads call them).

__device__ __forceinline__ int2 sp_scan2(int2 v, int2* sh, int2* total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  int2 incl = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int tx = __shfl_up_sync(0xffffffffu, incl.x, o);
    const int ty = __shfl_up_sync(0xffffffffu, incl.y, o);
    if (lane >= o) {
      incl.x += tx;
      incl.y += ty;
    }
  }
  __syncthreads();   // sh is free
  if (lane == 31) sh[warp] = incl;
  __syncthreads();
  int2 before = make_int2(0, 0), tot = make_int2(0, 0);
#pragma unroll
  for (int w = 0; w < kSpWarps; ++w) {
    const int2 x = sh[w];
    if (w < warp) {
      before.x += x.x;
      before.y += x.y;
    }
    tot.x += x.x;
    tot.y += x.y;
  }
  *total = tot;
  return make_int2(before.x + incl.x - v.x, before.y + incl.y - v.y);
}

__device__ __forceinline__ unsigned sp_scan(unsigned v, unsigned* sh, unsigned* total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  unsigned incl = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const unsigned t = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += t;
  }
  __syncthreads();
  if (lane == 31) sh[warp] = incl;
  __syncthreads();
  unsigned before = 0, tot = 0;
#pragma unroll
  for (int w = 0; w < kSpWarps; ++w) {
    const unsigned x = sh[w];
    if (w < warp) before += x;
    tot += x;
  }
  *total = tot;
  return before + incl - v;
}

// ---------------------------------------------------------------------------
// Phase 1: Quest page scores of this CTA's slice, keys to every CTA.

// One page's score: this lane's 8 channels of the min and max rows, the
// query channels of the group's heads (q+ / q- split for G <= 4, plain q for
// G = 8), the fixed summation order.
template <int G>
struct ScoreQ {
  static constexpr bool kSplit = G <= 4;
  // split form: q+ = max(q, 0) and q- = min(q, 0) as fp16 bit patterns (exact);
  // plain form: q as fp32
  uint32_t ap[kSplit ? G : 1][4], an[kSplit ? G : 1][4];   // channel pairs (2i, 2i + 1)
  float a[kSplit ? 1 : G][8];
};

// fp32 d = a * b + c for fp16 a, b: the product is exact in fp32 and the sum
// is rounded once, as fmaf on the converted operands.
__device__ __forceinline__ float fma_h(unsigned short a, unsigned short b, float c) {
  float d;
  asm("fma.rn.f32.f16 %0, %1, %2, %3;" : "=f"(d) : "h"(a), "h"(b), "f"(c));
  return d;
}

__device__ __forceinline__ unsigned short h_part(uint32_t w, int hi) {
  return (unsigned short)((w >> (16 * hi)) & 0xFFFFu);
}

// The lane's partial of head g over its 8 channels of a page, left to right:
// max(q_j min_j, q_j max_j) summed in fp32.
template <int G>
__device__ __forceinline__ float lane_partial(const ScoreQ<G>& Q, int g, const uint32_t (&wn)[4],
                                              const uint32_t (&wx)[4]) {
  if (ScoreQ<G>::kSplit) {
    const int gs = ScoreQ<G>::kSplit ? g : 0;
    // channel j: q+ max + q- min (one of the two is zero)
    float s = fma_h(h_part(Q.ap[gs][0], 0), h_part(wx[0], 0), -0.0f);
    s = fma_h(h_part(Q.an[gs][0], 0), h_part(wn[0], 0), s);
#pragma unroll
    for (int j = 1; j < 8; ++j) {
      s = fma_h(h_part(Q.ap[gs][j >> 1], j & 1), h_part(wx[j >> 1], j & 1), s);
      s = fma_h(h_part(Q.an[gs][j >> 1], j & 1), h_part(wn[j >> 1], j & 1), s);
    }
    return s;
  }
  const int ga = ScoreQ<G>::kSplit ? 0 : g;
  float s = fmaxf(__fmul_rn(Q.a[ga][0], sp_h(wn[0], 0)), __fmul_rn(Q.a[ga][0], sp_h(wx[0], 0)));
#pragma unroll
  for (int j = 1; j < 8; ++j) {
    const float mn = sp_h(wn[j >> 1], j & 1), mx = sp_h(wx[j >> 1], j & 1);
    s = __fadd_rn(s, fmaxf(__fmul_rn(Q.a[ga][j], mn), __fmul_rn(Q.a[ga][j], mx)));
  }
  return s;
}

// Scores of the NP (2 or 4) pages hw + 16 k of a ring stage, by the 16 lanes
// of half-warp hw: each lane's partials, then per head the 16-lane sum in the
// xor-butterfly order 8, 4, 2, 1, heads added in order.  The butterfly runs
// transposed: at offset 8 a lane keeps the half of the pages on its side and
// sends the other half, at offset 4 again, so each exchange moves one value
// per page-pair instead of one per page; every page's sum is formed by the
// same additions as a plain butterfly.  Lane l16 returns the score of page
// (l16 >> 2) & 3 (NP = 4) or (l16 >> 3) & 1 (NP = 2).
template <int G, int NP>
__device__ __forceinline__ float page_scores(const ScoreQ<G>& Q, const unsigned char* st, int hw,
                                             int l16, unsigned hmask) {
  uint32_t wn[NP][4], wx[NP][4];
#pragma unroll
  for (int k = 0; k < NP; ++k) {
    const uint4* rec = reinterpret_cast<const uint4*>(st + (hw + 16 * k) * 512);
    const uint4 mn = rec[l16], mx = rec[16 + l16];
    wn[k][0] = mn.x, wn[k][1] = mn.y, wn[k][2] = mn.z, wn[k][3] = mn.w;
    wx[k][0] = mx.x, wx[k][1] = mx.y, wx[k][2] = mx.z, wx[k][3] = mx.w;
  }
  const bool b = (l16 >> 3) & 1, c = (l16 >> 2) & 1;
  float total = 0.f;
#pragma unroll
  for (int g = 0; g < G; ++g) {
    float v[NP];
#pragma unroll
    for (int k = 0; k < NP; ++k) v[k] = lane_partial<G>(Q, g, wn[k], wx[k]);
    float r;
    if (NP == 4) {
      const float r0 = __shfl_xor_sync(hmask, b ? v[0] : v[2], 8, 16);
      const float r1 = __shfl_xor_sync(hmask, b ? v[1] : v[3], 8, 16);
      const float k0 = __fadd_rn(b ? v[2] : v[0], r0), k1 = __fadd_rn(b ? v[3] : v[1], r1);
      r = __fadd_rn(c ? k1 : k0, __shfl_xor_sync(hmask, c ? k0 : k1, 4, 16));
    } else {
      r = __fadd_rn(b ? v[1] : v[0], __shfl_xor_sync(hmask, b ? v[0] : v[1], 8, 16));
      r = __fadd_rn(r, __shfl_xor_sync(hmask, r, 4, 16));
    }
    r = __fadd_rn(r, __shfl_xor_sync(hmask, r, 2, 16));
    r = __fadd_rn(r, __shfl_xor_sync(hmask, r, 1, 16));
    total = (g == 0) ? r : __fadd_rn(total, r);
  }
  return total;
}

// Radix select of the K largest of P keys (ties to the lower index), by the
// whole CTA: returns through fx the threshold key and the number of keys
// equal to it that are kept (the lowest-index ones).  Thread t owns the E
// consecutive keys [t E, t E + E); kmin / kmax: the smallest and largest of
// the P keys.  Digits of kTopkDigitBits bits below the keys' common prefix.
// hist: 2^kTopkDigitBits ints (padded), zero on entry and exit.
template <typename KeyAt>
__device__ void topk_threshold(KeyAt key_at, int P, int K, uint32_t kmin, uint32_t kmax, int* hist,
                               SpFixed& fx) {
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int E = (P + kSpThreads - 1) / kSpThreads;
  const int i0 = tid * E, i1 = min(P, i0 + E);
  // the keys share the bits above the highest bit where the smallest and
  // largest differ; the digits start below that common prefix
  int nb = 32 - __clz((int)(kmin ^ kmax));
  uint32_t pmask = nb >= 32 ? 0u : ~((1u << nb) - 1u);
  uint32_t prefix = kmin & pmask;
  int need = K;
#pragma unroll 1
  for (int round = 0; nb > 0; ++round) {
    const int width = min(kTopkDigitBits, nb);
    const int shift = nb - width;
    const uint32_t dm = (1u << width) - 1u;
    nb = shift;
#pragma unroll 1
    for (int c = i0; c < i1; c += 8) {   // eight keys to registers, then their reductions
      uint32_t kv[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) kv[i] = c + i < i1 ? key_at(c + i) : 0u;
#pragma unroll
      for (int i = 0; i < 8; ++i)
        if (c + i < i1 && (kv[i] & pmask) == prefix)
          sm_red_add_u32(smem_u32(hist) + 4u * (uint32_t)sp_pad((int)((kv[i] >> shift) & dm)), 1u);
    }
    __syncthreads();
    // thread t holds digits [t bpt, t bpt + bpt); suffix sums from the top
    const int bins = 1 << width;
    const int bpt = bins > kSpThreads ? bins / kSpThreads : 1;
    const bool holder = tid * bpt < bins;
    int mine = 0;
    if (holder) {
#pragma unroll 1
      for (int k = 0; k < bpt; ++k) mine += (int)sm_ld_u32(smem_u32(&hist[sp_pad(tid * bpt + k)]));
    }
    int incl = mine;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int t = __shfl_down_sync(0xffffffffu, incl, o);
      if (lane + o < 32) incl += t;
    }
    if (lane == 0) fx.scan2[warp].x = incl;
    __syncthreads();
    int above = incl - mine;
#pragma unroll
    for (int w = 0; w < kSpWarps; ++w)
      if (w > warp) above += fx.scan2[w].x;
    // the digit d of the K-th largest key: suffix(d) >= need > suffix(d + 1);
    // when the keys of that digit are exactly the ones still needed, all of
    // them are kept and the search ends here
    if (holder) {
#pragma unroll 1
      for (int k = bpt - 1; k >= 0; --k) {
        const int d = tid * bpt + k;
        const int here = above + (int)sm_ld_u32(smem_u32(&hist[sp_pad(d)]));
        if (here >= need && above < need) {
          fx.sh_d = d;
          fx.sh_need = above;
          fx.blk[0] = here == need ? 1u : 0u;
        }
        above = here;
      }
    }
    __syncthreads();   // every thread is done reading the histogram
    if (holder) {
#pragma unroll 1
      for (int k = 0; k < bpt; ++k) sm_st_u32(smem_u32(&hist[sp_pad(tid * bpt + k)]), 0u);
    }
    need -= fx.sh_need;
    prefix |= (uint32_t)fx.sh_d << shift;
    pmask |= dm << shift;
    const bool whole = fx.blk[0] != 0u;
    __syncthreads();   // sh_d / sh_need / scan2 / blk are rewritten by the next round
    if (whole) {   // keep every key >= prefix: the keys equal to it count as ties, all taken
      need = 0x7FFFFFFF;
      break;
    }
  }
  if (tid == 0) {
    fx.sh_pref = prefix;
    fx.sh_need = need;
  }
  __syncthreads();
}

// ---------------------------------------------------------------------------
// Phase 2 helpers: MMA fragments of the estimate.

__device__ __forceinline__ void sp_mma16816(float (&d)[4], const uint32_t (&a)[4], uint32_t b0,
                                            uint32_t b1) {
  asm(   // no side effects: the compiler may interleave independent tiles
      "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
      "{%8,%9}, {%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// Nibbles e and e+4 of W as the half2 (c_e - 8, c_{e+4} - 8), exact.  A low
// nibble of a byte is masked into the mantissa of 1024 (giving 1024 + c, then
// minus 1032); a high nibble is masked in place (1024 + 16 c, then times 1/16
// minus 72), so bytes 2 and 3 need one shift of W by 8 and no other shifts.
__device__ __forceinline__ uint32_t sp_nib_pair(uint32_t W, int e) {
  const uint32_t src = e >= 2 ? (W >> 8) : W;
  uint32_t r;
  if ((e & 1) == 0) {
    const uint32_t x = (src & 0x000F000Fu) | 0x64006400u;   // 1024 + c
    asm("sub.rn.f16x2 %0, %1, %2;" : "=r"(r) : "r"(x), "r"(0x64086408u));   // minus 1032
  } else {
    const uint32_t x = (src & 0x00F000F0u) | 0x64006400u;   // 1024 + 16 c
    asm("fma.rn.f16x2 %0, %1, %2, %3;" : "=r"(r) : "r"(x), "r"(0x2C002C00u), "r"(0xD480D480u));   // x / 16 - 72
  }
  return r;
}

// 2-bit codes m and m+8 of W as the half2 (c_m - 2, c_{m+8} - 2), exact.
__device__ __forceinline__ uint32_t sp_crumb_pair(uint32_t W, int m) {
  uint32_t x = ((W >> (2 * m)) & 0x00030003u) | 0x64006400u;
  uint32_t r;
  asm("sub.rn.f16x2 %0, %1, %2;" : "=r"(r) : "r"(x), "r"(0x64026402u));   // minus 1026
  return r;
}

template <int BITS>
__device__ __forceinline__ uint32_t sp_code_pair(const uint32_t* W, int s, int j) {
  if (BITS == 4) return sp_nib_pair(W[s >> 1], 2 * (s & 1) + j);
  return sp_crumb_pair(W[s >> 2], 2 * (s & 3) + j);
}

__device__ __forceinline__ uint32_t sp_pack_h2(__half lo, __half hi) {
  return (uint32_t)__half_as_ushort(lo) | ((uint32_t)__half_as_ushort(hi) << 16);
}

// ---------------------------------------------------------------------------
// Phase 2: the threshold search.

struct SpSearch {
  uint32_t prefix, pmask;
  unsigned long long A, T;   // mass above the prefix range; target mass
};

__device__ __forceinline__ unsigned long long sp_mass(float w) {
  return __float2ull_rz(w * kSpMassScale);
}

__device__ __forceinline__ unsigned long long sp_join(uint32_t hi, uint32_t lo) {
  return ((unsigned long long)hi << 32) | lo;
}

// The weights of a selection set live in shared (or global) memory at
// wbuf[wi(lp)] for the CTA's local positions lp; thread t owns the R
// consecutive positions [t R, t R + R) (-1 marks an invalid position).
struct SpWeights {
  float* base;
  bool pad;        // in shared memory, positions padded one word per 32
  uint32_t sbase;  // shared address of base when pad
  int lp0, R, npos;
  __device__ __forceinline__ float at(int i) const {
    const int lp = lp0 + i;
    if (pad) return __uint_as_float(sm_ld_u32(sbase + 4u * (uint32_t)sp_pad(lp)));
    return base[lp];
  }
};

// Histogram the masses of this thread's weights that lie in the current
// prefix range by digit (key >> shift) & dm.  A bin is one 64-bit word
// holding two 32-bit sums: the low kSpLoBits bits of each mass in the low
// half, the rest in the high half, each added by a native 32-bit shared
// reduction (a 64-bit one costs a compare-and-swap loop under contention).
// Neither half overflows: a CTA holds at most kSpSharePages * kPage weights,
// so the low sums stay below 2^(kSpLoBits + 13), and the weights of a set sum
// to about 1, so the high sums stay near 2^(40 - kSpLoBits).  Weights are read
// eight at a time before their reductions.  Histogram word d holds digit
// d + dbase; every weight of nonzero mass has a digit >= dbase.
__device__ __forceinline__ void mass_hist(const SpWeights& W, int shift, uint32_t dm, int dbase,
                                          const SpSearch& s, unsigned long long* hist) {
  const uint32_t h0 = smem_u32(hist);
#pragma unroll 1
  for (int c = 0; c < W.R; c += 8) {
    float wv[8];
#pragma unroll
    for (int i = 0; i < 8; ++i)
      wv[i] = (c + i < W.R && W.lp0 + c + i < W.npos) ? W.at(c + i) : -1.0f;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const uint32_t key = __float_as_uint(wv[i]);
      const unsigned long long m = wv[i] >= 0.f ? sp_mass(wv[i]) : 0ull;
      // a weight of zero mass changes no sum (and lies below digit dbase)
      if (m != 0ull && (key & s.pmask) == s.prefix) {
        const int d = (int)((key >> shift) & dm) - dbase;
        const uint32_t a = h0 + 8u * (uint32_t)sp_pad(d);
        const uint32_t lo = (uint32_t)m & ((1u << kSpLoBits) - 1u), hi = (uint32_t)(m >> kSpLoBits);
        if (lo) sm_red_add_u32(a, lo);
        if (hi) sm_red_add_u32(a + 4u, hi);
      }
    }
  }
}

// The mass of a bin word written by mass_hist.
__device__ __forceinline__ unsigned long long sp_bin_mass(unsigned long long v) {
  return ((v >> 32) << kSpLoBits) + (v & 0xFFFFFFFFull);
}

// The masses of digits base + k * kSpThreads + tid (k < nk) summed over the
// CST CTAs of the cluster and written back, decoded, over this CTA's own
// words of those digits (no peer reads them).  Consecutive threads read
// consecutive words of a peer; nk * CST <= 16, and all of the remote words
// are requested before any is added.
template <int CST>
__device__ __forceinline__ void cluster_bins(unsigned long long* hist, int base, int nk) {
  constexpr int KMAX = 16 / CST;
  const int tid = threadIdx.x;
  unsigned long long v[KMAX][CST];
#pragma unroll
  for (int k = 0; k < KMAX; ++k)
#pragma unroll
    for (int r = 0; r < CST; ++r)
      v[k][r] = k < nk ? ld_peer_u64(peer_addr(&hist[sp_pad(base + k * kSpThreads + tid)], (uint32_t)r))
                       : 0ull;
#pragma unroll
  for (int k = 0; k < KMAX; ++k) {
    unsigned long long t = 0;
#pragma unroll
    for (int r = 0; r < CST; ++r) t += sp_bin_mass(v[k][r]);
    if (k < nk) sm_st_u64(smem_u32(&hist[sp_pad(base + k * kSpThreads + tid)]), t);
  }
}

// One digit of the threshold search (NB digits; NB = 4096 for the first).
// CTA cr owns the slice [cr NB / CS, (cr + 1) NB / CS) of the digits; thread t
// of it reduces bpt consecutive digits of the slice, summed over every CTA of
// the cluster (CS = 1: its own histogram only) and written back over this
// CTA's own words of those digits (no peer reads them).  The mass scan runs
// from the top digit down; the one thread whose digit holds the crossing of
// the target writes it into every CTA.  The first step also sets the target
// from the total mass and returns false if that is zero.  Leaves the low 512
// digits of this CTA's histogram zeroed.
__device__ bool digit_step(const SpWeights& W, int shift, uint32_t dm, int NB, int dbase, double p,
                           int CS, int cr, unsigned long long* hist, SpFixed& fx, SpSearch& s) {
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  mass_hist(W, shift, dm, dbase, s, hist);
  if (CS > 1) cluster_sync();   // every CTA's histogram is complete
  else __syncthreads();
  const int SB = NB / CS;                                    // digits of this CTA's slice
  const int bpt = SB > kSpThreads ? SB / kSpThreads : 1;     // digits per thread (<= 16)
  const int first = cr * SB + tid * bpt;
  const bool holder = tid * bpt < SB;
  // the slice's masses over the cluster, decoded in place: thread t reduces
  // digits cr * SB + k * 256 + t (coalesced), then holds bpt consecutive ones
  if (tid < SB) {
    switch (CS) {
      case 1:
#pragma unroll 1
        for (int k = 0; k < bpt; ++k) {
          const uint32_t ad = smem_u32(&hist[sp_pad(k * kSpThreads + tid)]);
          sm_st_u64(ad, sp_bin_mass(sm_ld_u64(ad)));
        }
        break;
      case 2: cluster_bins<2>(hist, cr * SB, bpt); break;
      case 4: cluster_bins<4>(hist, cr * SB, bpt); break;
      case 8: cluster_bins<8>(hist, cr * SB, bpt); break;
      default: cluster_bins<16>(hist, cr * SB, bpt); break;
    }
  }
  __syncthreads();
  unsigned long long mine = 0;   // this thread's digits' mass
  if (holder) {
#pragma unroll 1
    for (int k = 0; k < bpt; ++k) mine += sm_ld_u64(smem_u32(&hist[sp_pad(first + k)]));
  }
  unsigned long long incl = mine;   // suffix over this warp's higher lanes
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const unsigned long long t = __shfl_down_sync(0xffffffffu, incl, o);
    if (lane + o < 32) incl += t;
  }
  if (lane == 0) fx.wsuf[warp] = incl;
  __syncthreads();
  unsigned long long after = incl - mine;   // digits of this slice above this thread's
  unsigned long long slice = 0;
#pragma unroll
  for (int w2 = 0; w2 < kSpWarps; ++w2) {
    const unsigned long long x = fx.wsuf[w2];
    slice += x;
    if (w2 > warp) after += x;
  }
  unsigned long long total = slice, higher = 0;
  if (CS > 1) {
    if (tid == 0) fx.slice_tot = slice;
    cluster_sync();   // slice totals published; no peer reads this CTA's histogram any more
    unsigned long long t = lane < CS ? ld_peer_u64(peer_addr(&fx.slice_tot, (uint32_t)lane)) : 0ull;
    unsigned long long th = lane > cr ? t : 0ull;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      t += __shfl_xor_sync(0xffffffffu, t, o);
      th += __shfl_xor_sync(0xffffffffu, th, o);
    }
    total = t;
    higher = th;
  }
  bool ok = true;
  if (shift == kSpShift0) {
    if (total == 0) {
      ok = false;
    } else {
      const double tf = ceil((p - kSpMassEps) * (double)total);
      unsigned long long T = tf < 1.0 ? 1ull : (unsigned long long)tf;
      s.T = T > total ? total : T;
    }
  }
  if (ok && holder) {
    // the digit d with A + suffix(d) >= T > A + suffix(d + 1); one thread holds it
    unsigned long long above = s.A + higher + after;
#pragma unroll 1
    for (int k = bpt - 1; k >= 0; --k) {
      const int d = first + k;
      const unsigned long long here = above + sm_ld_u64(smem_u32(&hist[sp_pad(d)]));
      if (here >= s.T && above < s.T) {
        if (CS == 1) {   // this CTA alone (also inside a larger cluster)
          fx.sh_d = d;
          fx.sh_above = above - s.A;
        } else {
          for (int r = 0; r < CS; ++r) {
            st_peer_u32(peer_addr(&fx.sh_d, r), (uint32_t)d);
            st_peer_u64(peer_addr(&fx.sh_above, r), above - s.A);
          }
        }
      }
      above = here;
    }
  }
  __syncthreads();   // every thread is done with the histogram words it holds
  // the later digits (512 bins) need only the low words zeroed; the next set
  // zeroes the whole histogram
  for (int i = tid; i < sp_pad(512); i += kSpThreads) sm_st_u64(smem_u32(&hist[i]), 0ull);
  if (CS > 1) cluster_sync();   // the digit is in every CTA's shared memory
  else __syncthreads();
  if (ok) {
    s.A += fx.sh_above;
    s.prefix |= (uint32_t)(fx.sh_d + dbase) << shift;
    s.pmask |= dm << shift;
  }
  __syncthreads();   // sh_d / sh_above / wsuf are rewritten by the next step
  return ok;
}

// After the first digit: when the weights inside the threshold's digit number
// at most kSpBinList over the cluster, every CTA gathers all of them and runs
// the two remaining digits (9 + 9 bits) on that list alone, with block
// barriers only; otherwise (false, the same in every CTA) the caller runs them
// over the whole set, reduced across the cluster.  Both give the same digits:
// weights outside the first digit never match the prefix.  The CTA's own list
// and the gathered list live in the histogram's storage above the 512 words
// the later digits use (`ring`, at least kSpHistBytes).
__device__ bool resolve_small_bin(const SpWeights& W, SpSearch& s, int CS, double p, SpFixed& fx,
                                  unsigned long long* hist) {
  const int tid = threadIdx.x, lane = tid & 31;
  uint32_t* own = reinterpret_cast<uint32_t*>(hist + kSpListWord);   // this CTA's list
  uint32_t* all = own + kSpBinList;                                  // the gathered list
  if (tid == 0) fx.lst_n = 0;
  __syncthreads();
  auto add = [&](float w) {
    const uint32_t key = __float_as_uint(w);
    if (w >= 0.f && (key & s.pmask) == s.prefix) {
      const int slot = atomicAdd(&fx.lst_n, 1);
      if (slot < kSpBinList) own[slot] = key;
    }
  };
  if (W.pad) {   // shared memory: one weight at a time
#pragma unroll 1
    for (int i = 0; i < W.R && W.lp0 + i < W.npos; ++i) add(W.at(i));
  } else {       // global memory: eight weights loaded, then tested
#pragma unroll 1
    for (int c = 0; c < W.R; c += 8) {
      float wv[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) wv[i] = (c + i < W.R && W.lp0 + c + i < W.npos) ? W.at(c + i) : -1.0f;
#pragma unroll
      for (int i = 0; i < 8; ++i) add(wv[i]);
    }
  }
  if (CS > 1) cluster_sync();   // every CTA's list is complete
  else __syncthreads();
  // every CTA's count (lanes r < CS, in every warp) and their inclusive prefix
  int cnt = 0;
  if (lane < CS) cnt = CS == 1 ? fx.lst_n : (int)ld_peer_u32(peer_addr(&fx.lst_n, (uint32_t)lane));
  int before = cnt;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int t = __shfl_up_sync(0xffffffffu, before, o);
    if (lane >= o) before += t;
  }
  const int n = __shfl_sync(0xffffffffu, before, 31);
  const bool over = __any_sync(0xffffffffu, cnt > kSpBinList);
  if (over || n == 0 || n > kSpBinList) return false;   // uniform over the cluster
  // element t of the concatenated lists: CTA r holds [before_r - cnt_r, before_r)
  int ends[kSpMaxCluster];
#pragma unroll
  for (int r = 0; r < kSpMaxCluster; ++r) ends[r] = __shfl_sync(0xffffffffu, before, r);
  auto fetch = [&](int t) -> uint32_t {
    int src = 0, start = 0;
#pragma unroll
    for (int r = 0; r < kSpMaxCluster; ++r)
      if (r < CS && t >= ends[r]) {
        src = r + 1;
        start = ends[r];
      }
    return CS == 1 ? own[t] : ld_peer_u32(peer_addr(&own[t - start], (uint32_t)src));
  };
  if (n <= 32 * kSpSortPerLane) {
    // one warp: the <= 128 weights (element lane + 32 k in v[k]) sorted
    // descending by a bitonic network, their masses scanned in that order;
    // theta is the weight at which the running mass reaches the target, and
    // the mass of the list's weights above theta joins A
    if (threadIdx.x < 32) {
      constexpr int NK = kSpSortPerLane;
      uint32_t v[NK];
#pragma unroll
      for (int k = 0; k < NK; ++k) v[k] = lane + 32 * k < n ? fetch(lane + 32 * k) : 0u;
#pragma unroll
      for (int size = 2; size <= 32 * NK; size <<= 1) {
#pragma unroll
        for (int stride = size >> 1; stride > 0; stride >>= 1) {
          uint32_t o[NK];
#pragma unroll
          for (int k = 0; k < NK; ++k)
            o[k] = stride >= 32 ? v[k ^ (stride >> 5)] : __shfl_xor_sync(0xffffffffu, v[k], stride);
#pragma unroll
          for (int k = 0; k < NK; ++k) {
            const int e = lane + 32 * k;
            const bool lower = (e & stride) == 0, desc = (e & size) == 0;
            v[k] = (lower == desc) ? max(v[k], o[k]) : min(v[k], o[k]);
          }
        }
      }
      // element e of the sorted order is v[e / 32] of lane e % 32
      unsigned long long F[NK], inc[NK], base = 0ull;
#pragma unroll
      for (int k = 0; k < NK; ++k) {
        F[k] = v[k] ? sp_mass(__uint_as_float(v[k])) : 0ull;
        inc[k] = F[k];
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
          const unsigned long long t = __shfl_up_sync(0xffffffffu, inc[k], o);
          if (lane >= o) inc[k] += t;
        }
        inc[k] += base;
        base = __shfl_sync(0xffffffffu, inc[k], 31);
      }
      uint32_t cut = 0u;
#pragma unroll
      for (int k = 0; k < NK; ++k) {
        const unsigned long long cum = s.A + inc[k];
        if (F[k] && cum >= s.T && cum - F[k] < s.T) cut = v[k];
      }
      const uint32_t theta = __reduce_max_sync(0xffffffffu, cut);   // the one cut (others 0)
      unsigned long long above = 0ull;
#pragma unroll
      for (int k = 0; k < NK; ++k)
        if (v[k] > theta) above += F[k];
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) above += __shfl_xor_sync(0xffffffffu, above, o);
      if (lane == 0) {
        fx.res_theta = theta;
        fx.res_above = above;
      }
    }
    __syncthreads();
    s.prefix = fx.res_theta;
    s.pmask = 0xFFFFFFFFu;
    s.A += fx.res_above;
    return true;
  }
#pragma unroll 1
  for (int t = tid; t < n; t += kSpThreads) all[t] = fetch(t);
  __syncthreads();
  const int Rl = (n + kSpThreads - 1) / kSpThreads;
  const SpWeights L{reinterpret_cast<float*>(all), false, 0u, tid * Rl, Rl, n};
  digit_step(L, 9, 0x1FFu, 512, 0, p, 1, 0, hist, fx, s);
  digit_step(L, 0, 0x1FFu, 512, 0, p, 1, 0, hist, fx, s);
  return true;
}

// ---------------------------------------------------------------------------
template <int G, int BITS>
__global__ void __launch_bounds__(kSpThreads, G <= 4 ? 2 : 1) k_select_prune(SpArgs a) {
  using KW = SpKeyWidth<BITS>;
  extern __shared__ __align__(128) unsigned char sp_smem[];
  SpFixed& fx = *reinterpret_cast<SpFixed*>(sp_smem);
  unsigned char* region = sp_smem + kSpFixedBytes;
  const Layout& L = a.L;
  const int CS = (int)cluster_size(), cr = (int)cluster_rank();
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const bool do_select = a.meta != nullptr, do_prune = a.codes != nullptr;
  const bool paged = L.page_table != nullptr;
  if (tid == 0) {
    for (int s = 0; s < kSpMaxStages; ++s) {
      mbar_init(&fx.full1[s], paged ? kSpWarps * kMetaBulkLanes : 1);   // arrivals with bytes
      mbar_init(&fx.full2[s], kSpThreads);   // every thread's cp.async arrival
    }
    mbar_fence_init();
  }
  __syncthreads();
  griddep_wait();
  // Cluster c takes KV head c % Hk of the sequence of rank c / Hk in the order
  // longest first (ties to the lower index): when the clusters run in more
  // than one wave, the shortest sequences make up the last.
  const int hk = (int)((blockIdx.x / CS) % L.Hk), rb = (int)((blockIdx.x / CS) / L.Hk);
  int b = rb;
  if (L.B > 1 && L.seq_lens) {
#pragma unroll 1
    for (int j = tid; j < L.B; j += kSpThreads) {
      const int lj = L.len(j);
      int rank = 0;
#pragma unroll 1
      for (int i = 0; i < L.B; ++i) {
        const int li = L.len(i);
        rank += li > lj || (li == lj && i < j);
      }
      if (rank == rb) fx.seq = j;
    }
    __syncthreads();
    b = fx.seq;
  }
  const int u = b * L.Hk + hk;
  for (int i = tid; i < G * kHeadDim / 8; i += kSpThreads)   // 16-byte pieces of the G query rows
    reinterpret_cast<uint4*>(&fx.qs[0][0])[i] =
        __ldg(reinterpret_cast<const uint4*>(a.q + ((int64_t)b * a.Hq + hk * G) * kHeadDim) + i);
  __syncthreads();
  const int len = L.len(b);
  const int P = (len + kPage - 1) / kPage;
  int nsel = 0;          // candidate pages of the unit
  int s0 = 0, ns = 0;    // this CTA's share: list entries [s0, s0 + ns)
  bool failed = false;

  if (do_select) {
    // ---------------- phase 1: page scores of pages [pA, pB) ----------------
    const int pA = (int)((int64_t)cr * P / CS), pB = (int)((int64_t)(cr + 1) * P / CS);
    const int npg = pB - pA;
    constexpr int mp = kMetaStagePages;         // page records per stage
    const int nst = (npg + mp - 1) / mp;
    unsigned char* ring = region;
    const size_t stage1 = (size_t)mp * kMetaRecBytes;
    uint32_t* skeys = reinterpret_cast<uint32_t*>(region + (size_t)a.s1 * stage1);
    const bool gk = a.gkeys != nullptr;   // keys in global memory (P above the shared capacity)
    uint32_t* gkeys = gk ? a.gkeys + (int64_t)u * L.max_pages : nullptr;
    const __half* meta = a.meta;
    const int64_t meta_unit = (int64_t)u * L.max_pages;   // contiguous record index of page 0
    // Stage k (up to mp pages of the slice) into ring slot `slot`, completing
    // on the stage's full barrier with its byte count.  A contiguous cache's
    // records of the slice are one run: one bulk copy by thread 0.  A paged
    // cache's records are 512-byte pieces spread over the pool: one bulk copy
    // per record from warp 0 (pool pages from the staged page-table entries);
    // few large requests instead of 16-byte pieces from every thread.
    // lane i of a warp: the page-table entries of pages i and i + 32 of stage
    // k (0 past the slice), as loaded; nothing uses them until store_pt, so
    // the load's latency is not waited for here
    auto fetch_pt = [&](int k) -> int2 {
      int e[2] = {0, 0};
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const int pg = pA + k * mp + lane + 32 * h;
        if (paged && k < nst && lane + 32 * h < mp && pg < pB)
          e[h] = L.page_table[(int64_t)b * L.max_pages + pg];
      }
      return make_int2(e[0], e[1]);
    };
    // pool pages of the stage into the slot (an id outside the pool reads pool page 0)
    auto store_pt = [&](int slot, int2 e) {
      fx.pt1[slot][lane] = (unsigned)e.x < (unsigned)L.pool_pages ? e.x : 0;
      constexpr int kHi = kMetaStagePages > 32 ? 32 : 0;   // the second half of a 64-page stage
      if (kHi) fx.pt1[slot][lane + kHi] = (unsigned)e.y < (unsigned)L.pool_pages ? e.y : 0;
    };
    auto issue1 = [&](int k, int slot) {
      const int n = k < nst ? min(mp, npg - k * mp) : 0;
      unsigned char* dst = ring + (size_t)slot * stage1;
      if (paged) {
        // one bulk copy per page record, spread over the warps: lane j < 8 of
        // warp w copies page 8 w + j (mp <= 64), arriving on the stage's
        // barrier with its bytes (0 past the stage) before issuing the copy
        const int i = warp * 8 + lane;
        if (lane < kMetaBulkLanes) {
          mbar_arrive_tx(&fx.full1[slot], i < n ? 512u : 0u);
          if (i < n) {
            fence_proxy_async();   // the slot's earlier readers are ordered before the copy
            bulk_g2s(dst + i * 512, meta + ((int64_t)fx.pt1[slot][i] * L.Hk + hk) * (2 * kHeadDim),
                     512u, &fx.full1[slot]);
          }
        }
      } else if (tid == 0) {
        fence_proxy_async();   // the slot's earlier readers are ordered before the copy
        if (n > 0)
          bulk_g2s(dst, meta + (meta_unit + pA + (int64_t)k * mp) * (2 * kHeadDim),
                   (uint32_t)n * 512u, &fx.full1[slot]);
        mbar_arrive_tx(&fx.full1[slot], (uint32_t)n * 512u);
      }
    };
    // page-table entries: stages 0 .. S-1 staged now.  The entries of stage
    // k >= S are loaded by warp k % 8 into its registers kPtAhead iterations
    // before they are stored (at the end of iteration k - S, into the slot
    // stage k - S used), so a load's latency spreads over several iterations
    // and no barrier waits on one.
    int2 ptn = make_int2(0, 0);
    if (paged) {
      if (warp == 0) {
        int2 ptq[kSpMaxStages];
#pragma unroll
        for (int k = 0; k < kSpMaxStages; ++k) ptq[k] = k < a.s1 ? fetch_pt(k) : make_int2(0, 0);
#pragma unroll
        for (int k = 0; k < kSpMaxStages; ++k)
          if (k < a.s1) store_pt(k, ptq[k]);
      }
#pragma unroll 1
      for (int i = 0; i < kPtAhead; ++i)
        if (warp == (a.s1 + i) % kSpWarps) ptn = fetch_pt(a.s1 + i);
    }
    __syncthreads();
#pragma unroll 1
    for (int k = 0; k < a.s1 - 1; ++k) issue1(k, k);
    // the query channels of this lane (8 per head) for the group's heads
    const int l16 = lane & 15, hw = tid >> 4;
    const unsigned hmask = 0xFFFFu << (lane & 16);
    ScoreQ<G> Q;
#pragma unroll
    for (int g = 0; g < G; ++g) {
      const uint4 r = *reinterpret_cast<const uint4*>(&fx.qs[g][l16 * 8]);
      const uint32_t wq[4] = {r.x, r.y, r.z, r.w};
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        const unsigned short hbits = h_part(wq[j >> 1], j & 1);
        const float x = sp_h(wq[j >> 1], j & 1);
        if (ScoreQ<G>::kSplit) {
          const int gs = ScoreQ<G>::kSplit ? g : 0;
          const uint32_t sh = 16u * (uint32_t)(j & 1);
          if (!(j & 1)) Q.ap[gs][j >> 1] = Q.an[gs][j >> 1] = 0u;
          // q+ (+0 when q < 0) and q- (+0 when q >= 0)
          Q.ap[gs][j >> 1] |= (uint32_t)(x >= 0.f ? hbits : (unsigned short)0) << sh;
          Q.an[gs][j >> 1] |= (uint32_t)(x >= 0.f ? (unsigned short)0 : hbits) << sh;
        } else {
          Q.a[ScoreQ<G>::kSplit ? 0 : g][j] = x;
        }
      }
    }
    uint32_t kmin = 0xFFFFFFFFu, kmax = 0u;   // over the keys this lane computed
    for (int j = 0; j < nst; ++j) {
      // refill: stage j + S - 1 into the slot stage j - 1 used (freed by the
      // barrier that ended the previous iteration); then the page-table
      // entries of stage j + S into the slot stage j's entries used
      issue1(j + a.s1 - 1, (j + a.s1 - 1) % a.s1);
      const int slot = j % a.s1;
      const uint32_t par = (uint32_t)((j / a.s1) & 1);
      if (!failed) failed = !mbar_wait(&fx.full1[slot], par, a.status);
      const int n = min(mp, npg - j * mp);
      const unsigned char* st = ring + (size_t)slot * stage1;
      // every page of the stage is scored (records past n are stale and
      // their scores unused); lane l16 then holds page hw + 16 kp (+ 32 for
      // the second pass of G >= 4, which takes two pages per half-warp at a
      // time to stay in registers), shared with the other lanes of its group,
      // which split the stores
      auto emit = [&](float score, int i, int rr, int step) {
        if (i < n) {
          const uint32_t key = f_key(score);
          kmin = min(kmin, key);
          kmax = max(kmax, key);
          const int pg = pA + j * mp + i;
          if (gk) {
            if (rr == 0) gkeys[pg] = key;
          } else {
            for (int r = rr; r < CS; r += step) st_peer_u32(peer_addr(&skeys[sp_pad(pg)], (uint32_t)r), key);
          }
        }
      };
      if (kMetaStagePages == 32 || G >= 4) {
#pragma unroll
        for (int half = 0; half < kMetaStagePages / 32; ++half)
          emit(page_scores<G, 2>(Q, st + half * 32 * kMetaRecBytes, hw, l16, hmask),
               hw + 16 * ((l16 >> 3) & 1) + 32 * half, l16 & 7, 8);
      } else {
        emit(page_scores<G, 4>(Q, st, hw, l16, hmask), hw + 16 * ((l16 >> 2) & 3), l16 & 3, 4);
      }
      // the entries of stage j + S go where stage j's were (read when stage j
      // was issued, S - 1 iterations ago); stage j + S + kPtAhead's are loaded
      if (paged) {
        if (warp == (j + a.s1) % kSpWarps) store_pt(j % a.s1, ptn);
        if (warp == (j + a.s1 + kPtAhead) % kSpWarps) ptn = fetch_pt(j + a.s1 + kPtAhead);
      }
      __syncthreads();   // slot j is free; the staged entries are visible
    }
    // every warp's smallest and largest key, into every CTA
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      kmin = min(kmin, __shfl_xor_sync(0xffffffffu, kmin, o));
      kmax = max(kmax, __shfl_xor_sync(0xffffffffu, kmax, o));
    }
    if (lane < CS) {
      st_peer_u32(peer_addr(&fx.kmin[cr * kSpWarps + warp], (uint32_t)lane), kmin);
      st_peer_u32(peer_addr(&fx.kmax[cr * kSpWarps + warp], (uint32_t)lane), kmax);
    }
    cluster_sync();   // every CTA holds all P keys (or they are in global memory)
    {
      const int nw = CS * kSpWarps;   // <= 128: four per lane
#pragma unroll
      for (int x = 0; x < 4; ++x) {
        const int i = lane + 32 * x;
        if (i < nw) {
          kmin = min(kmin, fx.kmin[i]);
          kmax = max(kmax, fx.kmax[i]);
        }
      }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) {
        kmin = min(kmin, __shfl_xor_sync(0xffffffffu, kmin, o));
        kmax = max(kmax, __shfl_xor_sync(0xffffffffu, kmax, o));
      }
    }

    // ---------------- top-K_p and this CTA's share of the candidate list ----------------
    const int K = min(a.budget_pages, P);
    const uint32_t skeys_s = smem_u32(skeys);
    auto key_at = [&](int i) -> uint32_t {
      return gk ? __ldcg(gkeys + i) : sm_ld_u32(skeys_s + 4u * (uint32_t)sp_pad(i));
    };
    int* hist = reinterpret_cast<int*>(ring);   // the meta ring is idle now
    for (int i = tid; i < sp_pad(1 << kTopkDigitBits); i += kSpThreads) hist[i] = 0;
    __syncthreads();
    const bool all = K >= P;
    if (!all) topk_threshold(key_at, P, K, kmin, kmax, hist, fx);
    const uint32_t thr = all ? 0u : fx.sh_pref;
    const int need = all ? 0 : fx.sh_need;
    const int E = (P + kSpThreads - 1) / kSpThreads;
    const int i0 = tid * E, i1 = min(P, i0 + E);
    // bit i - c of the masks: key i of the chunk [c, c + 32) above / at the
    // threshold; the first chunk's masks are kept for the second pass (a
    // thread has one chunk unless P > 8192)
    auto chunk_masks = [&](int c, uint32_t& gtm, uint32_t& eqm) {
      gtm = eqm = 0u;
      const int ce = min(i1, c + 32);
#pragma unroll 1
      for (int i = c; i < ce; ++i) {
        const uint32_t k = all ? 1u : key_at(i);
        if (all || k > thr) gtm |= 1u << (i - c);
        else if (k == thr) eqm |= 1u << (i - c);
      }
    };
    uint32_t gtm0, eqm0;
    chunk_masks(i0, gtm0, eqm0);
    int n_gt = __popc(gtm0), n_eq = __popc(eqm0);
#pragma unroll 1
    for (int c = i0 + 32; c < i1; c += 32) {
      uint32_t g, e;
      chunk_masks(c, g, e);
      n_gt += __popc(g);
      n_eq += __popc(e);
    }
    int2 tot;
    const int2 ex = sp_scan2(make_int2(n_gt, n_eq), fx.scan2, &tot);
    nsel = K;
    s0 = (int)((int64_t)cr * K / CS);
    ns = (int)((int64_t)(cr + 1) * K / CS) - s0;
    // the kept keys: all above, and the lowest-index ones at the threshold
    int take = ex.y < need ? min(n_eq, need - ex.y) : 0;
    int pos = ex.x + min(need, ex.y);
    int32_t* cand_u = a.cand + (int64_t)u * a.cand_stride;
#pragma unroll 1
    for (int c = i0; c < i1; c += 32) {
      uint32_t sel = gtm0, m = eqm0;
      if (c != i0) chunk_masks(c, sel, m);
#pragma unroll 1
      for (; take > 0 && m; --take) {
        sel |= m & (0u - m);
        m &= m - 1;
      }
#pragma unroll 1
      while (sel) {
        const int i = c + __ffs(sel) - 1;
        sel &= sel - 1;
        if (pos >= s0 && pos < s0 + ns) {
          fx.pg[pos - s0] = (uint32_t)i;
          cand_u[pos] = i;
        }
        ++pos;
      }
    }
    if (cr == 0 && tid == 0) a.ncand[u] = K;
    __syncthreads();
  } else {
    // ---------------- caller's candidate pages, or every page ----------------
    if (a.cand) {
      const int lim = min(a.cand_stride, L.max_pages);
      nsel = max(0, min(a.ncand[u], lim));
    } else {
      nsel = P;
    }
    s0 = (int)((int64_t)cr * nsel / CS);
    ns = (int)((int64_t)(cr + 1) * nsel / CS) - s0;
    for (int i = tid; i < ns; i += kSpThreads)
      fx.pg[i] = a.cand ? (uint32_t)a.cand[(int64_t)u * a.cand_stride + s0 + i] : (uint32_t)(s0 + i);
    __syncthreads();
  }
  // physical rows of the share's pages (page ids outside the sequence: no rows)
  for (int i = tid; i < ns; i += kSpThreads) {
    const int pg = (int)fx.pg[i];
    const bool valid = pg >= 0 && pg < P;
    fx.nrow[i] = valid ? min(kPage, len - pg * kPage) : 0;
    fx.crow[i] = !valid ? 0 : ((!paged && pg * kPage + kPage > L.N) ? L.N - pg * kPage : kPage);
    fx.r0[i] = valid ? (uint32_t)L.page_row(b, hk, pg) : 0u;
  }
  __syncthreads();

  if (do_prune) {
    // ---------------- phase 2: weight estimate of the share ----------------
    const int nst = (ns + kEstStagePages - 1) / kEstStagePages;
    unsigned char* ring = region;
    const int ring_bytes = max(a.s2 * KW::kStageBytes, kSpHistBytes);
    // logits [head][local position]: in shared memory (positions padded one
    // word per 32, so a thread's run of R consecutive positions is free of
    // bank conflicts) or at the set's positions [s0 * 16, ..) of the global
    // logits
    float* lbase;
    int64_t hstride;
    const bool lpad = a.glogits == nullptr;
    if (!lpad) {
      lbase = a.glogits + (int64_t)u * G * a.lcap + (int64_t)s0 * kPage;
      hstride = a.lcap;
    } else {
      lbase = reinterpret_cast<float*>(region + ring_bytes);
      hstride = sp_pad(a.share_cap * kPage);
    }
    auto lidx = [&](int h, int lp) -> int64_t { return h * hstride + (lpad ? sp_pad(lp) : lp); };
    const uint8_t* codes = a.codes;
    const __half* scales = a.scales;
    const __half* zeros = a.zeros;
    // Stage k of the share (up to 16 candidate pages) into ring slot `slot`,
    // by all threads with cp.async: the pages' code rows in 16-byte pieces,
    // their scale and zero rows in 8-byte pieces; every thread then arrives
    // on the stage's full barrier when its copies have landed.  Rows copied
    // per page: the whole page, except where it runs past a contiguous
    // cache's allocation (length not a multiple of 16); pages outside the
    // sequence copy nothing.
    auto issue2 = [&](int k, int slot) {
      if (k < nst) {
        const int npgs = min(kEstStagePages, ns - k * kEstStagePages);
        unsigned char* st = ring + (size_t)slot * KW::kStageBytes;
        unsigned char* st_codes = st;
        unsigned char* st_scales = st + kEstStageTok * KW::kRowBytes;
        unsigned char* st_zeros = st_scales + kEstStageTok * kGroups * 2;
        constexpr int kPieces = KW::kRowBytes;   // 16-byte pieces of a page's code rows
#pragma unroll
        for (int x0 = 0; x0 < kEstStagePages * kPieces; x0 += kSpThreads) {
          const int x = x0 + tid, pi = x / kPieces, c = x % kPieces;
          if (pi < npgs) {
            const int e = k * kEstStagePages + pi;
            if (16 * c < fx.crow[e] * KW::kRowBytes)
              cp_async16_sm(st_codes + pi * kPage * KW::kRowBytes + 16 * c,
                            codes + (size_t)fx.r0[e] * KW::kRowBytes + 16 * c);
          }
        }
        {
          const int pi = tid >> 4, r = tid & 15;
          if (pi < npgs) {
            const int e = k * kEstStagePages + pi;
            if (r < fx.crow[e]) {
              cp_async8_sm(st_scales + tid * 8, scales + ((size_t)fx.r0[e] + r) * kGroups);
              cp_async8_sm(st_zeros + tid * 8, zeros + ((size_t)fx.r0[e] + r) * kGroups);
            }
          }
        }
      }
      cp_async_arrive_noinc(&fx.full2[slot]);
    };
#pragma unroll 1
    for (int k = 0; k < a.s2 - 1; ++k) issue2(k, k);
    constexpr int HP = (G + 1) / 2;   // head pairs: one MMA N-block of 8 (head, group) columns each
    const int gid = lane >> 2, t = lane & 3;
    const int g0 = 2 * (t & 1);
    uint32_t bfr[HP][8][2];
    float Qv[HP][2];
#pragma unroll
    for (int hp = 0; hp < HP; ++hp) {
      const int hb = 2 * hp + (gid >> 2);
      const bool on = ((gid & 3) == t) && hb < G;
      const __half* qb = fx.qs[min(hb, G - 1)];
      const __half z = __float2half_rn(0.f);
      const __half* qg = qb + kGroup * t;
#pragma unroll
      for (int s = 0; s < 8; ++s)
#pragma unroll
        for (int jj = 0; jj < 2; ++jj)
          bfr[hp][s][jj] = sp_pack_h2(on ? qg[KW::chan(s, jj, 0)] : z, on ? qg[KW::chan(s, jj, 1)] : z);
      const int he = 2 * hp + (t >> 1);
      const __half* qe = fx.qs[min(he, G - 1)];
      float q0 = 0.f, q1 = 0.f;
      for (int d = 0; d < kGroup; ++d) {
        q0 += __half2float(qe[g0 * kGroup + d]);
        q1 += __half2float(qe[(g0 + 1) * kGroup + d]);
      }
      Qv[hp][0] = q0;
      Qv[hp][1] = q1;
    }
    float Mrun[HP], Zrun[HP];   // this lane's head (he) running statistics, owner lanes
#pragma unroll
    for (int hp = 0; hp < HP; ++hp) {
      Mrun[hp] = -INFINITY;
      Zrun[hp] = 0.f;
    }
    const bool owner = (t & 1) == 0;   // lanes t and t^1 hold the same logits
    for (int j = 0; j < nst; ++j) {
      // refill: stage j + S - 1 into the slot stage j - 1 used (freed by the
      // barrier that ended the previous iteration)
      issue2(j + a.s2 - 1, (j + a.s2 - 1) % a.s2);
      const int slot = j % a.s2;
      const uint32_t par = (uint32_t)((j / a.s2) & 1);
      if (!failed) failed = !mbar_wait(&fx.full2[slot], par, a.status);
      const unsigned char* st = ring + (size_t)slot * KW::kStageBytes;
      const unsigned char* st_codes = st;
      const __half* st_scales = reinterpret_cast<const __half*>(st + kEstStageTok * KW::kRowBytes);
      const __half* st_zeros = st_scales + kEstStageTok * kGroups;
      float lg[2][HP][2];
#pragma unroll
      for (int k = 0; k < 2; ++k) {
        const int ca = warp * 32 + k * 16 + gid, cb = ca + 8;   // rows gid, gid + 8 of the tile
        uint32_t WA[4], WB[4];
        if (BITS == 4) {
          const uint4 wa = *reinterpret_cast<const uint4*>(st_codes + ca * KW::kRowBytes + KW::kLaneBytes * t);
          const uint4 wb = *reinterpret_cast<const uint4*>(st_codes + cb * KW::kRowBytes + KW::kLaneBytes * t);
          WA[0] = wa.x, WA[1] = wa.y, WA[2] = wa.z, WA[3] = wa.w;
          WB[0] = wb.x, WB[1] = wb.y, WB[2] = wb.z, WB[3] = wb.w;
        } else {
          const uint2 wa = *reinterpret_cast<const uint2*>(st_codes + ca * KW::kRowBytes + KW::kLaneBytes * t);
          const uint2 wb = *reinterpret_cast<const uint2*>(st_codes + cb * KW::kRowBytes + KW::kLaneBytes * t);
          WA[0] = wa.x, WA[1] = wa.y, WA[2] = WA[3] = 0u;
          WB[0] = wb.x, WB[1] = wb.y, WB[2] = WB[3] = 0u;
        }
        const int ea = j * kEstStagePages + (ca >> 4), eb = j * kEstStagePages + (cb >> 4);
        const bool va = ea < ns && (ca & 15) < fx.nrow[ea];
        const bool vb = eb < ns && (cb & 15) < fx.nrow[eb];
        // two accumulator chains (even and odd K-steps) halve the dependent MMA chain
        float acc[HP][4], acc2[HP][4];
#pragma unroll
        for (int hp = 0; hp < HP; ++hp)
#pragma unroll
          for (int i = 0; i < 4; ++i) acc[hp][i] = acc2[hp][i] = 0.f;
#pragma unroll
        for (int s = 0; s < 8; ++s) {
          const uint32_t af[4] = {sp_code_pair<BITS>(WA, s, 0), sp_code_pair<BITS>(WB, s, 0),
                                  sp_code_pair<BITS>(WA, s, 1), sp_code_pair<BITS>(WB, s, 1)};
#pragma unroll
          for (int hp = 0; hp < HP; ++hp)
            sp_mma16816((s & 1) ? acc2[hp] : acc[hp], af, bfr[hp][s][0], bfr[hp][s][1]);
        }
#pragma unroll
        for (int hp = 0; hp < HP; ++hp)
#pragma unroll
          for (int i = 0; i < 4; ++i) acc[hp][i] += acc2[hp][i];
        const float2 fsa = __half22float2(*reinterpret_cast<const __half2*>(&st_scales[ca * kGroups + g0]));
        const float2 fza = __half22float2(*reinterpret_cast<const __half2*>(&st_zeros[ca * kGroups + g0]));
        const float2 fsb = __half22float2(*reinterpret_cast<const __half2*>(&st_scales[cb * kGroups + g0]));
        const float2 fzb = __half22float2(*reinterpret_cast<const __half2*>(&st_zeros[cb * kGroups + g0]));
        const float zza0 = __fmaf_rn(KW::kCentre, fsa.x, fza.x);
        const float zza1 = __fmaf_rn(KW::kCentre, fsa.y, fza.y);
        const float zzb0 = __fmaf_rn(KW::kCentre, fsb.x, fzb.x);
        const float zzb1 = __fmaf_rn(KW::kCentre, fsb.y, fzb.y);
#pragma unroll
        for (int hp = 0; hp < HP; ++hp) {
          float pa = __fmaf_rn(fsa.x, acc[hp][0], zza0 * Qv[hp][0]);
          pa = __fmaf_rn(fsa.y, acc[hp][1], __fmaf_rn(zza1, Qv[hp][1], pa));
          float pb = __fmaf_rn(fsb.x, acc[hp][2], zzb0 * Qv[hp][0]);
          pb = __fmaf_rn(fsb.y, acc[hp][3], __fmaf_rn(zzb1, Qv[hp][1], pb));
          pa += __shfl_xor_sync(0xffffffffu, pa, 1);   // + the other two groups
          pb += __shfl_xor_sync(0xffffffffu, pb, 1);
          lg[k][hp][0] = va ? pa * kEstL2Scale : -INFINITY;
          lg[k][hp][1] = vb ? pb * kEstL2Scale : -INFINITY;
        }
      }
      const int cw0 = j * kEstStageTok + warp * 32;   // this warp's first local position
#pragma unroll
      for (int hp = 0; hp < HP; ++hp) {
        const int he = 2 * hp + (t >> 1);
        const bool hv = he < G;
        if (owner && hv) {
#pragma unroll
          for (int k = 0; k < 2; ++k) {
            const int c0 = cw0 + k * 16 + gid;
            if (c0 < ns * kPage) lbase[lidx(he, c0)] = lg[k][hp][0];
            if (c0 + 8 < ns * kPage) lbase[lidx(he, c0 + 8)] = lg[k][hp][1];
          }
        }
        // this lane's running (max, sum 2^(l - max)) over its own logits; the
        // lanes are merged once after the stream
        if (owner && hv) {
          const float m = fmaxf(fmaxf(lg[0][hp][0], lg[0][hp][1]), fmaxf(lg[1][hp][0], lg[1][hp][1]));
          if (m != -INFINITY) {
            const float mn = fmaxf(Mrun[hp], m);
            float z = Mrun[hp] == -INFINITY ? 0.f : Zrun[hp] * exp2f(Mrun[hp] - mn);
#pragma unroll
            for (int k = 0; k < 2; ++k) z += exp2f(lg[k][hp][0] - mn) + exp2f(lg[k][hp][1] - mn);
            Zrun[hp] = z;
            Mrun[hp] = mn;
          }
        }
      }
      __syncthreads();   // every warp is done with this slot before it is refilled
    }
    // merge the lanes' pairs of each head (lanes of one head differ in bits 2..4)
#pragma unroll
    for (int hp = 0; hp < HP; ++hp) {
      float m = Mrun[hp], z = Zrun[hp];
#pragma unroll
      for (int o = 4; o < 32; o <<= 1) {
        const float mo = __shfl_xor_sync(0xffffffffu, m, o), zo = __shfl_xor_sync(0xffffffffu, z, o);
        const float mn = fmaxf(m, mo);
        z = (m == -INFINITY ? 0.f : z * exp2f(m - mn)) + (mo == -INFINITY ? 0.f : zo * exp2f(mo - mn));
        m = mn;
      }
      Mrun[hp] = m;
      Zrun[hp] = z;
    }
    // per-warp statistics -> the CTA's -> every CTA's, merged in rank order
#pragma unroll
    for (int hp = 0; hp < HP; ++hp) {
      const int he = 2 * hp + (t >> 1);
      if (gid == 0 && owner && he < G) fx.wstat[warp][he] = make_float2(Mrun[hp], Zrun[hp]);
    }
    __syncthreads();
    if (tid < G) {
      float m = -INFINITY;
#pragma unroll
      for (int w = 0; w < kSpWarps; ++w) m = fmaxf(m, fx.wstat[w][tid].x);
      float z = 0.f;
#pragma unroll
      for (int w = 0; w < kSpWarps; ++w) {
        const float2 x = fx.wstat[w][tid];
        if (x.x != -INFINITY) z += x.y * exp2f(x.x - m);
      }
      fx.mz_loc[tid] = make_float2(m, z);
    }
    __syncthreads();
    if (tid < G * CS) {
      const int h = tid % G, r = tid / G;
      st_peer_f2(peer_addr(&fx.mz_all[cr][h], (uint32_t)r), fx.mz_loc[h]);
    }
    cluster_sync();
    float Mh[G], iZ[G];
#pragma unroll
    for (int h = 0; h < G; ++h) {
      float m = -INFINITY;
      for (int r = 0; r < CS; ++r) m = fmaxf(m, fx.mz_all[r][h].x);
      float z = 0.f;
      for (int r = 0; r < CS; ++r) {
        const float2 x = fx.mz_all[r][h];
        if (x.x != -INFINITY) z += x.y * exp2f(x.x - m);
      }
      Mh[h] = m;
      iZ[h] = z > 0.f ? 1.0f / z : 0.f;
    }

    // ---------------- top-p per selection set ----------------
    // the estimate ring is idle now: the digit histogram (and the small-bin work space)
    unsigned long long* hist = reinterpret_cast<unsigned long long*>(ring);
    const int npos = ns * kPage;                                  // local positions of the share
    const int R = (npos + kSpThreads - 1) / kSpThreads;   // <= 32 (host-checked)
    const int lp0 = tid * R;
    const int nsets_u = a.group_sets ? 1 : G;
    for (int hs = 0; hs < nsets_u; ++hs) {
      const int set = a.group_sets ? u : b * a.Hq + hk * G + hs;
      const int h0 = a.group_sets ? 0 : hs, nh = a.group_sets ? G : 1;
      __syncthreads();   // the ring (or the previous set's staged output) is free
      for (int i = tid; i < kSpHistWords; i += kSpThreads) hist[i] = 0ull;
      // The set's weights.  Logits in shared memory: written over the logits
      // of the set's first head, each thread on its own positions.  Logits in global memory: read with consecutive
      // threads on consecutive positions, and the weights written to shared
      // memory above the histogram when the idle ring has room (else over
      // the first head's logits); the search then reads them from there.
      const bool wsm = !lpad && ring_bytes >= kSpHistBytes + sp_pad(npos) * 4;
      float* wb = lpad ? lbase + h0 * hstride
                       : (wsm ? reinterpret_cast<float*>(ring + kSpHistBytes) : lbase + h0 * hstride);
      SpWeights W{wb, lpad || wsm, (lpad || wsm) ? smem_u32(wb) : 0u, lp0, R, npos};
      auto weight = [&](int lp, const float (&l)[G]) -> float {
        if ((lp & 15) >= fx.nrow[lp >> 4]) return -1.0f;
        float acc = 0.f;
#pragma unroll
        for (int h = 0; h < G; ++h)
          if (h >= h0 && h < h0 + nh) acc += exp2f(l[h] - Mh[h]) * iZ[h];
        if (nh > 1) acc *= 1.0f / (float)nh;
        return acc;
      };
      if (lpad) {
#pragma unroll 1
        for (int i = 0; i < R; ++i) {
          const int lp = lp0 + i;
          if (lp >= npos) break;
          float lv[G];
#pragma unroll
          for (int h = 0; h < G; ++h) lv[h] = (h >= h0 && h < h0 + nh) ? lbase[lidx(h, lp)] : 0.f;
          lbase[lidx(h0, lp)] = weight(lp, lv);
        }
      } else {
        constexpr int CH = G >= 8 ? 2 : 4;
#pragma unroll 1
        for (int lp0c = 0; lp0c < npos; lp0c += CH * kSpThreads) {
          float lv[CH][G];
#pragma unroll
          for (int i = 0; i < CH; ++i) {
            const int lp = lp0c + i * kSpThreads + tid;
#pragma unroll
            for (int h = 0; h < G; ++h)
              lv[i][h] = (lp < npos && h >= h0 && h < h0 + nh) ? lbase[lidx(h, lp)] : 0.f;
          }
#pragma unroll
          for (int i = 0; i < CH; ++i) {
            const int lp = lp0c + i * kSpThreads + tid;
            if (lp >= npos) break;
            const float w = weight(lp, lv[i]);
            if (wsm) sm_st_u32(W.sbase + 4u * (uint32_t)sp_pad(lp), __float_as_uint(w));
            else lbase[lidx(h0, lp)] = w;
          }
        }
        __syncthreads();   // the search reads positions other threads wrote
      }
      const bool keep_all = a.p >= 1.0;
      uint32_t theta = 0;
      unsigned long long r_need = 0;
      bool have = false;
      if (!keep_all) {
        SpSearch sr{0u, 0u, 0ull, 0ull};
        // digits of the 30-bit weight key: bits 29..18, 17..9, 8..0
        bool done_small = false;
#pragma unroll 1
        for (int step = 0; step < 3; ++step) {
          const bool ok = digit_step(W, step == 0 ? kSpShift0 : (step == 1 ? 9 : 0),
                                     step == 0 ? 0xFFFu : 0x1FFu, step == 0 ? kSpBins0 : 512,
                                     step == 0 ? kSpDigit0Base : 0, a.p, CS, cr, hist, fx, sr);
          if (step == 0) {
            have = ok;
            if (have) done_small = resolve_small_bin(W, sr, CS, a.p, fx, hist);
          }
          if (!have || done_small) break;   // the same in every CTA of the cluster
        }
        if (have) {
          theta = sr.prefix;
          unsigned long long Ft = sp_mass(__uint_as_float(theta));
          if (Ft == 0) Ft = 1;
          r_need = (sr.T - sr.A + Ft - 1) / Ft;
        }
      }
      // compaction in ascending position order: bit i of gtm / eqm marks
      // local position lp0 + i above / at theta
      unsigned gtm = 0, eqm = 0;
      auto mark = [&](int i, float w) {
        if (w < 0.f) return;
        const uint32_t key = __float_as_uint(w);
        if (keep_all || (have && key > theta)) gtm |= 1u << i;
        else if (have && key == theta) eqm |= 1u << i;
      };
      if (W.pad) {   // shared memory: one weight at a time
#pragma unroll 1
        for (int i = 0; i < R && lp0 + i < npos; ++i) mark(i, W.at(i));
      } else {       // global memory: eight weights loaded, then tested
#pragma unroll 1
        for (int c = 0; c < R; c += 8) {
          float wv[8];
#pragma unroll
          for (int i = 0; i < 8; ++i) wv[i] = (c + i < R && lp0 + c + i < npos) ? W.at(c + i) : -1.0f;
#pragma unroll
          for (int i = 0; i < 8; ++i) mark(c + i, wv[i]);
        }
      }
      const unsigned n_gt = __popc(gtm), n_eq = __popc(eqm);
      unsigned blk_total;
      const unsigned ex = sp_scan((n_gt << 16) | n_eq, fx.scan, &blk_total);
      unsigned gt_before = 0, eq_before = 0, gt_all = blk_total >> 16, eq_all = blk_total & 0xFFFFu;
      if (CS > 1) {
        if (tid == 0) {
          fx.blk[0] = blk_total >> 16;
          fx.blk[1] = blk_total & 0xFFFFu;
        }
        cluster_sync();
        if (warp == 0) {
          unsigned g = 0, e = 0, gb = 0, eb = 0;
          if (lane < CS) {
            g = ld_peer_u32(peer_addr(&fx.blk[0], (uint32_t)lane));
            e = ld_peer_u32(peer_addr(&fx.blk[1], (uint32_t)lane));
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
            fx.pre[0] = gb;
            fx.pre[1] = eb;
            fx.pre[2] = g;
            fx.pre[3] = e;
          }
        }
        __syncthreads();
        gt_before = fx.pre[0];
        eq_before = fx.pre[1];
        gt_all = fx.pre[2];
        eq_all = fx.pre[3];
      }
      const unsigned long long ties_before = (unsigned long long)eq_before + (ex & 0xFFFFu);
      unsigned take = 0;
      if (ties_before < r_need) take = (unsigned)min((unsigned long long)n_eq, r_need - ties_before);
      const unsigned first = gt_before + (unsigned)min(r_need, (unsigned long long)eq_before);
      const unsigned lpos0 = (ex >> 16) + (unsigned)min(r_need, ties_before) -
                             (unsigned)min(r_need, (unsigned long long)eq_before);
      unsigned sel = gtm;   // and the `take` lowest positions at theta
      {
        unsigned m = eqm;
#pragma unroll 1
        for (unsigned t = 0; t < take; ++t) {
          sel |= m & (0u - m);
          m &= m - 1;
        }
      }
      {
        // The thread's kept positions are consecutive outputs from lpos0 on.
        // They are staged in shared memory (the histogram's storage: ids,
        // then rows) when the CTA's outputs fit it, and copied out with
        // consecutive threads on consecutive words; else each thread stores
        // its own run.
        int32_t* oidx = a.idx + (int64_t)set * a.icap + first;
        uint32_t* orow = a.rows ? a.rows + (int64_t)set * a.icap + first : nullptr;
        const unsigned eq_blk = blk_total & 0xFFFFu;
        const unsigned n_out = (blk_total >> 16) +
            (r_need > eq_before ? (unsigned)min((unsigned long long)eq_blk, r_need - eq_before) : 0u);
        const bool staged = 2 * npos * 4 <= ring_bytes;   // uniform in the CTA
        uint32_t* sidx = reinterpret_cast<uint32_t*>(ring);
        uint32_t* srow = sidx + npos;
        unsigned m = sel;
#pragma unroll 1
        for (unsigned o = lpos0; m; ++o) {
          const int i = __ffs(m) - 1;
          m &= m - 1;
          const int e = (lp0 + i) >> 4, r = (lp0 + i) & 15;
          const uint32_t id = fx.pg[e] * kPage + (uint32_t)r, row = fx.r0[e] + (uint32_t)r;
          if (staged) {
            sidx[o] = id;
            srow[o] = row;
          } else {
            oidx[o] = (int32_t)id;
            if (orow) orow[o] = row;
          }
        }
        if (staged) {
          __syncthreads();
          for (unsigned o = tid; o < n_out; o += kSpThreads) {
            oidx[o] = (int32_t)sidx[o];
            if (orow) orow[o] = srow[o];
          }
        }
      }
      if (cr == 0 && tid == 0) {
        a.count[set] = (int32_t)(gt_all + (unsigned)min(r_need, (unsigned long long)eq_all));
        if (a.done) a.done[set] = 0;   // the attention kernel's per-set completion counter
      }
      if (CS > 1) cluster_sync();   // peers are done reading this CTA's totals
    }
  }
  if (failed) {   // a wait gave up: give any copy still in flight time to land before exit
    const unsigned long long t0 = global_ns();
    while (global_ns() - t0 < kWaitNs / 4) {
    }
  }
  griddep_launch();
  cluster_sync();   // no CTA leaves while a peer may still access its shared memory
}

// ---------------------------------------------------------------------------
template <int G, int BITS>
static cudaError_t sp_prepare() {
  static std::atomic<int> attr_set[kMaxDevices];
  return once_per_device(attr_set, [] {
    cudaError_t e = cudaFuncSetAttribute(k_select_prune<G, BITS>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)kSpMaxSmem);
    if (e == cudaSuccess)
      e = cudaFuncSetAttribute(k_select_prune<G, BITS>,
                               cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
    return e;
  });
}

static cudaLaunchConfig_t sp_config(int units, int cs, size_t smem, cudaStream_t st,
                                    cudaLaunchAttribute* attr, bool pdl) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)units * (unsigned)cs);
  cfg.blockDim = dim3(kSpThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  int na = 0;
  attr[na].id = cudaLaunchAttributeClusterDimension;
  attr[na].val.clusterDim.x = (unsigned)cs;
  attr[na].val.clusterDim.y = 1;
  attr[na].val.clusterDim.z = 1;
  ++na;
  if (pdl) {
    attr[na].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[na].val.programmaticStreamSerializationAllowed = 1;
    ++na;
  }
  cfg.attrs = attr;
  cfg.numAttrs = na;
  return cfg;
}

// Clusters of `cs` CTAs with `smem` bytes each that fit the device at once
// (cached per device, cluster size and shared-memory size).
template <int G, int BITS>
static int sp_max_clusters(int cs, size_t smem) {
  struct Entry { int dev, cs; size_t smem; int n; };
  static Entry cache[64];
  static std::atomic<int> ncache{0};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 0;
  const int n = ncache.load(std::memory_order_acquire);
  for (int i = 0; i < n && i < 64; ++i)
    if (cache[i].dev == dev && cache[i].cs == cs && cache[i].smem == smem) return cache[i].n;
  cudaLaunchAttribute attr[2];
  cudaLaunchConfig_t cfg = sp_config(cs, cs, smem, nullptr, attr, false);
  int m = 0;
  if (cudaOccupancyMaxActiveClusters(&m, k_select_prune<G, BITS>, &cfg) != cudaSuccess) {
    (void)cudaGetLastError();
    m = 0;
  }
  const int slot = ncache.load(std::memory_order_acquire);
  if (slot < 64) {   // a racing thread at worst stores the same answer twice
    cache[slot] = Entry{dev, cs, smem, m};
    ncache.store(slot + 1, std::memory_order_release);
  }
  return m;
}

// Shared memory of a launch with ring depths s1, s2.
static size_t sp_smem_bytes(const SpShape& s, int kbits, int G, int max_pages, bool do_select,
                      bool do_prune) {
  const size_t stage2 = (size_t)kEstStageTok * (kHeadDim * kbits / 8 + 2 * kGroups * 2);
  size_t ra = 0, rb = 0;
  if (do_select)
    ra = (size_t)s.s1 * kMetaStagePages * kMetaRecBytes + (s.keys_in_smem ? (size_t)sp_pad(max_pages) * 4 + 4 : 0);
  if (do_prune) {
    rb = (size_t)s.s2 * stage2 > (size_t)kSpHistBytes ? (size_t)s.s2 * stage2 : (size_t)kSpHistBytes;
    if (s.logits_in_smem) rb += (size_t)sp_pad(s.share_cap * kPage) * G * sizeof(float);
  }
  return (kSpFixedBytes + (ra > rb ? ra : rb) + 127) / 128 * 128;
}

// Launch shape.  Each CTA's share of the candidate pages must fit
// kSpSharePages.  When the units, one cluster each, can all run at once
// with one CTA per SM, the cluster is the largest that allows that (an
// occupancy query decides: a cluster of 16 needs 16 free SMs of one GPC),
// and the rings take the whole shared memory (the bytes in flight per SM
// set the streaming rate).  Otherwise the cluster is the smallest allowed
// and the shared memory is sized for two CTAs per SM.
template <int G, int BITS>
static int sp_shape(int units, int max_pages, int sel_pages, bool do_select, bool do_prune,
                    int num_sms, SpShape* out) {
  int cs_min = 1;
  while (cs_min < kSpMaxCluster && (sel_pages + cs_min - 1) / cs_min > kSpSharePages) cs_min *= 2;
  if ((sel_pages + cs_min - 1) / cs_min > kSpSharePages) return -1;
  const size_t stage2 = (size_t)kEstStageTok * (kHeadDim * BITS / 8 + 2 * kGroups * 2);
  auto fill = [&](int cs, size_t budget, SpShape* s) {
    s->cs = cs;
    s->share_cap = (sel_pages + cs - 1) / cs;
    s->keys_in_smem = max_pages <= kSpKeysCap;
    s->logits_in_smem = (size_t)sp_pad(s->share_cap * kPage) * G * 4 <= (size_t)kSpLogitsSmem;
    const size_t keys = s->keys_in_smem ? (size_t)sp_pad(max_pages) * 4 + 4 : 0;
    const size_t logits = s->logits_in_smem ? (size_t)sp_pad(s->share_cap * kPage) * G * 4 : 0;
    const size_t room1 = budget > kSpFixedBytes + keys ? budget - kSpFixedBytes - keys : 0;
    const size_t room2 = budget > kSpFixedBytes + logits ? budget - kSpFixedBytes - logits : 0;
    s->s1 = (int)(room1 / ((size_t)kMetaStagePages * kMetaRecBytes));
    s->s2 = (int)(room2 / stage2);
    const int need2 = (s->share_cap + kEstStagePages - 1) / kEstStagePages;   // stages of a share
    s->s1 = s->s1 < 2 ? 2 : (s->s1 > kSpMaxStages ? kSpMaxStages : s->s1);
    s->s2 = s->s2 < 2 ? 2 : (s->s2 > kSpMaxStages ? kSpMaxStages : s->s2);
    if (s->s2 > need2 && need2 >= 2) s->s2 = need2;
    s->smem = sp_smem_bytes(*s, BITS, G, max_pages, do_select, do_prune);
  };
  SpShape s;
  const size_t big = 200 * 1024, two_per_sm = 110 * 1024;
  // two CTAs per SM when the registers allow it (more warps to hide latency)
  static int regs = 0;
  if (regs == 0) {
    cudaFuncAttributes fa;
    regs = cudaFuncGetAttributes(&fa, k_select_prune<G, BITS>) == cudaSuccess ? fa.numRegs : 255;
  }
  if (regs * kSpThreads * 2 <= 65536) {
    for (int cs = kSpMaxCluster; cs >= cs_min; cs /= 2) {
      if ((long long)units * cs > 2LL * num_sms) continue;
      fill(cs, two_per_sm, &s);
      if (s.smem > kSpMaxSmem) continue;
      if (sp_max_clusters<G, BITS>(cs, s.smem) >= units) {
        *out = s;
        return 0;
      }
    }
  }
  for (int cs = kSpMaxCluster; cs >= cs_min; cs /= 2) {
    if ((long long)units * cs > num_sms) continue;
    fill(cs, big, &s);
    if (s.smem > kSpMaxSmem) continue;
    if (sp_max_clusters<G, BITS>(cs, s.smem) >= units) {
      *out = s;
      return 0;
    }
  }
  fill(cs_min, two_per_sm, &s);
  if (s.smem > kSpMaxSmem) return -1;
  *out = s;
  return 0;
}

template <int G, int BITS>
static cudaError_t sp_launch_t(SpArgs a, int sel_pages, int num_sms, cudaStream_t st, bool pdl) {
  const cudaError_t prepared = sp_prepare<G, BITS>();
  if (prepared != cudaSuccess) return prepared;
  const int units = a.L.B * a.L.Hk;
  SpShape sh;
  if (sp_shape<G, BITS>(units, a.L.max_pages, sel_pages, a.meta != nullptr, a.codes != nullptr,
                        num_sms, &sh) != 0)
    return cudaErrorInvalidValue;
  a.s1 = sh.s1;
  a.s2 = sh.s2;
  a.share_cap = sh.share_cap;
  if (sh.keys_in_smem) a.gkeys = nullptr;
  if (sh.logits_in_smem) a.glogits = nullptr;
  cudaLaunchAttribute attr[2];
  cudaLaunchConfig_t cfg = sp_config(units, sh.cs, sh.smem, st, attr, pdl);
  return cudaLaunchKernelEx(&cfg, k_select_prune<G, BITS>, a);
}

cudaError_t launch_select_prune(const SpArgs& a, int sel_pages, int num_sms, cudaStream_t st,
                                bool pdl) {
  const int G = a.Hq / a.L.Hk;
  if (a.L.B * a.L.Hk == 0) return cudaSuccess;
  const bool two = a.L.kbits == 2;
#define TW_SP(GG)                                                                      \
  case GG:                                                                             \
    return two ? sp_launch_t<GG, 2>(a, sel_pages, num_sms, st, pdl)                    \
               : sp_launch_t<GG, 4>(a, sel_pages, num_sms, st, pdl);
  switch (G) {
    TW_SP(1) TW_SP(2) TW_SP(4) TW_SP(8)
  }
#undef TW_SP
  return cudaErrorInvalidValue;
}

// Largest candidate pages per unit the selection stages accept.
int select_prune_max_pages() { return kSpSharePages * kSpMaxCluster; }

// Self-test of the bounded wait: one thread waits on an mbarrier that nothing
// arrives on; the wait must give up after kWaitNs and set kDevErrWait in
// *status, and the kernel must then return normally.
__global__ void k_wait_selftest(int* status) {
  __shared__ uint64_t bar;
  mbar_init(&bar, 1);
  mbar_fence_init();
  if (mbar_wait(&bar, 0u, status)) atomicOr(status, 2);   // 2: the wait did not give up
}

cudaError_t launch_wait_selftest(int* status, cudaStream_t st) {
  k_wait_selftest<<<1, 1, 0, st>>>(status);
  return cudaGetLastError();
}

}  // namespace tw
