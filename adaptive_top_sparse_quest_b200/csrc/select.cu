// Quest pre-selection: page bound scores and top-K_p page selection.
//
// Twilight prunes on top of a base selector; with Quest the base selector ranks
// 16-token pages by an upper bound of q.k computed from the page's channel-wise
// key min / max and keeps the top pages ("Twilight: Adaptive Attention Sparsity
// with Hierarchical Top-p Pruning", atlas.scime.ai summary, "Surprising
// findings": Quest's per-page max-pooled layout is why Twilight's pruning is
// hierarchical).  Bound: score = sum_j max(q_j * min_j, q_j * max_j); under GQA
// the KV head's score is the sum of its query heads' scores.
//
// The score is a deterministic fp32 sum in one fixed order, so the selected
// page ids are an exact integer result: products of two fp16 values are exact
// in fp32; each lane of a half-warp sums its 8 channels left to right; the 16
// lane sums are combined by xor-butterfly 8, 4, 2, 1 (fp32 addition is
// commutative, so both partners of a butterfly hold the same value); heads are
// added in head order.
//
// k_page_scores is persistent: each CTA owns a contiguous block of
// (kv unit, 64-page chunk) items and loads item i+1's metadata while scoring
// item i (k_page_scores_paged does the same over the paged pool's record
// order, all KV heads of a page at once).  k_page_topk keeps each unit's K_p best pages by a most-significant-
// digit-first radix select on the ordered score keys (12 bits, then 9 at a
// time, starting below the bits all of the unit's keys share), then compacts
// them in page order with one block scan; in the fused decode step it also
// writes each kept page's first physical row.
#include "tw_common.cuh"
#include "tw_kernels.h"

namespace tw {

constexpr int kScorePagesPerHalfWarp = 4;
constexpr int kScoreThreads = 256;
constexpr int kScorePagesPerItem = (kScoreThreads / 16) * kScorePagesPerHalfWarp;   // 64

struct MetaLoad {
  uint4 mn[kScorePagesPerHalfWarp], mx[kScorePagesPerHalfWarp];
};

__device__ __forceinline__ void score_issue(const Layout& L, const __half* meta, int chunks,
                                            int it, int hw, int l16, MetaLoad& d) {
  const int u = it / chunks;
  const int b = u / L.Hk, hk = u % L.Hk;
  const int P = (L.len(b) + kPage - 1) / kPage;
  const int pg0 = (it % chunks) * kScorePagesPerItem + hw;
#pragma unroll
  for (int k = 0; k < kScorePagesPerHalfWarp; ++k) {
    const int pg = pg0 + k * (kScoreThreads / 16);
    d.mn[k] = make_uint4(0u, 0u, 0u, 0u);
    d.mx[k] = make_uint4(0u, 0u, 0u, 0u);
    if (pg < P) {
      const __half* m = meta + L.meta_index(b, hk, pg) * (2 * kHeadDim) + l16 * 8;
      d.mn[k] = ld_stream16(m);
      d.mx[k] = ld_stream16(m + kHeadDim);
    }
  }
}

__device__ __forceinline__ float h_lo_hi(uint32_t w, int hi) {
  return __half2float(__ushort_as_half((unsigned short)((w >> (16 * hi)) & 0xFFFFu)));
}

template <int G>
__global__ void __launch_bounds__(kScoreThreads)
k_page_scores(Layout L, const __half* __restrict__ q, int Hq, const __half* __restrict__ meta,
              float* __restrict__ scores) {
  const int chunks = (L.max_pages + kScorePagesPerItem - 1) / kScorePagesPerItem;
  const int items = L.B * L.Hk * chunks;
  const int per = (items + gridDim.x - 1) / gridDim.x;
  const int it0 = blockIdx.x * per, it1 = min(items, it0 + per);
  if (it0 >= it1) return;
  const int lane = threadIdx.x & 31, l16 = lane & 15;
  const unsigned hmask = 0xFFFFu << (lane & 16);
  const int hw = threadIdx.x >> 4;
  griddep_wait();
  MetaLoad A, B;
  score_issue(L, meta, chunks, it0, hw, l16, A);
  float qv[G][8];
  int qunit = -1;
  for (int it = it0; it < it1; ++it) {
    if (it + 1 < it1) score_issue(L, meta, chunks, it + 1, hw, l16, B);
    const int u = it / chunks;
    const int b = u / L.Hk, hk = u % L.Hk;
    if (u != qunit) {
#pragma unroll
      for (int g = 0; g < G; ++g) {
        const uint4 r = *reinterpret_cast<const uint4*>(
            q + ((int64_t)b * Hq + hk * G + g) * kHeadDim + l16 * 8);
        const uint32_t w[4] = {r.x, r.y, r.z, r.w};
#pragma unroll
        for (int j = 0; j < 8; ++j) qv[g][j] = h_lo_hi(w[j >> 1], j & 1);
      }
      qunit = u;
    }
    const int P = (L.len(b) + kPage - 1) / kPage;
    const int pg0 = (it % chunks) * kScorePagesPerItem + hw;
#pragma unroll
    for (int k = 0; k < kScorePagesPerHalfWarp; ++k) {
      const int pg = pg0 + k * (kScoreThreads / 16);
      if (pg >= P) continue;   // uniform across the half-warp
      const uint32_t wn[4] = {A.mn[k].x, A.mn[k].y, A.mn[k].z, A.mn[k].w};
      const uint32_t wx[4] = {A.mx[k].x, A.mx[k].y, A.mx[k].z, A.mx[k].w};
      float mnv[8], mxv[8];
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        mnv[j] = h_lo_hi(wn[j >> 1], j & 1);
        mxv[j] = h_lo_hi(wx[j >> 1], j & 1);
      }
      float total = 0.0f;
#pragma unroll
      for (int g = 0; g < G; ++g) {
        float s = fmaxf(__fmul_rn(qv[g][0], mnv[0]), __fmul_rn(qv[g][0], mxv[0]));
#pragma unroll
        for (int j = 1; j < 8; ++j)
          s = __fadd_rn(s, fmaxf(__fmul_rn(qv[g][j], mnv[j]), __fmul_rn(qv[g][j], mxv[j])));
#pragma unroll
        for (int o = 8; o > 0; o >>= 1) s = __fadd_rn(s, __shfl_xor_sync(hmask, s, o, 16));
        total = (g == 0) ? s : __fadd_rn(total, s);
      }
      if (l16 == 0) scores[(int64_t)u * L.max_pages + pg] = total;
    }
#pragma unroll
    for (int k = 0; k < kScorePagesPerHalfWarp; ++k) {
      A.mn[k] = B.mn[k];
      A.mx[k] = B.mx[k];
    }
  }
  griddep_launch();
}

// Paged layout: a pool page stores the metadata records of all KV heads side by
// side, so an item here is (sequence, ppi pages, a block of hb <= 64 KV heads)
// with ppi * hb <= 64 records, read as whole runs of hb * 512 B instead of one
// scattered 512 B record per page.  Record r of an item is page r / hb, head
// r % hb of the block; a thread's four records (r = half-warp + 16 k) are the
// same in every item, so their offsets are computed once.  The query rows vary
// by record and come through the read-only cache.
struct PagedGeo {
  int hb, ppi, nhb, chunks;
};

struct PagedItem {
  int b, pg0, hk0, P;
};

__device__ __forceinline__ PagedItem paged_item(const Layout& L, const PagedGeo& g, int it) {
  PagedItem x;
  x.b = it / (g.chunks * g.nhb);
  const int rest = it % (g.chunks * g.nhb);
  x.pg0 = (rest / g.nhb) * g.ppi;
  x.hk0 = (rest % g.nhb) * g.hb;
  x.P = (L.len(x.b) + kPage - 1) / kPage;
  return x;
}

// Pool pages of this thread's four records of an item (loads issued, not waited for).
__device__ __forceinline__ void paged_pt(const Layout& L, const PagedGeo& g, const PagedItem& x,
                                         const int (&rp)[4], int (&pt)[4]) {
#pragma unroll
  for (int k = 0; k < kScorePagesPerHalfWarp; ++k) {
    const int pg = x.pg0 + rp[k];
    pt[k] = (rp[k] < g.ppi && pg < x.P) ? L.page_table[(int64_t)x.b * L.max_pages + pg] : 0;
  }
}

__device__ __forceinline__ void score_issue_paged(const Layout& L, const __half* meta,
                                                  const PagedGeo& g, const PagedItem& x,
                                                  const int (&rp)[4], const int (&rh)[4],
                                                  const int (&pt)[4], int l16, MetaLoad& d) {
#pragma unroll
  for (int k = 0; k < kScorePagesPerHalfWarp; ++k) {
    d.mn[k] = make_uint4(0u, 0u, 0u, 0u);
    d.mx[k] = make_uint4(0u, 0u, 0u, 0u);
    const int pg = x.pg0 + rp[k], hk = x.hk0 + rh[k];
    if (rp[k] < g.ppi && hk < L.Hk && pg < x.P) {
      const int64_t rec = (int64_t)((unsigned)pt[k] < (unsigned)L.pool_pages ? pt[k] : 0) * L.Hk + hk;
      const __half* m = meta + rec * (2 * kHeadDim) + l16 * 8;
      d.mn[k] = ld_stream16(m);
      d.mx[k] = ld_stream16(m + kHeadDim);
    }
  }
}

template <int G>
__global__ void __launch_bounds__(kScoreThreads)
k_page_scores_paged(Layout L, const __half* __restrict__ q, int Hq,
                    const __half* __restrict__ meta, float* __restrict__ scores, PagedGeo g) {
  const int items = L.B * g.chunks * g.nhb;
  const int per = (items + gridDim.x - 1) / gridDim.x;
  const int it0 = blockIdx.x * per, it1 = min(items, it0 + per);
  if (it0 >= it1) return;
  const int lane = threadIdx.x & 31, l16 = lane & 15;
  const unsigned hmask = 0xFFFFu << (lane & 16);
  const int hw = threadIdx.x >> 4;
  int rp[kScorePagesPerHalfWarp], rh[kScorePagesPerHalfWarp];
#pragma unroll
  for (int k = 0; k < kScorePagesPerHalfWarp; ++k) {
    const int r = hw + 16 * k;
    rp[k] = r / g.hb;
    rh[k] = r % g.hb;
  }
  griddep_wait();
  // items it, it+1 and it+2 are in flight as (records in A), (page-table
  // entries in ptn, records issued into B this iteration), (entries loading)
  MetaLoad A, B;
  int pt0[4], ptn[4];
  PagedItem xa = paged_item(L, g, it0), xb = xa;
  paged_pt(L, g, xa, rp, pt0);
  score_issue_paged(L, meta, g, xa, rp, rh, pt0, l16, A);
  if (it0 + 1 < it1) {
    xb = paged_item(L, g, it0 + 1);
    paged_pt(L, g, xb, rp, ptn);
  }
  int bA = xa.b, pgA = xa.pg0, hkA = xa.hk0, PA = xa.P;
  for (int it = it0; it < it1; ++it) {
    if (it + 1 < it1) {
      score_issue_paged(L, meta, g, xb, rp, rh, ptn, l16, B);
      if (it + 2 < it1) {   // the entries are consumed one iteration later
        const PagedItem xc = paged_item(L, g, it + 2);
        paged_pt(L, g, xc, rp, ptn);
        xa = xb;
        xb = xc;
      } else {
        xa = xb;
      }
    }
#pragma unroll
    for (int k = 0; k < kScorePagesPerHalfWarp; ++k) {
      const int pg = pgA + rp[k], hk = hkA + rh[k];
      if (!(rp[k] < g.ppi && hk < L.Hk && pg < PA)) continue;   // uniform across the half-warp
      const uint32_t wn[4] = {A.mn[k].x, A.mn[k].y, A.mn[k].z, A.mn[k].w};
      const uint32_t wx[4] = {A.mx[k].x, A.mx[k].y, A.mx[k].z, A.mx[k].w};
      float mnv[8], mxv[8];
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        mnv[j] = h_lo_hi(wn[j >> 1], j & 1);
        mxv[j] = h_lo_hi(wx[j >> 1], j & 1);
      }
      float total = 0.0f;
#pragma unroll
      for (int gg = 0; gg < G; ++gg) {
        const uint4 r = __ldg(reinterpret_cast<const uint4*>(
            q + ((int64_t)bA * Hq + hk * G + gg) * kHeadDim + l16 * 8));
        const uint32_t wq[4] = {r.x, r.y, r.z, r.w};
        float qv[8];
#pragma unroll
        for (int j = 0; j < 8; ++j) qv[j] = h_lo_hi(wq[j >> 1], j & 1);
        float s = fmaxf(__fmul_rn(qv[0], mnv[0]), __fmul_rn(qv[0], mxv[0]));
#pragma unroll
        for (int j = 1; j < 8; ++j)
          s = __fadd_rn(s, fmaxf(__fmul_rn(qv[j], mnv[j]), __fmul_rn(qv[j], mxv[j])));
#pragma unroll
        for (int o = 8; o > 0; o >>= 1) s = __fadd_rn(s, __shfl_xor_sync(hmask, s, o, 16));
        total = (gg == 0) ? s : __fadd_rn(total, s);
      }
      if (l16 == 0) scores[((int64_t)bA * L.Hk + hk) * L.max_pages + pg] = total;
    }
#pragma unroll
    for (int k = 0; k < kScorePagesPerHalfWarp; ++k) {
      A.mn[k] = B.mn[k];
      A.mx[k] = B.mx[k];
    }
    bA = xa.b;
    pgA = xa.pg0;
    hkA = xa.hk0;
    PA = xa.P;
  }
  griddep_launch();
}

// ---------------------------------------------------------------------------
constexpr int kTopkThreads = 512;
constexpr int kTopkWarps = kTopkThreads / 32;
constexpr int kTopkMaxCached = 16;   // keys per thread kept in registers (up to 8192 pages)
constexpr int kTopkBins = 4096;  // first digit: 12 bits (8 per thread), then 9 (1 per thread)

// Inclusive scan over the block, in thread order, of a pair of counts; returns
// the exclusive prefix and writes the block totals.  Uses sh[0..kTopkWarps].
__device__ __forceinline__ int2 block_excl_scan2(int2 v, int2* sh, int2* total) {
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
  if (lane == 31) sh[warp] = incl;
  __syncthreads();
  if (warp == 0) {
    const int2 x = lane < kTopkWarps ? sh[lane] : make_int2(0, 0);
    int2 xi = x;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int tx = __shfl_up_sync(0xffffffffu, xi.x, o);
      const int ty = __shfl_up_sync(0xffffffffu, xi.y, o);
      if (lane >= o) {
        xi.x += tx;
        xi.y += ty;
      }
    }
    if (lane < kTopkWarps) sh[lane] = make_int2(xi.x - x.x, xi.y - x.y);
    if (lane == 31) sh[kTopkWarps] = xi;
  }
  __syncthreads();
  const int2 r = make_int2(sh[warp].x + incl.x - v.x, sh[warp].y + incl.y - v.y);
  *total = sh[kTopkWarps];
  return r;
}

// One block per (b, kv head): the K_p largest page scores, ties to the lower
// page index, written in ascending page order (and, when row0 is given, each
// kept page's first physical row).  Thread t owns the E consecutive pages
// [t E, t E + E); the first EC keys stay in registers (EC is chosen from the
// cache's page count, so the unrolled loops are as long as the work), later
// ones are re-read from the score buffer.
template <int EC>
__global__ void __launch_bounds__(kTopkThreads, 2)
k_page_topk(Layout L, const float* __restrict__ scores, int budget_pages,
            int32_t* __restrict__ cand, int cand_stride, int32_t* __restrict__ ncand,
            uint32_t* __restrict__ row0) {
  __shared__ __align__(16) int hist[kTopkBins];
  __shared__ int wsuf[kTopkWarps];
  __shared__ uint32_t wmin[kTopkWarps], wmax[kTopkWarps];
  __shared__ int2 sh_scan[kTopkWarps + 1];
  __shared__ int sh_d, sh_above;
  const int u = blockIdx.x;
  const int b = u / L.Hk, hk = u % L.Hk;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  reinterpret_cast<int4*>(hist)[2 * tid] = make_int4(0, 0, 0, 0);
  reinterpret_cast<int4*>(hist)[2 * tid + 1] = make_int4(0, 0, 0, 0);
  griddep_wait();
  const int P = (L.len(b) + kPage - 1) / kPage;
  const int Kp = min(budget_pages, P);
  int32_t* out = cand + (int64_t)u * cand_stride;
  uint32_t* orow = row0 ? row0 + (int64_t)u * L.max_pages : nullptr;
  auto emit = [&](int pos, int pg) {
    out[pos] = pg;
    if (orow) orow[pos] = (uint32_t)L.page_row(b, hk, pg);
  };
  if (Kp >= P) {
    for (int i = tid; i < P; i += kTopkThreads) emit(i, i);
    if (tid == 0) ncand[u] = P;
    griddep_launch();
    return;
  }
  const float* sc = scores + (int64_t)u * L.max_pages;
  const int E = (P + kTopkThreads - 1) / kTopkThreads;
  const int i0 = tid * E;
  uint32_t key[EC];
  int ptc[EC];   // page-table entries of the cached pages (paged layout, row0 wanted)
  const bool want_pt = orow && L.page_table;
#pragma unroll
  for (int k = 0; k < EC; ++k) {
    const bool in = k < E && i0 + k < P;
    key[k] = in ? f_key(sc[i0 + k]) : 0u;
    ptc[k] = (want_pt && in) ? L.page_table[(int64_t)b * L.max_pages + i0 + k] : 0;
  }
  // f(k, key, pt) over this thread's valid pages i0 + k in order: the cached
  // keys with static register indices, then any further ones from memory
  auto for_keys = [&](auto&& f) {
#pragma unroll
    for (int k = 0; k < EC; ++k)
      if (k < E && i0 + k < P) f(k, key[k], ptc[k]);
    for (int k = EC; k < E; ++k)
      if (i0 + k < P) f(k, f_key(sc[i0 + k]), 0);
  };
  // the keys of one unit's pages share their top bits (scores of similar
  // magnitude), so the digits start below the common prefix of the block's
  // smallest and largest key: 12 bits, then 9 at a time
  uint32_t kmin = 0xFFFFFFFFu, kmax = 0u;
  for_keys([&](int, uint32_t kk, int) {
    kmin = min(kmin, kk);
    kmax = max(kmax, kk);
  });
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    kmin = min(kmin, __shfl_xor_sync(0xffffffffu, kmin, o));
    kmax = max(kmax, __shfl_xor_sync(0xffffffffu, kmax, o));
  }
  if (lane == 0) {
    wmin[warp] = kmin;
    wmax[warp] = kmax;
  }
  __syncthreads();
#pragma unroll
  for (int w = 0; w < kTopkWarps; ++w) {
    kmin = min(kmin, wmin[w]);
    kmax = max(kmax, wmax[w]);
  }
  int nb = 32 - __clz((int)(kmin ^ kmax));   // low bits still to resolve (0: all keys equal)
  uint32_t pmask = nb >= 32 ? 0u : ~((1u << nb) - 1u);
  uint32_t prefix = kmin & pmask;
  int need = Kp;   // keys matching `prefix` that still belong to the top K_p
  for (int round = 0; nb > 0; ++round) {
    const int width = min(round == 0 ? 12 : 9, nb);
    const int shift = nb - width;
    const uint32_t dm = (1u << width) - 1u;
    nb = shift;
    for_keys([&](int, uint32_t kk, int) {
      if ((kk & pmask) == prefix) atomicAdd(&hist[(kk >> shift) & dm], 1);
    });
    __syncthreads();
    // this thread's digits: 8 tid .. 8 tid + 7 in the first round, tid after
    int sl[8];
    if (round == 0) {
      const int4 a4 = reinterpret_cast<const int4*>(hist)[2 * tid];
      const int4 b4 = reinterpret_cast<const int4*>(hist)[2 * tid + 1];
      sl[7] = b4.w;
      sl[6] = b4.z + sl[7];
      sl[5] = b4.y + sl[6];
      sl[4] = b4.x + sl[5];
      sl[3] = a4.w + sl[4];
      sl[2] = a4.z + sl[3];
      sl[1] = a4.y + sl[2];
      sl[0] = a4.x + sl[1];
    } else {
      sl[0] = hist[tid];
#pragma unroll
      for (int k = 1; k < 8; ++k) sl[k] = 0;
    }
    int incl = sl[0];
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int t = __shfl_down_sync(0xffffffffu, incl, o);
      if (lane + o < 32) incl += t;
    }
    if (lane == 0) wsuf[warp] = incl;
    __syncthreads();
    int after = incl - sl[0];
#pragma unroll
    for (int w = 0; w < kTopkWarps; ++w)
      if (w > warp) after += wsuf[w];
    // the digit d of the K_p-th largest key: suffix(d) >= need > suffix(d + 1)
    const int bpt = round == 0 ? 8 : 1;
#pragma unroll
    for (int k = 0; k < 8; ++k) {
      if (k < bpt) {
        const int here = sl[k] + after;
        const int next = (k + 1 < bpt ? sl[k + 1] : 0) + after;
        if (here >= need && next < need) {
          sh_d = bpt * tid + k;
          sh_above = next;
        }
      }
    }
    if (round == 0) {
      reinterpret_cast<int4*>(hist)[2 * tid] = make_int4(0, 0, 0, 0);
      reinterpret_cast<int4*>(hist)[2 * tid + 1] = make_int4(0, 0, 0, 0);
    } else {
      hist[tid] = 0;
    }
    __syncthreads();
    need -= sh_above;
    prefix |= (uint32_t)sh_d << shift;
    pmask |= dm << shift;
  }
  // keep every key above prefix and the `need` lowest-index pages equal to it
  int n_gt = 0, n_eq = 0;
  for_keys([&](int, uint32_t kk, int) {
    n_gt += kk > prefix ? 1 : 0;
    n_eq += kk == prefix ? 1 : 0;
  });
  int2 tot;
  const int2 ex = block_excl_scan2(make_int2(n_gt, n_eq), sh_scan, &tot);
  int take = ex.y < need ? min(n_eq, need - ex.y) : 0;
  int pos = ex.x + min(need, ex.y);
  for_keys([&](int k, uint32_t kk, int p) {
    bool sel = kk > prefix;
    if (!sel && kk == prefix && take > 0) {
      sel = true;
      --take;
    }
    if (sel) {
      const int pg = i0 + k;
      out[pos] = pg;
      if (orow) {
        int64_t r;
        if (want_pt && k < EC)
          r = ((int64_t)((unsigned)p < (unsigned)L.pool_pages ? p : 0) * L.Hk + hk) * kPage;
        else
          r = L.page_row(b, hk, pg);
        orow[pos] = (uint32_t)r;
      }
      ++pos;
    }
  });
  if (tid == 0) ncand[u] = tot.x + min(need, tot.y);
  griddep_launch();
}

template <int G>
static int score_grid(int num_sms) {
  static int per_sm = 0;
  if (per_sm == 0) {
    int n = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, k_page_scores<G>, kScoreThreads, 0) !=
            cudaSuccess || n < 1)
      n = 1;
    per_sm = n;
  }
  return num_sms * per_sm;
}

template <int G>
static int score_grid_paged(int num_sms) {
  static int per_sm = 0;
  if (per_sm == 0) {
    int n = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, k_page_scores_paged<G>, kScoreThreads,
                                                      0) != cudaSuccess || n < 1)
      n = 1;
    per_sm = n;
  }
  return num_sms * per_sm;
}

cudaError_t launch_page_scores(const Layout& L, const __half* q, int Hq, const __half* meta,
                               float* scores, cudaStream_t st, int num_sms, bool pdl) {
  const int G = Hq / L.Hk;
  if (L.page_table) {
    PagedGeo g;
    g.hb = L.Hk < kScorePagesPerItem ? L.Hk : kScorePagesPerItem;
    g.ppi = kScorePagesPerItem / g.hb;
    g.nhb = (L.Hk + g.hb - 1) / g.hb;
    g.chunks = (L.max_pages + g.ppi - 1) / g.ppi;
    const long long items64 = (long long)L.B * g.chunks * g.nhb;
    if (items64 > 0x7FFFFFFF) return cudaErrorInvalidValue;
    const int items = (int)items64;
    switch (G) {
#define TW_SCP(GG)                                                                          \
  case GG: {                                                                                \
    const int grid = items < score_grid_paged<GG>(num_sms) ? items : score_grid_paged<GG>(num_sms); \
    return launch_k(k_page_scores_paged<GG>, dim3(grid), dim3(kScoreThreads), 0, st, pdl, L, q, \
                    Hq, meta, scores, g);                                                   \
  }
      TW_SCP(1) TW_SCP(2) TW_SCP(4) TW_SCP(8)
#undef TW_SCP
    }
    return cudaErrorInvalidValue;
  }
  const int items = L.B * L.Hk * ((L.max_pages + kScorePagesPerItem - 1) / kScorePagesPerItem);
  switch (G) {
#define TW_SC(GG)                                                                           \
  case GG: {                                                                                \
    const int grid = items < score_grid<GG>(num_sms) ? items : score_grid<GG>(num_sms);    \
    return launch_k(k_page_scores<GG>, dim3(grid), dim3(kScoreThreads), 0, st, pdl, L, q,   \
                    Hq, meta, scores);                                                      \
  }
    TW_SC(1) TW_SC(2) TW_SC(4) TW_SC(8)
#undef TW_SC
  }
  return cudaErrorInvalidValue;
}

cudaError_t launch_page_topk(const Layout& L, const float* scores, int budget_pages,
                             int32_t* cand, int cand_stride, int32_t* ncand, uint32_t* row0,
                             cudaStream_t st, bool pdl) {
  const int e = (L.max_pages + kTopkThreads - 1) / kTopkThreads;
#define TW_TK(EE)                                                                             \
  if (e <= EE || EE == kTopkMaxCached)                                                        \
    return launch_k(k_page_topk<EE>, dim3(L.B * L.Hk), dim3(kTopkThreads), 0, st, pdl, L,     \
                    scores, budget_pages, cand, cand_stride, ncand, row0);
  TW_TK(1) TW_TK(2) TW_TK(4) TW_TK(8) TW_TK(16)
#undef TW_TK
  return cudaErrorInvalidValue;
}

}  // namespace tw
