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
// item i.  k_page_topk keeps each unit's K_p best pages by a most-significant-
// digit-first radix select on the ordered score keys (histograms replicated 8
// ways against same-address contention), then compacts them in page order.
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

// ---------------------------------------------------------------------------
constexpr int kTopkThreads = 1024;
constexpr int kTopkCached = 8;   // keys per thread kept in registers (8192 pages)
constexpr int kTopkReps = 8;

// Exclusive prefix count of a 0/1 flag over the block in thread order; returns
// the flag's rank and writes the block total to *total.  Uses sh[0..32].
__device__ __forceinline__ int block_rank(bool flag, int* sh, int* total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = blockDim.x >> 5;
  const unsigned bal = __ballot_sync(0xffffffffu, flag);
  const int in_warp = __popc(bal & ((1u << lane) - 1u));
  if (lane == 0) sh[warp] = __popc(bal);
  __syncthreads();
  if (warp == 0) {
    const int v = lane < nw ? sh[lane] : 0;
    int incl = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int t = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += t;
    }
    if (lane < nw) sh[lane] = incl - v;
    if (lane == 31) sh[32] = incl;
  }
  __syncthreads();
  const int r = sh[warp] + in_warp;
  *total = sh[32];
  __syncthreads();
  return r;
}

// One block per (b, kv head): the K_p largest page scores, ties to the lower
// page index, written in ascending page order.
__global__ void __launch_bounds__(kTopkThreads)
k_page_topk(Layout L, const float* __restrict__ scores, int budget_pages,
            int32_t* __restrict__ cand, int cand_stride, int32_t* __restrict__ ncand) {
  __shared__ int hrep[kTopkReps][256];
  __shared__ int wsum[8];
  __shared__ int sh_scan[33];
  __shared__ int sh_d, sh_above;
  const int u = blockIdx.x;
  const int b = u / L.Hk;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  griddep_wait();
  const int P = (L.len(b) + kPage - 1) / kPage;
  const int Kp = min(budget_pages, P);
  int32_t* out = cand + (int64_t)u * cand_stride;
  const float* sc = scores + (int64_t)u * L.max_pages;
  if (Kp >= P) {
    for (int i = tid; i < P; i += kTopkThreads) out[i] = i;
    if (tid == 0) ncand[u] = P;
    griddep_launch();
    return;
  }
  uint32_t key[kTopkCached];
#pragma unroll
  for (int j = 0; j < kTopkCached; ++j) {
    const int i = j * kTopkThreads + tid;
    key[j] = i < P ? f_key(sc[i]) : 0u;
  }
  const int chunks = (P + kTopkThreads - 1) / kTopkThreads;
  auto key_at = [&](int j) -> uint32_t {   // key of page j * kTopkThreads + tid
    if (j < kTopkCached) {
      uint32_t r = 0u;
#pragma unroll
      for (int t = 0; t < kTopkCached; ++t)
        if (t == j) r = key[t];
      return r;
    }
    const int i = j * kTopkThreads + tid;
    return i < P ? f_key(sc[i]) : 0u;
  };
  uint32_t prefix = 0, pmask = 0;
  int need = Kp;   // elements matching `prefix` that still belong to the top K_p
  int* hflat = &hrep[0][0];
  const int rep = lane & (kTopkReps - 1);
  for (int round = 0; round < 4; ++round) {
    const int shift = 24 - 8 * round;
    for (int i = tid; i < kTopkReps * 256; i += kTopkThreads) hflat[i] = 0;
    __syncthreads();
    for (int j = 0; j < chunks; ++j) {
      const int i = j * kTopkThreads + tid;
      const uint32_t k = key_at(j);
      if (i < P && (k & pmask) == prefix) atomicAdd(&hrep[rep][(k >> shift) & 255], 1);
    }
    __syncthreads();
    // suffix sums over the 256 digits: suf[j] = sum_{d >= j} hist[d]
    int suf = 0;
    if (tid < 256) {
#pragma unroll
      for (int r = 0; r < kTopkReps; ++r) suf += hrep[r][tid];
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int t = __shfl_down_sync(0xffffffffu, suf, o);
        if (lane + o < 32) suf += t;
      }
      if (lane == 0) wsum[warp] = suf;
    }
    __syncthreads();
    if (tid < 256)
      for (int w = warp + 1; w < 8; ++w) suf += wsum[w];
    // the digit of the K_p-th largest key is the largest j with suf[j] >= need
    const int cnt = __syncthreads_count(tid < 256 && suf >= need);
    const int d = cnt - 1;
    if (tid == d + 1) sh_above = suf;   // elements strictly above digit d (0 when d = 255)
    if (tid == 0) sh_d = d;
    __syncthreads();
    need -= sh_above;
    prefix |= (uint32_t)sh_d << shift;
    pmask |= 255u << shift;
    __syncthreads();
  }
  // keep every key above prefix and the `need` lowest-index pages equal to it
  int ties_before = 0, written = 0;
  for (int j = 0; j < chunks; ++j) {
    const int i = j * kTopkThreads + tid;
    const uint32_t k = key_at(j);
    const bool gt = i < P && k > prefix;
    const bool eq = i < P && k == prefix;
    int eq_total;
    const int eq_rank = ties_before + block_rank(eq, sh_scan, &eq_total);
    const bool sel = gt || (eq && eq_rank < need);
    int sel_total;
    const int pos = written + block_rank(sel, sh_scan, &sel_total);
    if (sel) out[pos] = i;
    ties_before += eq_total;
    written += sel_total;
  }
  if (tid == 0) ncand[u] = written;
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

cudaError_t launch_page_scores(const Layout& L, const __half* q, int Hq, const __half* meta,
                               float* scores, cudaStream_t st, int num_sms, bool pdl) {
  const int G = Hq / L.Hk;
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
                             int32_t* cand, int cand_stride, int32_t* ncand, cudaStream_t st,
                             bool pdl) {
  return launch_k(k_page_topk, dim3(L.B * L.Hk), dim3(kTopkThreads), 0, st, pdl, L, scores,
                  budget_pages, cand, cand_stride, ncand);
}

}  // namespace tw
