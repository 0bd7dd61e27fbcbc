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
#include "tw_common.cuh"
#include "tw_kernels.h"

namespace tw {

constexpr int kScorePagesPerHalfWarp = 4;
constexpr int kScoreThreads = 256;
constexpr int kScorePagesPerBlock = (kScoreThreads / 16) * kScorePagesPerHalfWarp;

template <int G>
__global__ void __launch_bounds__(kScoreThreads)
k_page_scores(Layout L, const __half* __restrict__ q, int Hq, const __half* __restrict__ meta,
              float* __restrict__ scores) {
  const int u = blockIdx.y;  // (b, kv head)
  const int b = u / L.Hk, hk = u % L.Hk;
  const int P = (L.len(b) + kPage - 1) / kPage;
  const int pg0 = blockIdx.x * kScorePagesPerBlock;
  if (pg0 >= P) return;
  const int lane = threadIdx.x & 31;
  const int l16 = lane & 15;
  const unsigned hmask = 0xFFFFu << (lane & 16);
  const int hw = threadIdx.x >> 4;

  float qv[G][8];
#pragma unroll
  for (int g = 0; g < G; ++g) {
    const uint4 r = *reinterpret_cast<const uint4*>(q + ((int64_t)b * Hq + hk * G + g) * kHeadDim +
                                                    l16 * 8);
    const uint32_t w[4] = {r.x, r.y, r.z, r.w};
#pragma unroll
    for (int j = 0; j < 8; ++j)
      qv[g][j] = __half2float(__ushort_as_half((unsigned short)((w[j >> 1] >> (16 * (j & 1))) & 0xFFFF)));
  }

  int pgs[kScorePagesPerHalfWarp];
  uint4 mnr[kScorePagesPerHalfWarp], mxr[kScorePagesPerHalfWarp];
#pragma unroll
  for (int k = 0; k < kScorePagesPerHalfWarp; ++k) {
    pgs[k] = pg0 + hw + k * (kScoreThreads / 16);
    if (pgs[k] < P) {
      const __half* m = meta + L.meta_index(b, hk, pgs[k]) * (2 * kHeadDim) + l16 * 8;
      mnr[k] = ld_stream16(m);
      mxr[k] = ld_stream16(m + kHeadDim);
    }
  }
#pragma unroll
  for (int k = 0; k < kScorePagesPerHalfWarp; ++k) {
    if (pgs[k] >= P) continue;  // uniform across the half-warp
    const uint32_t wn[4] = {mnr[k].x, mnr[k].y, mnr[k].z, mnr[k].w};
    const uint32_t wx[4] = {mxr[k].x, mxr[k].y, mxr[k].z, mxr[k].w};
    float mnv[8], mxv[8];
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      mnv[j] = __half2float(__ushort_as_half((unsigned short)((wn[j >> 1] >> (16 * (j & 1))) & 0xFFFF)));
      mxv[j] = __half2float(__ushort_as_half((unsigned short)((wx[j >> 1] >> (16 * (j & 1))) & 0xFFFF)));
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
    if (l16 == 0) scores[(int64_t)u * L.max_pages + pgs[k]] = total;
  }
}

// ---------------------------------------------------------------------------
// Block-wide helpers for the 1024-thread selection kernels.

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

constexpr int kTopkThreads = 1024;

// One block per (b, kv head): the K_p largest page scores (ties to the lower
// page index) by a most-significant-digit-first radix select on the ordered
// score keys, then a stable compaction in page order.
__global__ void __launch_bounds__(kTopkThreads)
k_page_topk(Layout L, const float* __restrict__ scores, int budget_pages,
            int32_t* __restrict__ cand, int cand_stride, int32_t* __restrict__ ncand) {
  __shared__ int hist[256];
  __shared__ int wsum[33];
  __shared__ int sh_scan[33];
  __shared__ int sh_d, sh_above;
  const int u = blockIdx.x;
  const int b = u / L.Hk;
  const int P = (L.len(b) + kPage - 1) / kPage;
  const int Kp = min(budget_pages, P);
  int32_t* out = cand + (int64_t)u * cand_stride;
  const float* sc = scores + (int64_t)u * L.max_pages;
  const int tid = threadIdx.x;
  if (Kp >= P) {
    for (int i = tid; i < P; i += blockDim.x) out[i] = i;
    if (tid == 0) ncand[u] = P;
    return;
  }
  uint32_t prefix = 0, pmask = 0;
  int need = Kp;  // how many of the elements matching `prefix` still belong to the top K_p
  for (int round = 0; round < 4; ++round) {
    const int shift = 24 - 8 * round;
    for (int i = tid; i < 256; i += blockDim.x) hist[i] = 0;
    __syncthreads();
    for (int i = tid; i < P; i += blockDim.x) {
      const uint32_t key = f_key(sc[i]);
      if ((key & pmask) == prefix) atomicAdd(&hist[(key >> shift) & 255], 1);
    }
    __syncthreads();
    // suffix sums over the 256 digits: suf[j] = sum_{d >= j} hist[d]
    int suf = 0;
    const int lane = tid & 31, warp = tid >> 5;
    if (tid < 256) {
      suf = hist[tid];
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int t = __shfl_down_sync(0xffffffffu, suf, o);
        if (lane + o < 32) suf += t;
      }
      if (lane == 0) wsum[warp] = suf;
    }
    __syncthreads();
    if (tid < 256) {
      for (int w = warp + 1; w < 8; ++w) suf += wsum[w];
    }
    // the digit of the K_p-th largest key is the largest j with suf[j] >= need
    const int cnt = __syncthreads_count(tid < 256 && suf >= need);
    const int d = cnt - 1;
    if (tid == d + 1) sh_above = suf;   // elements strictly above digit d
    if (tid == 0) sh_d = d;
    __syncthreads();
    need -= sh_above;
    prefix |= (uint32_t)sh_d << shift;
    pmask |= 255u << shift;
    __syncthreads();
  }
  // prefix is the K_p-th largest key; keep every key above it and the `need`
  // lowest-index pages equal to it, in ascending page order.
  int ties_before = 0, written = 0;
  for (int base = 0; base < P; base += blockDim.x) {
    const int i = base + tid;
    uint32_t key = 0;
    if (i < P) key = f_key(sc[i]);
    const bool gt = i < P && key > prefix;
    const bool eq = i < P && key == prefix;
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
}

void launch_page_scores(const Layout& L, const __half* q, int Hq, const __half* meta,
                        float* scores, cudaStream_t st) {
  const int G = Hq / L.Hk;
  dim3 grid((L.max_pages + kScorePagesPerBlock - 1) / kScorePagesPerBlock, L.B * L.Hk);
  switch (G) {
    case 1: k_page_scores<1><<<grid, kScoreThreads, 0, st>>>(L, q, Hq, meta, scores); break;
    case 2: k_page_scores<2><<<grid, kScoreThreads, 0, st>>>(L, q, Hq, meta, scores); break;
    case 4: k_page_scores<4><<<grid, kScoreThreads, 0, st>>>(L, q, Hq, meta, scores); break;
    case 8: k_page_scores<8><<<grid, kScoreThreads, 0, st>>>(L, q, Hq, meta, scores); break;
  }
}

void launch_page_topk(const Layout& L, const float* scores, int budget_pages, int32_t* cand,
                      int cand_stride, int32_t* ncand, cudaStream_t st) {
  k_page_topk<<<L.B * L.Hk, kTopkThreads, 0, st>>>(L, scores, budget_pages, cand, cand_stride,
                                                  ncand);
}

}  // namespace tw
