// Twilight weight estimation from the 4-bit key cache, with fused softmax
// statistics ("Twilight: Adaptive Attention Sparsity with Hierarchical Top-p
// Pruning", atlas.scime.ai summary, "Approach": the candidates' attention
// weights are estimated from INT4 keys before top-p pruning).
//
// For candidate i, query head h and 32-channel group g with scale s, zero z:
//   k_hat = z + s * c = (z + 8 s) + s * (c - 8),  c in 0..15
//   l[i,h] = sum_g ( s_ig * D[h,g,i] + (z_ig + 8 s_ig) * Q[h,g] ) / sqrt(128)
//   D[h,g,i] = sum_{j in g} q_hj * (c_ij - 8),   Q[h,g] = sum_{j in g} q_hj
// The D terms are a small dense contraction, run on the tensor cores with
// mma.sync m16n8k16 (fp16 operands, fp32 accumulation): (c - 8) and the fp16
// queries are exact in fp16 and their products exact in fp32.  The MMA's M
// rows are (head, group) pairs (row 4h + g), N is 8 candidates, K is 16
// channels per step; each row keeps only its own group's channels, so after 8
// K-steps every row holds one D[h,g,*] and the per-group scales are applied in
// the fp32 epilogue.  The K order is permuted so that lane (gid, t) feeds
// exactly the codes of candidate gid, group t it loaded: 16 B of codes become
// 8 half2 B-fragments with one shift, one LOP3 (nibbles -> 0x6400|c, i.e.
// 1024 + c) and one half2 subtract of 1032 each.  M = 16 rows cover 4 heads
// (GQA 4:1); 8 heads take two row blocks.
//
// Persistent kernel: each CTA owns a contiguous block of (kv unit,
// 256-candidate) items, 32 candidates per warp (4 MMA tiles of 8), and loads
// item i+1's codes and item i+2's candidate page ids while computing item i.
// Each warp writes the per-head max and sum exp(l - max) of its 32 logits so
// the top-p kernel starts from softmax statistics without another pass.
#include "tw_common.cuh"
#include "tw_kernels.h"

namespace tw {

constexpr int kEstThreads = 256;
constexpr int kEstTiles = 4;                  // 4 MMA tiles x 8 candidates = 32 per warp
constexpr float kInvSqrtD = 0.08838834764831845f;

struct EstLoad {
  uint4 cw[kEstTiles];       // 16 B of codes: candidate gid of tile k, group t
  uint32_t sz[kEstTiles];    // fp16 scale (low half) and zero (high half) of that group
};

struct EstIds {
  int len, C;
  int pg[kEstTiles];
};

__device__ __forceinline__ void est_issue_ids(const Layout& L, const int32_t* cand,
                                              int cand_stride, const int32_t* ncand, int cmax,
                                              int tiles, int it, int warp, int gid, EstIds& r) {
  const int u = it / tiles;
  const int b = u / L.Hk;
  r.len = L.len(b);
  r.C = cand ? ncand[u] * kPage : r.len;
#pragma unroll
  for (int k = 0; k < kEstTiles; ++k) {
    const int c = (it % tiles) * kEstTile + warp * 32 + k * 8 + gid;
    r.pg[k] = 0;
    if (cand && (c >> 4) < cand_stride && c < cmax) r.pg[k] = cand[(int64_t)u * cand_stride + (c >> 4)];
  }
}

__device__ __forceinline__ void est_tokens(const EstIds& r, bool has_cand, int cmax, int tiles,
                                           int it, int warp, int gid, int tok[kEstTiles]) {
  const int C = min(r.C, cmax);
#pragma unroll
  for (int k = 0; k < kEstTiles; ++k) {
    const int c = (it % tiles) * kEstTile + warp * 32 + k * 8 + gid;
    int t = -1;
    if (c < C) {
      t = has_cand ? r.pg[k] * kPage + (c & 15) : c;
      if (t < 0 || t >= r.len) t = -1;
    }
    tok[k] = t;
  }
}

__device__ __forceinline__ void est_issue_codes(const Layout& L, const uint8_t* codes,
                                                const __half* scales, const __half* zeros,
                                                int tiles, int it, int t,
                                                const int tok[kEstTiles], EstLoad& d) {
  const int u = it / tiles;
  const int b = u / L.Hk, hk = u % L.Hk;
#pragma unroll
  for (int k = 0; k < kEstTiles; ++k) {
    d.cw[k] = make_uint4(0x88888888u, 0x88888888u, 0x88888888u, 0x88888888u);
    d.sz[k] = 0u;
    if (tok[k] >= 0) {
      const int64_t row = L.row(b, hk, tok[k]);
      d.cw[k] = ld_stream16(codes + row * (kHeadDim / 2) + t * 16);
      d.sz[k] = (uint32_t)__half_as_ushort(scales[row * kGroups + t]) |
                ((uint32_t)__half_as_ushort(zeros[row * kGroups + t]) << 16);
    }
  }
}

__device__ __forceinline__ void mma16816(float (&d)[4], const uint32_t (&a)[4], uint32_t b0,
                                         uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
      "{%8,%9}, {%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// Nibbles e and e+4 of W as the half2 (c_e - 8, c_{e+4} - 8), exact.
__device__ __forceinline__ uint32_t nib_pair(uint32_t W, int e) {
  uint32_t x = ((W >> (4 * e)) & 0x000F000Fu) | 0x64006400u;   // (1024 + c) as fp16
  uint32_t r;
  asm("sub.rn.f16x2 %0, %1, %2;" : "=r"(r) : "r"(x), "r"(0x64086408u));   // minus 1032
  return r;
}

__device__ __forceinline__ uint32_t pack_h2(__half lo, __half hi) {
  return (uint32_t)__half_as_ushort(lo) | ((uint32_t)__half_as_ushort(hi) << 16);
}

// RB: 16-row blocks of (head, group) pairs, ceil(G / 4).
template <int G>
__global__ void __launch_bounds__(kEstThreads)
k_estimate(Layout L, const __half* __restrict__ q, int Hq, const uint8_t* __restrict__ codes,
           const __half* __restrict__ scales, const __half* __restrict__ zeros,
           const int32_t* __restrict__ cand, int cand_stride, const int32_t* __restrict__ ncand,
           int lcap, int cmax, float* __restrict__ logits, float2* __restrict__ stats) {
  constexpr int RB = (G + 3) / 4;
  const int tiles = lcap / kEstTile;
  const int items = L.B * L.Hk * tiles;
  const int per = (items + gridDim.x - 1) / gridDim.x;
  const int it0 = blockIdx.x * per;
  const int it1 = min(items, it0 + per);
  if (it0 >= it1) return;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int gid = lane >> 2, t = lane & 3;
  const int g = gid & 3;                 // group of the MMA rows this lane holds
  const int nspan = lcap / kStatSpan;
  const bool has_cand = cand != nullptr;

  int tokA[kEstTiles], tokB[kEstTiles];
  EstIds ids;
  EstLoad A, B;
  griddep_wait();
  est_issue_ids(L, cand, cand_stride, ncand, cmax, tiles, it0, warp, gid, ids);
  est_tokens(ids, has_cand, cmax, tiles, it0, warp, gid, tokA);
  est_issue_codes(L, codes, scales, zeros, tiles, it0, t, tokA, A);
  if (it0 + 1 < it1) {
    est_issue_ids(L, cand, cand_stride, ncand, cmax, tiles, it0 + 1, warp, gid, ids);
    est_tokens(ids, has_cand, cmax, tiles, it0 + 1, warp, gid, tokB);
  }
  uint32_t afr[RB][8][4];
  float qsum[RB][2];
  int staged = -1;
  for (int it = it0; it < it1; ++it) {
    if (it + 1 < it1) est_issue_codes(L, codes, scales, zeros, tiles, it + 1, t, tokB, B);
    if (it + 2 < it1) est_issue_ids(L, cand, cand_stride, ncand, cmax, tiles, it + 2, warp, gid, ids);
    const int u = it / tiles;
    const int b = u / L.Hk, hk = u % L.Hk;
    if (u != staged) {
      // A fragments: row gid = (head rb*4 + gid/4, group g), row gid+8 = head + 2.
      // They are non-zero only where the K slots belong to the row's group (t == g).
#pragma unroll
      for (int rb = 0; rb < RB; ++rb) {
        const int h0 = rb * 4 + (gid >> 2), h1 = h0 + 2;
        const __half* q0 = q + ((int64_t)b * Hq + hk * G + h0) * kHeadDim;
        const __half* q1 = q + ((int64_t)b * Hq + hk * G + h1) * kHeadDim;
        const bool on = (t == g);
        const bool v0 = on && h0 < G, v1 = on && h1 < G;
        float s0 = 0.f, s1 = 0.f;
#pragma unroll
        for (int s = 0; s < 8; ++s) {
          const int e = (s & 1) * 2, base = 32 * t + 8 * (s >> 1);
          const __half z = __float2half_rn(0.f);
          const __half x00 = v0 ? q0[base + e] : z, x01 = v0 ? q0[base + e + 4] : z;
          const __half x02 = v0 ? q0[base + e + 1] : z, x03 = v0 ? q0[base + e + 5] : z;
          const __half x10 = v1 ? q1[base + e] : z, x11 = v1 ? q1[base + e + 4] : z;
          const __half x12 = v1 ? q1[base + e + 1] : z, x13 = v1 ? q1[base + e + 5] : z;
          afr[rb][s][0] = pack_h2(x00, x01);
          afr[rb][s][1] = pack_h2(x10, x11);
          afr[rb][s][2] = pack_h2(x02, x03);
          afr[rb][s][3] = pack_h2(x12, x13);
          s0 += (__half2float(x00) + __half2float(x01)) + (__half2float(x02) + __half2float(x03));
          s1 += (__half2float(x10) + __half2float(x11)) + (__half2float(x12) + __half2float(x13));
        }
        qsum[rb][0] = s0;   // Q[h0][g] on lanes with t == g
        qsum[rb][1] = s1;
      }
      staged = u;
    }
    const int cw0 = (it % tiles) * kEstTile + warp * 32;
    const int Cu = min(has_cand ? __ldg(ncand + u) * kPage : L.len(b), cmax);
    float mlo[RB], mhi[RB];
    float lgv[kEstTiles][RB][4];
#pragma unroll
    for (int rb = 0; rb < RB; ++rb) mlo[rb] = mhi[rb] = -INFINITY;
#pragma unroll
    for (int k = 0; k < kEstTiles; ++k) {
      float acc[RB][4];
#pragma unroll
      for (int rb = 0; rb < RB; ++rb) acc[rb][0] = acc[rb][1] = acc[rb][2] = acc[rb][3] = 0.f;
      const uint32_t w[4] = {A.cw[k].x, A.cw[k].y, A.cw[k].z, A.cw[k].w};
#pragma unroll
      for (int s = 0; s < 8; ++s) {
        const uint32_t W = w[s >> 1];
        const int e = (s & 1) * 2;
        const uint32_t b0 = nib_pair(W, e), b1 = nib_pair(W, e + 1);
#pragma unroll
        for (int rb = 0; rb < RB; ++rb) mma16816(acc[rb], afr[rb][s], b0, b1);
      }
      // epilogue: this lane holds rows (h0, g), (h1, g) for candidates 2t, 2t+1
      const uint32_t sz0 = __shfl_sync(0xffffffffu, A.sz[k], (2 * t) * 4 + g);
      const uint32_t sz1 = __shfl_sync(0xffffffffu, A.sz[k], (2 * t + 1) * 4 + g);
      const int tk0 = __shfl_sync(0xffffffffu, tokA[k], (2 * t) * 4);
      const int tk1 = __shfl_sync(0xffffffffu, tokA[k], (2 * t + 1) * 4);
      const float sc0 = __half2float(__ushort_as_half((unsigned short)(sz0 & 0xFFFF)));
      const float sc1 = __half2float(__ushort_as_half((unsigned short)(sz1 & 0xFFFF)));
      const float zz0 = __fmaf_rn(8.f, sc0, __half2float(__ushort_as_half((unsigned short)(sz0 >> 16))));
      const float zz1 = __fmaf_rn(8.f, sc1, __half2float(__ushort_as_half((unsigned short)(sz1 >> 16))));
#pragma unroll
      for (int rb = 0; rb < RB; ++rb) {
        const float Qlo = __shfl_sync(0xffffffffu, qsum[rb][0], gid * 4 + g);
        const float Qhi = __shfl_sync(0xffffffffu, qsum[rb][1], gid * 4 + g);
        float v[4];
        v[0] = __fmaf_rn(sc0, acc[rb][0], zz0 * Qlo);
        v[1] = __fmaf_rn(sc1, acc[rb][1], zz1 * Qlo);
        v[2] = __fmaf_rn(sc0, acc[rb][2], zz0 * Qhi);
        v[3] = __fmaf_rn(sc1, acc[rb][3], zz1 * Qhi);
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          v[j] += __shfl_xor_sync(0xffffffffu, v[j], 4);
          v[j] += __shfl_xor_sync(0xffffffffu, v[j], 8);
        }
        lgv[k][rb][0] = tk0 >= 0 ? v[0] * kInvSqrtD : -INFINITY;
        lgv[k][rb][1] = tk1 >= 0 ? v[1] * kInvSqrtD : -INFINITY;
        lgv[k][rb][2] = tk0 >= 0 ? v[2] * kInvSqrtD : -INFINITY;
        lgv[k][rb][3] = tk1 >= 0 ? v[3] * kInvSqrtD : -INFINITY;
        mlo[rb] = fmaxf(mlo[rb], fmaxf(lgv[k][rb][0], lgv[k][rb][1]));
        mhi[rb] = fmaxf(mhi[rb], fmaxf(lgv[k][rb][2], lgv[k][rb][3]));
      }
    }
    if (cw0 < Cu) {
      // logits [unit][lcap][G], written by the lanes with g == 0
      if (g == 0) {
#pragma unroll
        for (int k = 0; k < kEstTiles; ++k) {
          const int c0 = cw0 + k * 8 + 2 * t;
#pragma unroll
          for (int rb = 0; rb < RB; ++rb) {
            const int h0 = rb * 4 + (gid >> 2), h1 = h0 + 2;
            float* lp = logits + ((int64_t)u * lcap + c0) * G;
            if (h0 < G) {
              if (c0 < Cu) lp[h0] = lgv[k][rb][0];
              if (c0 + 1 < Cu) lp[G + h0] = lgv[k][rb][1];
            }
            if (h1 < G) {
              if (c0 < Cu) lp[h1] = lgv[k][rb][2];
              if (c0 + 1 < Cu) lp[G + h1] = lgv[k][rb][3];
            }
          }
        }
      }
      // this warp's softmax statistics per head (32 candidates)
#pragma unroll
      for (int h = 0; h < G; ++h) {
        const int rb = h >> 2, hh = h & 3;   // head hh of block rb: slot lo if hh < 2, gid>>2 == hh & 1
        const bool mine = g == 0 && ((gid >> 2) == (hh & 1));
        const bool lo = hh < 2;
        float m = mine ? (lo ? mlo[rb] : mhi[rb]) : -INFINITY;
        m = warp_max(m);
        float z = 0.f;
        if (mine && m != -INFINITY) {
#pragma unroll
          for (int k = 0; k < kEstTiles; ++k) {
            const float a = lo ? lgv[k][rb][0] : lgv[k][rb][2];
            const float c = lo ? lgv[k][rb][1] : lgv[k][rb][3];
            if (a != -INFINITY) z += expf(a - m);
            if (c != -INFINITY) z += expf(c - m);
          }
        }
        z = warp_sum(z);
        if (lane == 0) stats[((int64_t)u * nspan + cw0 / kStatSpan) * G + h] = make_float2(m, z);
      }
    }
    if (it + 2 < it1) est_tokens(ids, has_cand, cmax, tiles, it + 2, warp, gid, tokA);
    // rotate the pipeline: A <- B (item it+1), tokB <- candidates of item it+2
#pragma unroll
    for (int k = 0; k < kEstTiles; ++k) {
      const int t2 = tokA[k];
      tokA[k] = tokB[k];
      tokB[k] = t2;
      A.cw[k] = B.cw[k];
      A.sz[k] = B.sz[k];
    }
  }
  griddep_launch();
}

template <int G>
static int est_grid(int num_sms) {
  static int per_sm = 0;
  if (per_sm == 0) {
    int n = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, k_estimate<G>, kEstThreads, 0) !=
            cudaSuccess || n < 1)
      n = 1;
    per_sm = n;
  }
  return num_sms * per_sm;
}

cudaError_t launch_estimate(const Layout& L, const __half* q, int Hq, const uint8_t* codes,
                            const __half* scales, const __half* zeros, const int32_t* cand,
                            int cand_stride, const int32_t* ncand, int lcap, int cmax,
                            float* logits, float2* stats, cudaStream_t st, int num_sms,
                            bool pdl) {
  const int G = Hq / L.Hk;
  const int items = L.B * L.Hk * (lcap / kEstTile);
  switch (G) {
#define TW_EST(GG)                                                                          \
  case GG: {                                                                                \
    const int grid = items < est_grid<GG>(num_sms) ? items : est_grid<GG>(num_sms);        \
    return launch_k(k_estimate<GG>, dim3(grid), dim3(kEstThreads), 0, st, pdl, L, q, Hq,    \
                    codes, scales, zeros, cand, cand_stride, ncand, lcap, cmax, logits,     \
                    stats);                                                                 \
  }
    TW_EST(1) TW_EST(2) TW_EST(4) TW_EST(8)
#undef TW_EST
  }
  return cudaErrorInvalidValue;
}

}  // namespace tw
