// Exact attention over the tokens that survive Twilight's top-p pruning:
// split-K flash decoding with a log-sum-exp merge.
//
// After pruning, attention runs only over the selected tokens' fp16 K/V
// ("Twilight: Adaptive Attention Sparsity with Hierarchical Top-p Pruning",
// atlas.scime.ai summary, "Approach": select-then-prune, then sparse attention;
// its kernels build on FlashInfer, "Experimental setup").
//
// k_sparse_decode: block (split, set); the split covers idx[split*T, split*T+T).
//   Each warp walks every 4th selected token; lane l owns channels 4l..4l+3,
//   so a gathered 256-byte K or V row is one coalesced 8-byte load per lane.
//   Rows for 8 tokens are loaded before any math (64 B of K + V per lane in
//   flight per batch).  The NH query heads that share the set reuse every
//   gathered row.  Online softmax in the log2 domain; the 4 warps' partial
//   (max, sum, acc) are combined in shared memory and one record per (query
//   head, split) is written: {m, l, -, -, acc[128]} fp32.
// k_merge: one block per (b, query head); out = sum_s 2^(m_s-M) acc_s /
//   sum_s 2^(m_s-M) l_s, lse = ln 2 * (M + log2 sum_s 2^(m_s-M) l_s).
#include "tw_common.cuh"
#include "tw_kernels.h"

namespace tw {

constexpr int kDecThreads = 128;
constexpr int kDecWarps = kDecThreads / 32;
constexpr int kDecBatch = 8;
constexpr float kLog2e = 1.4426950408889634f;

__device__ __forceinline__ void h4_to_f4(uint2 r, float* f) {
  const __half2 a = *reinterpret_cast<const __half2*>(&r.x);
  const __half2 b = *reinterpret_cast<const __half2*>(&r.y);
  const float2 fa = __half22float2(a), fb = __half22float2(b);
  f[0] = fa.x;
  f[1] = fa.y;
  f[2] = fb.x;
  f[3] = fb.y;
}

template <int NH>
__global__ void __launch_bounds__(kDecThreads)
k_sparse_decode(Layout L, const __half* __restrict__ q, int Hq, int G, int group_sets,
                const __half* __restrict__ K, const __half* __restrict__ V,
                const int32_t* __restrict__ idx, int icap, const int32_t* __restrict__ count,
                int T, int S, float* __restrict__ part) {
  __shared__ float sm_m[kDecWarps][NH], sm_l[kDecWarps][NH];
  __shared__ __align__(16) float sm_acc[kDecWarps][NH][kHeadDim];
  const int set = blockIdx.y, split = blockIdx.x;
  const int n = min(count[set], icap);
  const int start = split * T;
  if (start >= n) return;
  const int end = min(n, start + T);
  int b, hk, hq0;
  if (group_sets) {
    b = set / L.Hk;
    hk = set % L.Hk;
    hq0 = hk * G;
  } else {
    b = set / Hq;
    hq0 = set % Hq;
    hk = hq0 / G;
  }
  const int len = L.len(b);
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const float qscale = kLog2e * 0.08838834764831845f;   // log2(e) / sqrt(128)
  float qf[NH][4];
#pragma unroll
  for (int h = 0; h < NH; ++h) {
    const uint2 r = *reinterpret_cast<const uint2*>(q + ((int64_t)b * Hq + hq0 + h) * kHeadDim + 4 * lane);
    h4_to_f4(r, qf[h]);
#pragma unroll
    for (int j = 0; j < 4; ++j) qf[h][j] *= qscale;
  }
  float m[NH], l[NH], acc[NH][4];
#pragma unroll
  for (int h = 0; h < NH; ++h) {
    m[h] = -INFINITY;
    l[h] = 0.f;
#pragma unroll
    for (int j = 0; j < 4; ++j) acc[h][j] = 0.f;
  }
  const int32_t* ids = idx + (int64_t)set * icap;
  for (int i0 = start + warp; i0 < end; i0 += kDecWarps * kDecBatch) {
    uint2 kr[kDecBatch], vr[kDecBatch];
    bool ok[kDecBatch];
#pragma unroll
    for (int j = 0; j < kDecBatch; ++j) {
      const int i = i0 + j * kDecWarps;
      ok[j] = false;
      if (i < end) {
        const int t = ids[i];
        ok[j] = (unsigned)t < (unsigned)len;   // ids outside [0, len) are ignored
        if (ok[j]) {
          const int64_t row = L.row(b, hk, t);
          kr[j] = ld_stream8(K + row * kHeadDim + 4 * lane);
          vr[j] = ld_stream8(V + row * kHeadDim + 4 * lane);
        }
      }
    }
#pragma unroll
    for (int j = 0; j < kDecBatch; ++j) {
      if (!ok[j]) continue;   // uniform across the warp
      float kf[4], vf[4];
      h4_to_f4(kr[j], kf);
      h4_to_f4(vr[j], vf);
#pragma unroll
      for (int h = 0; h < NH; ++h) {
        float s = qf[h][0] * kf[0];
        s = __fmaf_rn(qf[h][1], kf[1], s);
        s = __fmaf_rn(qf[h][2], kf[2], s);
        s = __fmaf_rn(qf[h][3], kf[3], s);
        s = warp_sum(s);
        const float mn = fmaxf(m[h], s);
        const float corr = exp2f(m[h] - mn);
        const float pr = exp2f(s - mn);
        l[h] = l[h] * corr + pr;
#pragma unroll
        for (int d = 0; d < 4; ++d) acc[h][d] = __fmaf_rn(pr, vf[d], acc[h][d] * corr);
        m[h] = mn;
      }
    }
  }
#pragma unroll
  for (int h = 0; h < NH; ++h) {
    if (lane == 0) {
      sm_m[warp][h] = m[h];
      sm_l[warp][h] = l[h];
    }
    *reinterpret_cast<float4*>(&sm_acc[warp][h][4 * lane]) =
        make_float4(acc[h][0], acc[h][1], acc[h][2], acc[h][3]);
  }
  __syncthreads();
  // thread tid combines channel tid of every head across the 4 warps
#pragma unroll
  for (int h = 0; h < NH; ++h) {
    float M = -INFINITY;
#pragma unroll
    for (int w = 0; w < kDecWarps; ++w) M = fmaxf(M, sm_m[w][h]);
    float Ls = 0.f, A = 0.f;
#pragma unroll
    for (int w = 0; w < kDecWarps; ++w) {
      const float f = sm_m[w][h] == -INFINITY ? 0.f : exp2f(sm_m[w][h] - M);
      Ls += sm_l[w][h] * f;
      A += sm_acc[w][h][tid] * f;
    }
    float* rec = part + (((int64_t)b * Hq + hq0 + h) * S + split) * kPartStride;
    rec[kPartAcc + tid] = A;
    if (tid == 0) {
      rec[0] = M;
      rec[1] = Ls;
    }
  }
}

__global__ void __launch_bounds__(kHeadDim)
k_merge(int Hq, int Hk, int G, int group_sets, const int32_t* __restrict__ count, int icap, int T,
        int S, const float* __restrict__ part, __half* __restrict__ out, float* __restrict__ lse) {
  const int bh = blockIdx.x;
  const int b = bh / Hq, hq = bh % Hq;
  const int set = group_sets ? b * Hk + hq / G : bh;
  const int n = max(0, min(count[set], icap));
  const int ns = (n + T - 1) / T;
  const int d = threadIdx.x;
  const float* rec = part + (int64_t)bh * S * kPartStride;
  if (ns == 0) {
    out[(int64_t)bh * kHeadDim + d] = __float2half_rn(0.f);
    if (lse && d == 0) lse[bh] = -INFINITY;
    return;
  }
  float M = -INFINITY;
  for (int s = 0; s < ns; ++s) M = fmaxf(M, rec[s * kPartStride]);
  float Ls = 0.f, A = 0.f;
  for (int s = 0; s < ns; ++s) {
    const float ms = rec[s * kPartStride];
    const float f = ms == -INFINITY ? 0.f : exp2f(ms - M);
    Ls += rec[s * kPartStride + 1] * f;
    A += rec[s * kPartStride + kPartAcc + d] * f;
  }
  out[(int64_t)bh * kHeadDim + d] = __float2half_rn(Ls > 0.f ? A / Ls : 0.f);
  if (lse && d == 0) lse[bh] = Ls > 0.f ? (M + log2f(Ls)) * 0.6931471805599453f : -INFINITY;
}

int decode_split_tokens(int sets, int icap) {
  int T = 1024;
  while (T > 64 && (int64_t)sets * ((icap + T - 1) / T) < 4 * kTargetSms) T >>= 1;
  return T;
}

void launch_sparse_decode(const Layout& L, const __half* q, int Hq, int group_sets,
                          const __half* K, const __half* V, const int32_t* idx, int icap,
                          const int32_t* count, float* part, __half* out, float* lse,
                          cudaStream_t st, bool merge_only, bool decode_only) {
  const int G = Hq / L.Hk;
  const int NH = group_sets ? G : 1;
  const int sets = group_sets ? L.B * L.Hk : L.B * Hq;
  const int T = decode_split_tokens(sets, icap);
  const int S = (icap + T - 1) / T;
  if (!merge_only) {
    dim3 grid(S, sets);
    switch (NH) {
#define TW_DEC(NN)                                                                          \
  case NN:                                                                                  \
    k_sparse_decode<NN><<<grid, kDecThreads, 0, st>>>(L, q, Hq, G, group_sets, K, V, idx,    \
                                                      icap, count, T, S, part);              \
    break;
      TW_DEC(1) TW_DEC(2) TW_DEC(4) TW_DEC(8)
#undef TW_DEC
    }
  }
  if (!decode_only)
    k_merge<<<L.B * Hq, kHeadDim, 0, st>>>(Hq, L.Hk, G, group_sets, count, icap, T, S, part, out,
                                           lse);
}

}  // namespace tw
