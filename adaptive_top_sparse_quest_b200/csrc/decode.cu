// Exact attention over the tokens that survive Twilight's top-p pruning:
// load-balanced split-K flash decoding with a fused log-sum-exp merge.
//
// After pruning, attention runs only over the selected tokens' fp16 K/V
// ("Twilight: Adaptive Attention Sparsity with Hierarchical Top-p Pruning",
// atlas.scime.ai summary, "Approach": select-then-prune, then sparse attention;
// its kernels build on FlashInfer, "Experimental setup").
//
// Work split.  The selected-token counts are only known on the device and
// differ per set (head or KV group) by an order of magnitude, so a fixed split
// per set leaves most of the GPU idle.  The selected tokens of all sets are
// viewed as one concatenated list of S tokens and a grid of n CTAs (up to
// kDecCtas, fewer for a few wide GQA sets; see decode_grid) takes equal
// contiguous ranges: CTA c owns [c*S/n, (c+1)*S/n).  Each CTA
// derives the set offsets from the counts.  For every set its range touches,
// the CTA writes one partial record {m, l, acc[128]} per query head to slot
// (c + set), unique because (c, set) pairs advance monotonically along the
// list.
//
// Data path.  The kept tokens arrive as physical K/V row indices (the top-p
// kernel, or a resolve kernel for caller-given ids, maps ids through the page
// table; kNoRow marks an id outside the sequence), so no page-table load sits
// in front of a gather.  The rows of a window of the range are staged in
// shared memory once; the gathered 256-byte K and V rows then stream through a
// 6-stage cp.async ring of 16 tokens per stage (40 KB in flight per CTA, four
// CTAs per SM: about the whole working set of a 32k-context step at once), so
// a CTA pays one dependent round trip per window instead of one per batch.
// Each half-warp takes 2 tokens of a stage; lane l of the half-warp holds
// channels 8l..8l+7, the scores are reduced with 4 xor-shuffles and the online
// softmax is kept in the log2 domain.  The NH query heads of a KV group reuse
// every staged row.
//
// Merge.  After writing its record for a set, a CTA bumps the set's counter;
// the CTA that completes the set folds all of its records:
//   out = sum_r 2^(m_r-M) acc_r / sum_r 2^(m_r-M) l_r,
//   lse = ln 2 * (M + log2 sum_r 2^(m_r-M) l_r),
// and resets the counter.  Sets with no selected token get out = 0, lse = -inf.
#include "tw_common.cuh"
#include "tw_kernels.h"

namespace tw {

constexpr int kDecThreads = 128;
constexpr int kDecHW = kDecThreads / 16;       // half-warps
constexpr int kStageTok = 16;                  // tokens per pipeline stage
constexpr int kStages = 6;                     // 5 stages (40 KB) in flight per CTA
constexpr int kWin = 512;                      // token rows staged per window
constexpr int kMinTokPerCta = 64;              // few-set path: tokens per CTA at least
constexpr float kLog2e = 1.4426950408889634f;

__device__ __forceinline__ void h8_to_f8(uint4 r, float* f) {
  const uint32_t w[4] = {r.x, r.y, r.z, r.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const float2 t = __half22float2(*reinterpret_cast<const __half2*>(&w[i]));
    f[2 * i] = t.x;
    f[2 * i + 1] = t.y;
  }
}

__device__ __forceinline__ void cp_async16(void* smem, const void* gmem) {
  const unsigned s = (unsigned)__cvta_generic_to_shared(smem);
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(s), "l"(gmem) : "memory");
}
__device__ __forceinline__ void cp_async_commit() {
  asm volatile("cp.async.commit_group;" ::: "memory");
}
template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

__device__ __forceinline__ int64_t block_sum_i64(int64_t v, int64_t* sh) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  v = warp_sum(v);
  __syncthreads();
  if (lane == 0) sh[warp] = v;
  __syncthreads();
  int64_t t = 0;
#pragma unroll
  for (int i = 0; i < kDecThreads / 32; ++i) t += sh[i];
  return t;
}

__device__ __forceinline__ bool range_has(int64_t c, int64_t S, int n, int64_t off, int cnt) {
  const int64_t lo = c * S / n, hi = (c + 1) * S / n;
  return lo < hi && lo < off + cnt && hi > off;
}

// Merge layout: 32 lanes with a float4 each cover one head's 128 channels.
// With fewer than 4 heads the warps also split the records (RS ways); with 8
// heads each thread carries two heads.  The records' accumulator rows are
// staged in shared memory (the idle K/V ring) by cp.async, kMergeStageBytes
// at a time.
constexpr int kMergeStageBytes = 36 * 1024;

template <int NH>
struct MergeShape {
  static constexpr int RS = NH >= 4 ? 1 : 4 / NH;    // record split
  static constexpr int HPT = NH > 4 ? NH / 4 : 1;    // heads per thread
  static constexpr int CAP = kMergeStageBytes / (NH * kHeadDim * 4);   // records per staged batch
};

template <int NH>
struct DecSmem {
  uint32_t rows[kWin];
  union {
    __half kv[kStages][kStageTok][2][kHeadDim];                 // K row, V row
    struct {
      float m[kDecHW][NH], l[kDecHW][NH];
      float acc[kDecHW][NH][kHeadDim];
    } comb;
    struct {
      float4 stage[MergeShape<NH>::CAP][NH][kHeadDim / 4];      // staged accumulator rows
      float f[NH][kDecThreads];                                 // weights of a chunk of records
      float red[kDecThreads / 32][NH];
      float4 acc[MergeShape<NH>::RS][NH][kHeadDim / 4];         // per-split partial sums
    } merge;
  } u;
  int64_t red64[kDecThreads / 32];
  int list_set[kDecThreads];
  long long list_off[kDecThreads];
  unsigned wcnt[kDecThreads / 32];
  int nlist;
  int last;
};

// Fold the records of `set` into out / lse (called by the CTA that completes
// it).  All heads are folded together.  The records were written by other
// CTAs of this launch, so they are read through L2 only (ld.global.cg and
// cp.async.cg).  The first batch of accumulator rows is requested before the
// (m, l) pairs, so a set whose records fit one batch costs one round trip.
template <int NH>
__device__ void merge_set(DecSmem<NH>& sm, int set, int64_t c0, int nspan, bool conc, int64_t off,
                          int cnt, int64_t S, int n_ctas, int Hq, int hq0, int b,
                          const float* part, __half* out, float* lse) {
  using MS = MergeShape<NH>;
  const int t = threadIdx.x, lane = t & 31, warp = t >> 5;
  // the set's records sit in the slots of CTAs c0 .. c0 + nrec - 1; with the
  // concatenated split some of those CTAs may have had an empty range
  const int nrec = conc ? (int)(((off + cnt) * n_ctas + S - 1) / S - 1 - c0 + 1) : nspan;
  auto rec_ptr = [&](int r, int h) { return part + ((c0 + r + set) * NH + h) * kPartStride; };
  auto valid = [&](int r) { return !conc || range_has(c0 + r, S, n_ctas, off, cnt); };
  // stage the accumulator rows of records [r0, r0 + nr); a slot of a record
  // that was never written (an empty range) is copied too but gets weight 0
  auto stage = [&](int r0, int nr) {
    for (int x = t; x < nr * NH * (kHeadDim / 4); x += kDecThreads) {
      const int r = x / (NH * (kHeadDim / 4)), h = (x / (kHeadDim / 4)) % NH, q4 = x % (kHeadDim / 4);
      cp_async16(&sm.u.merge.stage[r][h][q4], rec_ptr(r0 + r, h) + kPartAcc + 4 * q4);
    }
    cp_async_commit();
  };
  __syncthreads();   // the shared union was used by the caller
  stage(0, min(nrec, MS::CAP));
  // 1. per-head max over the records; the first chunk's (m, l) stay in registers
  float m0[NH], l0[NH], mx[NH];
  const bool v0 = t < nrec && valid(t);
#pragma unroll
  for (int h = 0; h < NH; ++h) {
    const float2 ml = v0 ? __ldcg(reinterpret_cast<const float2*>(rec_ptr(t, h)))
                         : make_float2(-INFINITY, 0.f);
    m0[h] = ml.x;
    l0[h] = ml.y;
    mx[h] = ml.x;
  }
  for (int r = t + kDecThreads; r < nrec; r += kDecThreads)
    if (valid(r))
#pragma unroll
      for (int h = 0; h < NH; ++h) mx[h] = fmaxf(mx[h], __ldcg(rec_ptr(r, h)));
#pragma unroll
  for (int h = 0; h < NH; ++h) {
    const float v = warp_max(mx[h]);
    if (lane == 0) sm.u.merge.red[warp][h] = v;
  }
  __syncthreads();
  float M[NH];
#pragma unroll
  for (int h = 0; h < NH; ++h) {
    M[h] = sm.u.merge.red[0][h];
#pragma unroll
    for (int w = 1; w < kDecThreads / 32; ++w) M[h] = fmaxf(M[h], sm.u.merge.red[w][h]);
  }
  // 2. chunks of 128 records: weights 2^(m_r - M), then the staged rows
  const int rs = warp / (NH >= 4 ? 4 : NH) % MS::RS;    // this warp's record split
  const int hbase = NH >= 4 ? warp : warp % NH;          // first head of this thread
  float Lp[NH];
  float4 A[MS::HPT];
#pragma unroll
  for (int h = 0; h < NH; ++h) Lp[h] = 0.f;
#pragma unroll
  for (int k = 0; k < MS::HPT; ++k) A[k] = make_float4(0.f, 0.f, 0.f, 0.f);
  bool staged_first = true;
  for (int w0 = 0; w0 < nrec; w0 += kDecThreads) {
    const int r = w0 + t;
    bool vr = v0;
    float mr[NH], lr[NH];
#pragma unroll
    for (int h = 0; h < NH; ++h) {
      mr[h] = m0[h];
      lr[h] = l0[h];
    }
    if (w0 > 0) {
      vr = r < nrec && valid(r);
#pragma unroll
      for (int h = 0; h < NH; ++h) {
        const float2 ml = vr ? __ldcg(reinterpret_cast<const float2*>(rec_ptr(r, h)))
                             : make_float2(-INFINITY, 0.f);
        mr[h] = ml.x;
        lr[h] = ml.y;
      }
    }
    __syncthreads();   // the previous chunk's weights are no longer read
#pragma unroll
    for (int h = 0; h < NH; ++h) {
      const float f = (vr && mr[h] != -INFINITY) ? exp2f(mr[h] - M[h]) : 0.f;
      Lp[h] += lr[h] * f;
      sm.u.merge.f[h][t] = f;
    }
    const int wn = min(kDecThreads, nrec - w0);
    for (int b0 = w0; b0 < w0 + wn; b0 += MS::CAP) {
      const int nr = min(MS::CAP, w0 + wn - b0);
      if (!staged_first) stage(b0, nr);
      staged_first = false;
      cp_async_wait<0>();
      __syncthreads();   // staged rows and weights visible
      for (int i = rs; i < nr; i += MS::RS) {
#pragma unroll
        for (int k = 0; k < MS::HPT; ++k) {
          const int h = hbase + 4 * k;
          const float f = sm.u.merge.f[h][b0 - w0 + i];
          if (f != 0.f) {
            const float4 x = sm.u.merge.stage[i][h][lane];
            A[k].x = __fmaf_rn(f, x.x, A[k].x);
            A[k].y = __fmaf_rn(f, x.y, A[k].y);
            A[k].z = __fmaf_rn(f, x.z, A[k].z);
            A[k].w = __fmaf_rn(f, x.w, A[k].w);
          }
        }
      }
      __syncthreads();   // the stage is refilled by the next batch
    }
  }
  // 3. totals: sum of l-weights per head, the record splits' partial rows
#pragma unroll
  for (int h = 0; h < NH; ++h) {
    const float v = warp_sum(Lp[h]);
    if (lane == 0) sm.u.merge.red[warp][h] = v;
  }
#pragma unroll
  for (int k = 0; k < MS::HPT; ++k) sm.u.merge.acc[rs][hbase + 4 * k][lane] = A[k];
  __syncthreads();
  if (rs == 0) {
#pragma unroll
    for (int k = 0; k < MS::HPT; ++k) {
      const int h = hbase + 4 * k;
      float Ls = 0.f;
#pragma unroll
      for (int w = 0; w < kDecThreads / 32; ++w) Ls += sm.u.merge.red[w][h];
      float4 a = sm.u.merge.acc[0][h][lane];
#pragma unroll
      for (int s2 = 1; s2 < MS::RS; ++s2) {
        const float4 e = sm.u.merge.acc[s2][h][lane];
        a.x += e.x;
        a.y += e.y;
        a.z += e.z;
        a.w += e.w;
      }
      const float inv = Ls > 0.f ? 1.0f / Ls : 0.f;
      const int64_t bh = (int64_t)b * Hq + hq0 + h;
      __half2 o2[2] = {__floats2half2_rn(a.x * inv, a.y * inv), __floats2half2_rn(a.z * inv, a.w * inv)};
      *reinterpret_cast<uint2*>(out + bh * kHeadDim + 4 * lane) = *reinterpret_cast<uint2*>(o2);
      if (lse && lane == 0) lse[bh] = Ls > 0.f ? (M[h] + log2f(Ls)) * 0.6931471805599453f : -INFINITY;
    }
  }
}

template <int NH>
__global__ void __launch_bounds__(kDecThreads, NH >= 8 ? 2 : 4)   // 4 CTAs per SM: kDecCtas in one wave
k_sparse_decode(Layout L, const __half* __restrict__ q, int Hq, int G, int group_sets,
                const __half* __restrict__ K, const __half* __restrict__ V,
                const uint32_t* __restrict__ rows, int icap, const int32_t* __restrict__ count,
                int nsets, float* __restrict__ part, int32_t* __restrict__ done,
                __half* __restrict__ out, float* __restrict__ lse) {
  extern __shared__ __align__(16) unsigned char dec_smem_raw[];
  DecSmem<NH>& sm = *reinterpret_cast<DecSmem<NH>*>(dec_smem_raw);
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int hw = tid >> 4, l16 = tid & 15;
  const unsigned hmask = 0xFFFFu << (lane & 16);
  const int n = gridDim.x, c = blockIdx.x;
  griddep_wait();

  auto set_heads = [&](int set, int& b, int& hk, int& hq0) {
    if (group_sets) {
      b = set / L.Hk;
      hk = set % L.Hk;
      hq0 = hk * G;
    } else {
      b = set / Hq;
      hq0 = set % Hq;
      hk = hq0 / G;
    }
  };

  // total selected tokens; sets with none get out = 0 here (one CTA each)
  int64_t loc = 0;
  for (int s = tid; s < nsets; s += kDecThreads) loc += max(0, min(count[s], icap));
  const int64_t S = block_sum_i64(loc, sm.red64);
  for (int s = c; s < nsets; s += n) {
    if (max(0, min(count[s], icap)) == 0) {
      int b, hk, hq0;
      set_heads(s, b, hk, hq0);
      for (int h = 0; h < NH; ++h) {
        const int64_t bh = (int64_t)b * Hq + hq0 + h;
        out[bh * kHeadDim + tid] = __float2half_rn(0.f);
        if (lse && tid == 0) lse[bh] = -INFINITY;
      }
    }
  }
  const float qscale = kLog2e * 0.08838834764831845f;   // log2(e) / sqrt(128)

  // Attention over tokens [lo, hi) of `set` (offsets within the set's list
  // plus soff), writing this CTA's record to slot (c + set); the set has nrec
  // records starting at CTA c0 (conc: some of those CTAs may have empty ranges).
  auto process = [&](int set, int64_t soff, int64_t lo, int64_t hi, int64_t c0, int nrec,
                     bool conc) {
    const int scnt = max(0, min(count[set], icap));
    int b, hk, hq0;
    set_heads(set, b, hk, hq0);
    float qf[NH][8];
#pragma unroll
    for (int h = 0; h < NH; ++h) {
      const uint4 r = *reinterpret_cast<const uint4*>(q + ((int64_t)b * Hq + hq0 + h) * kHeadDim + 8 * l16);
      h8_to_f8(r, qf[h]);
#pragma unroll
      for (int j = 0; j < 8; ++j) qf[h][j] *= qscale;
    }
    float m[NH], l[NH], acc[NH][8];
#pragma unroll
    for (int h = 0; h < NH; ++h) {
      m[h] = -INFINITY;
      l[h] = 0.f;
#pragma unroll
      for (int j = 0; j < 8; ++j) acc[h][j] = 0.f;
    }
    const uint32_t* srows = rows + (int64_t)set * icap;
    for (int64_t w0 = lo; w0 < hi; w0 += kWin) {
      const int wn = (int)min((int64_t)kWin, hi - w0);
      __syncthreads();   // previous window's rows and ring are no longer read
      for (int i = tid; i < wn; i += kDecThreads) {
        sm.rows[i] = srows[w0 - soff + i];
      }
      __syncthreads();
      const int nst = (wn + kStageTok - 1) / kStageTok;
      auto issue = [&](int st) {
        if (st < nst) {
          const int slot = st % kStages;
#pragma unroll
          for (int x = tid; x < kStageTok * 32; x += kDecThreads) {
            const int j = x >> 5, part_ = x & 31;
            const int pos = st * kStageTok + j;
            const uint32_t r = pos < wn ? sm.rows[pos] : kNoRow;
            if (r != kNoRow) {
              const int64_t row = r;
              const __half* src = (part_ < 16 ? K : V) + row * kHeadDim + (part_ & 15) * 8;
              cp_async16(&sm.u.kv[slot][j][part_ >> 4][(part_ & 15) * 8], src);
            }
          }
        }
        cp_async_commit();
      };
#pragma unroll
      for (int st = 0; st < kStages - 1; ++st) issue(st);
      for (int st = 0; st < nst; ++st) {
        issue(st + kStages - 1);
        cp_async_wait<kStages - 1>();
        __syncthreads();
        const int slot = st % kStages;
        float sc[NH][2];
        bool ok[2];
#pragma unroll
        for (int jj = 0; jj < 2; ++jj) {
          const int j = 2 * hw + jj;
          const int pos = st * kStageTok + j;
          ok[jj] = pos < wn && sm.rows[pos] != kNoRow;
          float kf[8];
          h8_to_f8(ok[jj] ? *reinterpret_cast<const uint4*>(&sm.u.kv[slot][j][0][8 * l16])
                          : make_uint4(0u, 0u, 0u, 0u),
                   kf);
#pragma unroll
          for (int h = 0; h < NH; ++h) {
            float s0 = qf[h][0] * kf[0];
#pragma unroll
            for (int dd = 1; dd < 8; ++dd) s0 = __fmaf_rn(qf[h][dd], kf[dd], s0);
            sc[h][jj] = s0;
          }
        }
#pragma unroll
        for (int o = 8; o > 0; o >>= 1)
#pragma unroll
          for (int h = 0; h < NH; ++h) {
            sc[h][0] += __shfl_xor_sync(hmask, sc[h][0], o, 16);
            sc[h][1] += __shfl_xor_sync(hmask, sc[h][1], o, 16);
          }
        if (ok[0] || ok[1]) {   // uniform across the half-warp
          float vf[2][8];
#pragma unroll
          for (int jj = 0; jj < 2; ++jj)
            h8_to_f8(ok[jj] ? *reinterpret_cast<const uint4*>(&sm.u.kv[slot][2 * hw + jj][1][8 * l16])
                            : make_uint4(0u, 0u, 0u, 0u),
                     vf[jj]);
#pragma unroll
          for (int h = 0; h < NH; ++h) {
            float mb = m[h];
            if (ok[0]) mb = fmaxf(mb, sc[h][0]);
            if (ok[1]) mb = fmaxf(mb, sc[h][1]);
            const float corr = exp2f(m[h] - mb);
            const float p0 = ok[0] ? exp2f(sc[h][0] - mb) : 0.f;
            const float p1 = ok[1] ? exp2f(sc[h][1] - mb) : 0.f;
            l[h] = l[h] * corr + (p0 + p1);
#pragma unroll
            for (int dd = 0; dd < 8; ++dd)
              acc[h][dd] = __fmaf_rn(p1, vf[1][dd], __fmaf_rn(p0, vf[0][dd], acc[h][dd] * corr));
            m[h] = mb;
          }
        }
        __syncthreads();   // this slot is refilled by a later issue()
      }
      cp_async_wait<0>();
    }
    // fold the 8 half-warps and write this CTA's record for the set
    __syncthreads();
#pragma unroll
    for (int h = 0; h < NH; ++h) {
      if (l16 == 0) {
        sm.u.comb.m[hw][h] = m[h];
        sm.u.comb.l[hw][h] = l[h];
      }
      *reinterpret_cast<float4*>(&sm.u.comb.acc[hw][h][8 * l16]) =
          make_float4(acc[h][0], acc[h][1], acc[h][2], acc[h][3]);
      *reinterpret_cast<float4*>(&sm.u.comb.acc[hw][h][8 * l16 + 4]) =
          make_float4(acc[h][4], acc[h][5], acc[h][6], acc[h][7]);
    }
    __syncthreads();
    float* rec = part + ((int64_t)(c + set) * NH) * kPartStride;
#pragma unroll
    for (int h = 0; h < NH; ++h) {
      float M = -INFINITY;
#pragma unroll
      for (int w = 0; w < kDecHW; ++w) M = fmaxf(M, sm.u.comb.m[w][h]);
      float Ls = 0.f, A = 0.f;
#pragma unroll
      for (int w = 0; w < kDecHW; ++w) {
        const float f = sm.u.comb.m[w][h] == -INFINITY ? 0.f : exp2f(sm.u.comb.m[w][h] - M);
        Ls += sm.u.comb.l[w][h] * f;
        A += sm.u.comb.acc[w][h][tid] * f;
      }
      rec[h * kPartStride + kPartAcc + tid] = A;
      if (tid == 0) {
        rec[h * kPartStride] = M;
        rec[h * kPartStride + 1] = Ls;
      }
    }
    // publish the record; the CTA that completes the set merges it
    __threadfence();
    __syncthreads();
    if (tid == 0) {
      const int prev = atomicAdd(&done[set], 1);
      sm.last = (prev == nrec - 1);
    }
    __syncthreads();
    if (sm.last) {
      __threadfence();
      merge_set<NH>(sm, set, c0, nrec, conc, soff, scnt, S, n, Hq, hq0, b, part, out, lse);
      if (tid == 0) done[set] = 0;   // ready for the next call
    }
  };

  if ((long long)nsets * 8 <= n) {
    // Few sets: every set gets whole CTAs, so no CTA's range straddles two
    // sets (a straddling CTA pays a second row staging and ring ramp-up, and
    // the set's merge waits for it).  A set with cnt tokens gets
    // 1 + floor(cnt * np / S) CTAs, E the number of non-empty sets and
    // np = min(n - E, S / kMinTokPerCta), so the shares add up to at most n;
    // CTAs past them have no set and exit.
    int64_t ne = 0;
    for (int s = tid; s < nsets; s += kDecThreads) ne += count[s] > 0 && icap > 0 ? 1 : 0;
    const int64_t E = block_sum_i64(ne, sm.red64);
    // at least kMinTokPerCta tokens per CTA: a few small sets leave CTAs
    // idle rather than split into ranges whose fixed costs (row staging,
    // ring ramp-up, one more record in the merge) outweigh their tokens
    int64_t np = n - E;
    if (np > S / kMinTokPerCta) np = S / kMinTokPerCta;
    if (tid == 0) sm.nlist = -1;
    int64_t before = 0;   // CTAs given to the sets of earlier chunks
    for (int base = 0; base < nsets; base += kDecThreads) {
      const int s = base + tid;
      const int cnt = s < nsets ? max(0, min(count[s], icap)) : 0;
      const int ns = cnt > 0 ? 1 + (int)((int64_t)cnt * np / S) : 0;
      int incl = ns;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int t = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += t;
      }
      __syncthreads();
      if (lane == 31) sm.wcnt[warp] = incl;
      __syncthreads();
      int wbefore = 0, chunk = 0;
#pragma unroll
      for (int i = 0; i < kDecThreads / 32; ++i) {
        const int v = (int)sm.wcnt[i];
        if (i < warp) wbefore += v;
        chunk += v;
      }
      const int64_t start = before + wbefore + incl - ns;
      if (ns > 0 && c >= start && c < start + ns) {
        sm.nlist = s;
        sm.list_off[0] = start;
        sm.list_set[0] = ns;
      }
      before += chunk;
    }
    __syncthreads();
    const int set = sm.nlist;
    if (set >= 0) {
      const int64_t start = sm.list_off[0];
      const int ns = sm.list_set[0];
      const int cnt = max(0, min(count[set], icap));
      const int64_t j = c - start;
      process(set, 0, j * cnt / ns, (j + 1) * cnt / ns, start, ns, false);
    }
    griddep_launch();
    return;
  }

  // Many sets: CTA c takes [c*S/n, (c+1)*S/n) of the concatenated list.
  const int64_t begin = (int64_t)c * S / n, end = (int64_t)(c + 1) * S / n;
  if (begin >= end) {
    griddep_launch();
    return;
  }
  int64_t running = 0;
  for (int base = 0; base < nsets && running < end; base += kDecThreads) {
    // offsets of this chunk of sets, and the sets that overlap [begin, end)
    const int s = base + tid;
    const int cnt = s < nsets ? max(0, min(count[s], icap)) : 0;
    int incl = cnt;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int t = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += t;
    }
    __syncthreads();
    if (lane == 31) sm.wcnt[warp] = incl;
    if (tid == 0) sm.nlist = 0;
    __syncthreads();
    int wbefore = 0, chunk = 0;
#pragma unroll
    for (int i = 0; i < kDecThreads / 32; ++i) {
      const int v = (int)sm.wcnt[i];
      if (i < warp) wbefore += v;
      chunk += v;
    }
    const int64_t off = running + wbefore + incl - cnt;
    const bool hit = cnt > 0 && off < end && off + cnt > begin;
    const unsigned bal = __ballot_sync(0xffffffffu, hit);
    __syncthreads();
    if (lane == 0 && bal) sm.wcnt[warp] = atomicAdd(&sm.nlist, __popc(bal));
    __syncthreads();
    if (hit) {
      const int slot = sm.wcnt[warp] + __popc(bal & ((1u << lane) - 1u));
      sm.list_set[slot] = s;
      sm.list_off[slot] = off;
    }
    __syncthreads();
    const int nl = sm.nlist;   // record slots depend only on (c, set): order does not matter
    running += chunk;
    for (int li = 0; li < nl; ++li) {
      const int set = sm.list_set[li];
      const int64_t soff = sm.list_off[li];
      const int scnt = max(0, min(count[set], icap));
      // the records of the set: CTAs c0..c1, some possibly with empty ranges
      const int64_t c0 = ((soff + 1) * n + S - 1) / S - 1;
      const int64_t c1 = ((soff + scnt) * n + S - 1) / S - 1;
      int nrec = 0;
      if (S >= n) {
        nrec = (int)(c1 - c0 + 1);
      } else {
        for (int64_t cc = c0; cc <= c1; ++cc) nrec += range_has(cc, S, n, soff, scnt) ? 1 : 0;
      }
      process(set, soff, max(begin, soff), min(end, soff + scnt), c0, nrec, true);
    }
    __syncthreads();
  }
  griddep_launch();
}

// Grid of the attention kernel: kDecCtas CTAs share the concatenated selected
// tokens, but a set's partial records are folded by one CTA, which reads them
// through L2 at a few tens of GB/s.  So few, wide sets (GQA at batch 1) get
// fewer CTAs: at most about 128 / NH records of 512 B per head and set (64 KB),
// never fewer than two CTAs per SM.
static int decode_grid(int nsets, int NH) {
  const long long want = (long long)nsets * (128 / NH);
  const int lo = 2 * kTargetSms;
  return want < lo ? lo : (want > kDecCtas ? kDecCtas : (int)want);
}

template <int NH>
static cudaError_t dec_prepare() {
  static std::atomic<int> done[kMaxDevices];
  return once_per_device(done, [] {
    return cudaFuncSetAttribute(k_sparse_decode<NH>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                (int)sizeof(DecSmem<NH>));
  });
}

size_t decode_part_floats(int B, int Hq, int Hk) {
  const int G = Hq / Hk;
  const size_t grp = (size_t)(kDecCtas + B * Hk) * G * kPartStride;
  const size_t head = (size_t)(kDecCtas + B * Hq) * kPartStride;
  return grp > head ? grp : head;
}

cudaError_t launch_sparse_decode(const Layout& L, const __half* q, int Hq, int group_sets,
                                 const __half* K, const __half* V, const uint32_t* rows, int icap,
                                 const int32_t* count, float* part, int32_t* done, __half* out,
                                 float* lse, cudaStream_t st, bool pdl) {
  const int G = Hq / L.Hk;
  const int NH = group_sets ? G : 1;
  const int nsets = group_sets ? L.B * L.Hk : L.B * Hq;
  switch (NH) {
#define TW_DEC(NN)                                                                           \
  case NN: {                                                                                 \
    const cudaError_t e = dec_prepare<NN>();                                                 \
    if (e != cudaSuccess) return e;                                                          \
    return launch_k(k_sparse_decode<NN>, dim3(decode_grid(nsets, NN)), dim3(kDecThreads),    \
                    sizeof(DecSmem<NN>), st, pdl, L, q, Hq, G, group_sets, K, V, rows, icap, \
                    count, nsets, part, done, out, lse);                                     \
  }
    TW_DEC(1) TW_DEC(2) TW_DEC(4) TW_DEC(8)
#undef TW_DEC
  }
  return cudaErrorInvalidValue;
}

}  // namespace tw
