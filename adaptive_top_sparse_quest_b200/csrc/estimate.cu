// Twilight weight estimation from the quantised key cache, with fused softmax
// statistics ("Twilight: Adaptive Attention Sparsity with Hierarchical Top-p
// Pruning", atlas.scime.ai summary, "Approach": the candidates' attention
// weights are estimated from INT4 keys before top-p pruning; the 2-bit cache
// of its quantisation ablation, table of measured effects, runs through the
// same kernel).
//
// For candidate i, query head h and 32-channel group g with scale s, zero z,
// codes c in 0..n (n = 15 at 4 bits, 3 at 2 bits) and centre o = 8 or 2:
//   k_hat = z + s * c = (z + o s) + s * (c - o)
//   l[i,h] = sum_g ( s_ig * D[i,h,g] + (z_ig + o s_ig) * Q[h,g] ) / sqrt(128)
//   D[i,h,g] = sum_{j in g} (c_ij - o) * q_hj,   Q[h,g] = sum_{j in g} q_hj
// The D terms are a small dense contraction, run on the tensor cores with
// mma.sync m16n8k16 (fp16 operands, fp32 accumulation): (c - o) and the fp16
// queries are exact in fp16 and their products exact in fp32.  M = 16
// candidates, N = 8 columns = (head, group) pairs of two heads, K = 16
// channels per step; column (h, g) keeps only group g's channels of q_h, so
// after 8 K-steps every column holds one D[*,h,g] and the per-group scales are
// applied in the fp32 epilogue, where one xor-shuffle adds the lane pair that
// holds the other two groups.  The K order is permuted so that lane (gid, t)
// feeds exactly the codes of candidates gid and gid+8, group t, it reads
// (16 B at 4 bits, 8 B at 2 bits): each code pair becomes a half2 A-fragment
// with one shift, one LOP3 (codes -> 0x6400|c, i.e. 1024 + c) and one half2
// subtract of 1024 + o.  Logits are kept in log2 units (log2(e) folded into
// the 1/sqrt(128) factor), so the statistics and the top-p kernel use exp2.
//
// Data path.  Persistent CTAs (two per SM) each own a contiguous block of
// work items (kv unit, 16 candidate pages = 256 candidates: 16 KB of codes at
// 4 bits or 8 KB at 2 bits, + 2 KB of scales + 2 KB of zeros).  A 4-stage shared-memory ring is filled
// with cp.async by all threads (16-byte chunks of codes, 8-byte rows of
// scales and zeros) three items ahead.  A page's rows are located from the
// candidate list and a list of first physical rows written by the selector
// (no page-table walk here); warp 0 issues those lookups two items before
// their gathers and stores them one iteration later, so neither the lookups
// nor the gathers sit on the critical path.  Each of the eight warps then takes 32 candidates (two MMA
// tiles) and writes the fp32 logits [unit][G][cap] plus its per-head
// (max, sum 2^(l - max)).
#include "tw_common.cuh"
#include "tw_kernels.h"

namespace tw {

constexpr int kEstThreads = 256;
constexpr int kEstStages = 4;
constexpr int kEstTiles = 2;                             // MMA tiles of 16 candidates per warp
constexpr int kPagesPerItem = kEstTile / kPage;          // 16
constexpr float kL2Scale = 1.4426950408889634f * 0.08838834764831845f;   // log2(e) / sqrt(128)

// Key-cache width: bytes of codes per row, the centre o subtracted from the
// codes, and the channel that feeds MMA k-slot pair j (0: k = 2t, 2t+1; 1:
// k = 2t+8, 2t+9), element hi of the pair, at K-step s, as an offset in the
// lane's group.  4 bits: the word s / 2 of the lane's 16 B holds channels
// 8 (s / 2) + 0..7, and nib_pair takes nibbles (e, e + 4).  2 bits: the word
// s / 4 of the lane's 8 B holds channels 16 (s / 4) + 0..15, and crumb_pair
// takes crumbs (m, m + 8).
template <int BITS>
struct KeyWidth {
  static_assert(BITS == 4 || BITS == 2, "key-cache width");
  static constexpr int kRowBytes = kHeadDim * BITS / 8;
  static constexpr int kLaneBytes = kGroup * BITS / 8;   // one group of one candidate
  static constexpr float kCentre = BITS == 4 ? 8.f : 2.f;
  __device__ static constexpr int chan(int s, int j, int hi) {
    return BITS == 4 ? 8 * (s >> 1) + 2 * (s & 1) + j + 4 * hi
                     : 16 * (s >> 2) + 2 * (s & 3) + j + 8 * hi;
  }
};

template <int BITS>
struct EstStage {
  uint8_t codes[kEstTile][KeyWidth<BITS>::kRowBytes];
  __half scales[kEstTile][kGroups];
  __half zeros[kEstTile][kGroups];
};

// Where the 16 pages of an item live: first global row and valid rows (0 = none).
struct EstPages {
  uint32_t row0[kPagesPerItem];   // physical rows fit 32 bits (checked on the host)
  int rows[kPagesPerItem];
};

template <int BITS>
struct EstSmem {
  EstStage<BITS> st[kEstStages];
  EstPages pg[kEstStages + 2];   // items j .. j+S+1 around iteration j
};

__device__ __forceinline__ void cp_async16(void* smem, const void* gmem) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(
                   (unsigned)__cvta_generic_to_shared(smem)),
               "l"(gmem)
               : "memory");
}
__device__ __forceinline__ void cp_async8(void* smem, const void* gmem) {
  asm volatile("cp.async.ca.shared.global [%0], [%1], 8;" ::"r"(
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

// 2-bit codes m and m+8 of W as the half2 (c_m - 2, c_{m+8} - 2), exact.
__device__ __forceinline__ uint32_t crumb_pair(uint32_t W, int m) {
  uint32_t x = ((W >> (2 * m)) & 0x00030003u) | 0x64006400u;   // (1024 + c) as fp16
  uint32_t r;
  asm("sub.rn.f16x2 %0, %1, %2;" : "=r"(r) : "r"(x), "r"(0x64026402u));   // minus 1026
  return r;
}

// A-fragment half2 of k-slot pair j at K-step s from the lane's codes of one
// candidate (4 words at 4 bits, 2 at 2 bits): channels chan(s, j, 0 / 1).
template <int BITS>
__device__ __forceinline__ uint32_t code_pair(const uint32_t* W, int s, int j) {
  if (BITS == 4) return nib_pair(W[s >> 1], 2 * (s & 1) + j);
  return crumb_pair(W[s >> 2], 2 * (s & 3) + j);
}

__device__ __forceinline__ uint32_t pack_h2(__half lo, __half hi) {
  return (uint32_t)__half_as_ushort(lo) | ((uint32_t)__half_as_ushort(hi) << 16);
}

// Page lookup of one candidate page of item `it`: its page id, the first
// physical row of the page (from the row list the selector or the resolve
// kernel wrote), the unit's candidate count and sequence length.  The loads
// are independent; est_fetch only issues them, est_store consumes them.
struct EstLook {
  int page, C, len;
  uint32_t r0;
};

__device__ __forceinline__ EstLook est_fetch(const Layout& L, const int32_t* cand, int cand_stride,
                                             const int32_t* ncand, const uint32_t* row0,
                                             int cmax, int tiles, int it, int lane) {
  EstLook k;
  const int u = it / tiles;
  const int b = u / L.Hk;
  const int lp = (it % tiles) * kPagesPerItem + lane;   // logical candidate page
  k.len = L.len(b);
  k.C = cand ? ncand[u] * kPage : k.len;
  k.C = min(k.C, cmax);
  k.page = cand ? (lp < cand_stride ? cand[(int64_t)u * cand_stride + lp] : -1) : lp;
  // without a candidate list (every page a candidate) the row is computed here
  k.r0 = lp >= L.max_pages ? 0u
         : row0            ? row0[(int64_t)u * L.max_pages + lp]
                           : (uint32_t)L.page_row(b, u % L.Hk, lp);
  k.C = lp * kPage < k.C ? k.C : 0;   // this page is a candidate only if lp * 16 < C
  return k;
}

__device__ __forceinline__ void est_store(const EstLook& k, int lane, EstPages& out) {
  int rows = 0;
  if (k.C > 0 && k.page >= 0 && (int64_t)k.page * kPage < k.len)
    rows = min(kPage, k.len - k.page * kPage);
  out.rows[lane] = rows;
  out.row0[lane] = rows > 0 ? k.r0 : 0u;
}

// All threads: gather item `it` (pages already looked up) into a ring stage.
template <int BITS>
__device__ __forceinline__ void est_issue(const EstPages& pg, const uint8_t* codes,
                                          const __half* scales, const __half* zeros,
                                          EstStage<BITS>& st) {
  constexpr int kRowBytes = KeyWidth<BITS>::kRowBytes;
  constexpr int kChunks = kRowBytes / 16;   // 16-byte chunks per row: 4 or 2
  const int tid = threadIdx.x;
#pragma unroll
  for (int k = 0; k < kChunks; ++k) {   // codes: 256 rows x kChunks chunks of 16 B
    const int x = tid + k * kEstThreads;
    const int c = x / kChunks, part = x % kChunks, p = c >> 4, r = c & 15;
    if (r < pg.rows[p])
      cp_async16(&st.codes[c][16 * part],
                 codes + (size_t)(pg.row0[p] + r) * kRowBytes + 16 * part);
  }
  {   // scales and zeros: one 8-byte row each per thread
    const int c = tid, p = c >> 4, r = c & 15;
    if (r < pg.rows[p]) {
      cp_async8(&st.scales[c][0], scales + (size_t)(pg.row0[p] + r) * kGroups);
      cp_async8(&st.zeros[c][0], zeros + (size_t)(pg.row0[p] + r) * kGroups);
    }
  }
}

template <int G, int BITS>
__global__ void __launch_bounds__(kEstThreads, 2)
k_estimate(Layout L, const __half* __restrict__ q, int Hq, const uint8_t* __restrict__ codes,
           const __half* __restrict__ scales, const __half* __restrict__ zeros,
           const int32_t* __restrict__ cand, int cand_stride, const int32_t* __restrict__ ncand,
           const uint32_t* __restrict__ row0, int lcap, int cmax, float* __restrict__ logits,
           float2* __restrict__ stats) {
  constexpr int HP = (G + 1) / 2;   // head pairs: one MMA N-block of 8 (head, group) columns each
  using KW = KeyWidth<BITS>;
  extern __shared__ __align__(128) unsigned char est_smem_raw[];
  EstSmem<BITS>& sm = *reinterpret_cast<EstSmem<BITS>*>(est_smem_raw);
  const int tiles = lcap / kEstTile;
  const int items = L.B * L.Hk * tiles;
  const int per = (items + gridDim.x - 1) / gridDim.x;
  const int it0 = blockIdx.x * per;
  const int it1 = min(items, it0 + per);
  if (it0 >= it1) return;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  griddep_wait();
  // pipeline prologue: page lookups of items it0 .. it0+S by all threads at
  // once, the lookups of item it0+S+1 left in flight in warp 0's registers,
  // then the gathers of items it0 .. it0+S-2
  constexpr int kPgRing = kEstStages + 2;
  if (tid < (kEstStages + 1) * kPagesPerItem) {
    const int j = tid / kPagesPerItem, lp = tid % kPagesPerItem;
    if (it0 + j < it1)
      est_store(est_fetch(L, cand, cand_stride, ncand, row0, cmax, tiles, it0 + j, lp), lp,
                sm.pg[j]);
  }
  EstLook ahead = {};
  if (warp == 0 && lane < kPagesPerItem && it0 + kEstStages + 1 < it1)
    ahead = est_fetch(L, cand, cand_stride, ncand, row0, cmax, tiles, it0 + kEstStages + 1, lane);
  __syncthreads();
#pragma unroll
  for (int j = 0; j < kEstStages - 1; ++j) {
    if (it0 + j < it1) est_issue(sm.pg[j], codes, scales, zeros, sm.st[j]);
    cp_async_commit();
  }
  const int gid = lane >> 2, t = lane & 3;
  const int g0 = 2 * (t & 1);            // this lane's two groups in the epilogue: g0, g0 + 1
  const int nspan = lcap / kStatSpan;
  uint32_t bfr[HP][8][2];                // B fragments: column gid = (head 2hp + gid/4, group gid%4)
  float Qv[HP][2];                       // Q[h][g0], Q[h][g0+1] for the lane's epilogue head
  int staged = -1;
  int u = it0 / tiles, tile = it0 % tiles;   // item it = (unit u, candidate tile)
  int b = u / L.Hk, hk = u % L.Hk;
  int Cu = 0;                                // candidates of unit u
  for (int it = it0; it < it1; ++it) {
    const int j = it - it0, slot = j % kEstStages;
    // refill: gather item j+S-1 into the slot item j-1 used, and look up the
    // pages of item j+S (their ring entries were last read one iteration ago)
    __syncthreads();
    if (it + kEstStages - 1 < it1)
      est_issue(sm.pg[(j + kEstStages - 1) % kPgRing], codes, scales, zeros,
                sm.st[(j + kEstStages - 1) % kEstStages]);
    cp_async_commit();
    // warp 0: store the lookups of item j+S+1 (issued one iteration ago) into
    // the slot item j-1 used, and issue those of item j+S+2
    if (warp == 0 && lane < kPagesPerItem) {
      if (it + kEstStages + 1 < it1) est_store(ahead, lane, sm.pg[(j + kEstStages + 1) % kPgRing]);
      if (it + kEstStages + 2 < it1)
        ahead = est_fetch(L, cand, cand_stride, ncand, row0, cmax, tiles, it + kEstStages + 2,
                          lane);
    }
    if (it > it0 && ++tile == tiles) {
      tile = 0;
      ++u;
      if (++hk == L.Hk) {
        hk = 0;
        ++b;
      }
    }
    if (u != staged) {
      Cu = min(cand ? __ldg(ncand + u) * kPage : L.len(b), cmax);
#pragma unroll
      for (int hp = 0; hp < HP; ++hp) {
        const int hb = 2 * hp + (gid >> 2);   // head of B column gid
        const bool on = ((gid & 3) == t) && hb < G;
        const __half* qb = q + ((int64_t)b * Hq + hk * G + min(hb, G - 1)) * kHeadDim;
        const __half z = __float2half_rn(0.f);
        const __half* qg = qb + kGroup * t;   // group t of the column's head
#pragma unroll
        for (int s = 0; s < 8; ++s) {
#pragma unroll
          for (int jj = 0; jj < 2; ++jj)
            bfr[hp][s][jj] = pack_h2(on ? qg[KW::chan(s, jj, 0)] : z,
                                     on ? qg[KW::chan(s, jj, 1)] : z);
        }
        const int he = 2 * hp + (t >> 1);     // head of this lane's epilogue columns
        const __half* qe = q + ((int64_t)b * Hq + hk * G + min(he, G - 1)) * kHeadDim;
        float s0 = 0.f, s1 = 0.f;
        for (int d = 0; d < kGroup; ++d) {
          s0 += __half2float(qe[g0 * kGroup + d]);
          s1 += __half2float(qe[(g0 + 1) * kGroup + d]);
        }
        Qv[hp][0] = s0;
        Qv[hp][1] = s1;
      }
      staged = u;
    }
    cp_async_wait<kEstStages - 1>();
    __syncthreads();
    const EstPages& pgs = sm.pg[j % kPgRing];
    const EstStage<BITS>& st = sm.st[slot];
    const int cw0 = tile * kEstTile + warp * 32;   // this warp's first candidate
    float lg[kEstTiles][HP][2];
#pragma unroll
    for (int k = 0; k < kEstTiles; ++k) {
      const int ca = warp * 32 + k * 16 + gid, cb = ca + 8;   // candidates (rows gid, gid+8)
      uint32_t WA[4], WB[4];
      if (BITS == 4) {
        const uint4 wa = *reinterpret_cast<const uint4*>(&st.codes[ca][KW::kLaneBytes * t]);
        const uint4 wb = *reinterpret_cast<const uint4*>(&st.codes[cb][KW::kLaneBytes * t]);
        WA[0] = wa.x, WA[1] = wa.y, WA[2] = wa.z, WA[3] = wa.w;
        WB[0] = wb.x, WB[1] = wb.y, WB[2] = wb.z, WB[3] = wb.w;
      } else {
        const uint2 wa = *reinterpret_cast<const uint2*>(&st.codes[ca][KW::kLaneBytes * t]);
        const uint2 wb = *reinterpret_cast<const uint2*>(&st.codes[cb][KW::kLaneBytes * t]);
        WA[0] = wa.x, WA[1] = wa.y, WA[2] = WA[3] = 0u;
        WB[0] = wb.x, WB[1] = wb.y, WB[2] = WB[3] = 0u;
      }
      const bool va = (ca & 15) < pgs.rows[ca >> 4];
      const bool vb = (cb & 15) < pgs.rows[cb >> 4];
      float acc[HP][4];
#pragma unroll
      for (int hp = 0; hp < HP; ++hp) acc[hp][0] = acc[hp][1] = acc[hp][2] = acc[hp][3] = 0.f;
#pragma unroll
      for (int s = 0; s < 8; ++s) {
        const uint32_t a[4] = {code_pair<BITS>(WA, s, 0), code_pair<BITS>(WB, s, 0),
                               code_pair<BITS>(WA, s, 1), code_pair<BITS>(WB, s, 1)};
#pragma unroll
        for (int hp = 0; hp < HP; ++hp) mma16816(acc[hp], a, bfr[hp][s][0], bfr[hp][s][1]);
      }
      // scales / zeros of groups g0, g0+1 for both candidates (fp16 pairs)
      const __half2 sa = *reinterpret_cast<const __half2*>(&st.scales[ca][g0]);
      const __half2 za = *reinterpret_cast<const __half2*>(&st.zeros[ca][g0]);
      const __half2 sb = *reinterpret_cast<const __half2*>(&st.scales[cb][g0]);
      const __half2 zb = *reinterpret_cast<const __half2*>(&st.zeros[cb][g0]);
      const float2 fsa = __half22float2(sa), fza = __half22float2(za);
      const float2 fsb = __half22float2(sb), fzb = __half22float2(zb);
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
        lg[k][hp][0] = va ? pa * kL2Scale : -INFINITY;
        lg[k][hp][1] = vb ? pb * kL2Scale : -INFINITY;
      }
    }
    if (cw0 < Cu) {
      const bool owner = (t & 1) == 0;   // lanes t and t^1 hold the same logits
#pragma unroll
      for (int hp = 0; hp < HP; ++hp) {
        const int he = 2 * hp + (t >> 1);
        const bool hv = he < G;
        // logits [unit][G][lcap]: 8 lanes store 8 consecutive candidates of a head
        if (owner && hv) {
          float* lrow = logits + ((int64_t)u * G + he) * lcap;
#pragma unroll
          for (int k = 0; k < kEstTiles; ++k) {
            const int c0 = cw0 + k * 16 + gid;
            if (c0 < Cu) lrow[c0] = lg[k][hp][0];
            if (c0 + 8 < Cu) lrow[c0 + 8] = lg[k][hp][1];
          }
        }
        // (max, sum 2^(l - max)) over this warp's 32 candidates for head he:
        // the max over the 8 lanes (gid) that share t first, then one exp2
        // per logit against it, then the sum over the same lanes
        float m = -INFINITY;
        if (owner && hv) {
#pragma unroll
          for (int k = 0; k < kEstTiles; ++k) m = fmaxf(m, fmaxf(lg[k][hp][0], lg[k][hp][1]));
        }
#pragma unroll
        for (int o = 4; o < 32; o <<= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
        float z = 0.f;
        if (owner && hv && m != -INFINITY) {
#pragma unroll
          for (int k = 0; k < kEstTiles; ++k) {   // exp2(-inf - m) = 0 for masked slots
            z += exp2f(lg[k][hp][0] - m);
            z += exp2f(lg[k][hp][1] - m);
          }
        }
#pragma unroll
        for (int o = 4; o < 32; o <<= 1) z += __shfl_xor_sync(0xffffffffu, z, o);
        if (gid == 0 && owner && hv)
          stats[((int64_t)u * nspan + cw0 / kStatSpan) * G + he] = make_float2(m, z);
      }
    }
  }
  griddep_launch();
}

template <int G, int BITS>
static cudaError_t est_prepare() {
  static std::atomic<int> done[kMaxDevices];
  return once_per_device(done, [] {
    return cudaFuncSetAttribute(k_estimate<G, BITS>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                (int)sizeof(EstSmem<BITS>));
  });
}

template <int G, int BITS>
static cudaError_t est_launch(const Layout& L, const __half* q, int Hq, const uint8_t* codes,
                              const __half* scales, const __half* zeros, const int32_t* cand,
                              int cand_stride, const int32_t* ncand, const uint32_t* row0,
                              int lcap, int cmax, float* logits, float2* stats, cudaStream_t st,
                              int grid, bool pdl) {
  const cudaError_t e = est_prepare<G, BITS>();
  if (e != cudaSuccess) return e;
  return launch_k(k_estimate<G, BITS>, dim3(grid), dim3(kEstThreads), sizeof(EstSmem<BITS>), st,
                  pdl, L, q, Hq, codes, scales, zeros, cand, cand_stride, ncand, row0, lcap, cmax,
                  logits, stats);
}

cudaError_t launch_estimate(const Layout& L, const __half* q, int Hq, const uint8_t* codes,
                            const __half* scales, const __half* zeros, const int32_t* cand,
                            int cand_stride, const int32_t* ncand, const uint32_t* row0,
                            int lcap, int cmax, float* logits, float2* stats, cudaStream_t st,
                            int num_sms, bool pdl) {
  const int G = Hq / L.Hk;
  const int items = L.B * L.Hk * (lcap / kEstTile);
  const int grid = items < 2 * num_sms ? items : 2 * num_sms;
  const bool two = L.kbits == 2;
  switch (G) {
#define TW_EST(GG)                                                                               \
  case GG:                                                                                       \
    return (two ? est_launch<GG, 2> : est_launch<GG, 4>)(L, q, Hq, codes, scales, zeros, cand,  \
                                                         cand_stride, ncand, row0, lcap, cmax,  \
                                                         logits, stats, st, grid, pdl);
    TW_EST(1) TW_EST(2) TW_EST(4) TW_EST(8)
#undef TW_EST
  }
  return cudaErrorInvalidValue;
}

}  // namespace tw
