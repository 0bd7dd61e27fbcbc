// Logical -> physical row resolution for the single-call entry points.
//
// The streaming kernels gather rows through lists of physical row indices so
// that no page-table load sits in front of a gather.  In the fused decode step
// the page selector and the top-p kernel write those lists as a by-product;
// when a caller hands the library its own candidate pages or token ids, these
// two kernels build the lists first.  A page id outside [0, max_pages) maps to
// row 0 (the estimate kernel masks such pages itself); a token id outside
// [0, len) maps to kNoRow, which the attention kernel skips.
#include "tw_common.cuh"
#include "tw_kernels.h"

namespace tw {

// row0[u][lp] = first physical row of candidate page cand[u][lp].
__global__ void k_resolve_pages(Layout L, const int32_t* __restrict__ cand, int cand_stride,
                                uint32_t* __restrict__ row0) {
  const int u = blockIdx.x;
  const int b = u / L.Hk, hk = u % L.Hk;
  const int n = min(cand_stride, L.max_pages);
  griddep_wait();
  for (int lp = blockIdx.y * blockDim.x + threadIdx.x; lp < n; lp += gridDim.y * blockDim.x) {
    const int page = cand[(int64_t)u * cand_stride + lp];
    row0[(int64_t)u * L.max_pages + lp] =
        (page >= 0 && page < L.max_pages) ? (uint32_t)L.page_row(b, hk, page) : 0u;
  }
  griddep_launch();
}

// rows[s][i] = physical K/V row of token idx[s][i] of set s, for i < count[s].
__global__ void k_resolve_rows(Layout L, int Hq, int G, int group_sets,
                               const int32_t* __restrict__ idx, int icap,
                               const int32_t* __restrict__ count, uint32_t* __restrict__ rows) {
  const int s = blockIdx.x;
  int b, hk;
  if (group_sets) {
    b = s / L.Hk;
    hk = s % L.Hk;
  } else {
    b = s / Hq;
    hk = (s % Hq) / G;
  }
  griddep_wait();
  const int n = max(0, min(count[s], icap));
  const int len = L.len(b);
  for (int i = blockIdx.y * blockDim.x + threadIdx.x; i < n; i += gridDim.y * blockDim.x) {
    const int tk = idx[(int64_t)s * icap + i];
    rows[(int64_t)s * icap + i] = (unsigned)tk < (unsigned)len ? (uint32_t)L.row(b, hk, tk) : kNoRow;
  }
  griddep_launch();
}

cudaError_t launch_resolve_pages(const Layout& L, const int32_t* cand, int cand_stride,
                                 uint32_t* row0, cudaStream_t st, bool pdl) {
  const int n = cand_stride < L.max_pages ? cand_stride : L.max_pages;
  const int bx = (n + 255) / 256 < 64 ? (n + 255) / 256 : 64;
  if (L.B * L.Hk == 0 || n <= 0) return cudaSuccess;
  return launch_k(k_resolve_pages, dim3(L.B * L.Hk, bx), dim3(256), 0, st, pdl, L, cand,
                  cand_stride, row0);
}

cudaError_t launch_resolve_rows(const Layout& L, int Hq, int group_sets, const int32_t* idx,
                                int icap, const int32_t* count, uint32_t* rows, cudaStream_t st,
                                bool pdl) {
  const int G = Hq / L.Hk;
  const int sets = group_sets ? L.B * L.Hk : L.B * Hq;
  const int bx = (icap + 255) / 256 < 64 ? (icap + 255) / 256 : 64;
  if (sets == 0) return cudaSuccess;
  return launch_k(k_resolve_rows, dim3(sets, bx), dim3(256), 0, st, pdl, L, Hq, G, group_sets,
                  idx, icap, count, rows);
}

}  // namespace tw
