// Logical -> physical row resolution for the single attention call.
//
// The attention kernel gathers rows through a list of physical row indices so
// that no page-table load sits in front of a gather.  In the fused decode step
// the selection kernel writes that list as a by-product; when a caller hands
// tw_sparse_decode its own token ids, this kernel builds the list first.  A
// token id outside [0, len) maps to kNoRow, which the attention kernel skips.
#include "tw_common.cuh"
#include "tw_kernels.h"

namespace tw {

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
