// Launch interface of the token-level label-channel base selector (label.cu),
// used by capi_label.cu.
#pragma once

#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "tw_common.cuh"

namespace tw {

constexpr int kMaxLabelChannels = 32;
constexpr int kMaxLabelGroup = 8;

// labels[row][j] = K[row][channels[h][j]] for every valid token row.
cudaError_t launch_label_cache(const Layout& L, const __half* K, const int32_t* channels, int r,
                               __half* labels, cudaStream_t st, int num_sms);
// scores[u][t] for unit u = b * Hk + h and t < len(b).
cudaError_t launch_label_scores(const Layout& L, const __half* q, int Hq, const __half* labels,
                                const int32_t* channels, int r, float* scores, cudaStream_t st);
// The min(budget, len(b)) best-scored tokens of each unit, ascending.
cudaError_t launch_token_topk(const Layout& L, const float* scores, int budget, int32_t* cand,
                              int cand_stride, int32_t* ncand, cudaStream_t st);
// Quantised key rows of each unit's candidate tokens into a contiguous cache
// of B * Hk units x cand_stride rows.
cudaError_t launch_gather_keys(const Layout& L, const int32_t* cand, int cand_stride,
                               const int32_t* ncand, const uint8_t* codes, const __half* scales,
                               const __half* zeros, uint8_t* vcodes, __half* vscales,
                               __half* vzeros, cudaStream_t st, int num_sms);
// idx[s][i] = cand[unit(s)][idx[s][i]] for i < count[s].
cudaError_t launch_map_tokens(int nsets, int G, int group_sets, const int32_t* cand,
                              int cand_stride, int32_t* idx, int icap, const int32_t* count,
                              cudaStream_t st);

}  // namespace tw
