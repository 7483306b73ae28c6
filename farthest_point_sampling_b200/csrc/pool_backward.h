// Launchers of the mean-pool backward kernels (pool_backward.cu).
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

namespace fpstok {

struct WsHeader;

// grad_feats[i,:] = grad_pooled[b, token_id[i], :] / counts[b, token_id[i]]
// (0 for token -1 or count 0).  quot: float32 [B, K, F] scratch.  Records
// kDevBadOffsets / kDevBadToken in hdr.
cudaError_t launch_pool_bwd_voronoi(const float* grad_pooled, int F, const int64_t* offsets, int B, int64_t P,
                                    int K, const int32_t* token_id, const int32_t* counts, float* quot,
                                    float* grad_feats, WsHeader* hdr, cudaStream_t s);

// grad_feats[i,:] = sum over rows r gathering i of grad_pooled[r,:] / counts[r];
// acc: float64 [2, P, F] scratch (cleared here).  offsets (may be null) lets
// the rows of each event be summed in shared memory first.
cudaError_t launch_pool_bwd_knn(const float* grad_pooled, int F, const int64_t* offsets, int B, int K, int k,
                                const int32_t* knn_idx, const int32_t* counts, int64_t P, double* acc,
                                float* grad_feats, WsHeader* hdr, cudaStream_t s);

}  // namespace fpstok
