// Launcher of the charge-weighted token summaries (token_summary.cu).
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

namespace fpstok {

struct WsHeader;

// Accumulator copies the summaries use for B events, K tokens, F features.
int token_summary_replicas(int B, int K, int F);

// wsum [B,K], wcoords [B,K,4], wfeats [B,K,F] from the Voronoi labels;
// acc: float64 [replicas, B, K, 5 + F] scratch (cleared here).
cudaError_t launch_token_summaries(const float* coords, const float* feats, int F, int charge_col,
                                   const int64_t* offsets, int B, int64_t P, int K, const int32_t* token_id,
                                   double* acc, float* wsum, float* wcoords, float* wfeats, WsHeader* hdr,
                                   cudaStream_t s);

}  // namespace fpstok
