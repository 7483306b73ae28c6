// Launcher of the charge-weighted token summaries (token_summary.cu).
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

namespace fpstok {

struct WsHeader;

// CTAs (contiguous point ranges) the summaries use at most for K tokens and
// F features, and the bytes of their float64 partial sums (2 K (5 + F) each).
int token_summary_ctas(int K, int F);
size_t token_summary_partial_bytes(int K, int F);

// wsum [B,K], wcoords [B,K,4], wfeats [B,K,F] from the Voronoi labels;
// partial: token_summary_partial_bytes(K, F) of scratch (no clearing needed).
cudaError_t launch_token_summaries(const float* coords, const float* feats, int F, int charge_col,
                                   const int64_t* offsets, int B, int64_t P, int K, const int32_t* token_id,
                                   double* partial, float* wsum, float* wcoords, float* wfeats, WsHeader* hdr,
                                   cudaStream_t s);

}  // namespace fpstok
