// Launchers of the packed token layout kernels (token_pack.cu).
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

namespace fpstok {

struct WsHeader;

// tok_offsets [B+1] = exclusive scan of v_b (valid[b], else min(N_b, K));
// dst [tok_offsets[B], D] <- the first v_b rows of src [B, K, D] per event;
// doc_id [tok_offsets[B]] <- the event of each packed row.
cudaError_t launch_pack_tokens(const float* src, int D, const int64_t* offsets, const int32_t* valid, int B, int K,
                               float* dst, int32_t* doc_id, int64_t* tok_offsets, WsHeader* hdr, cudaStream_t s);

// dst [B, K, D] <- packed rows of src [n_tok, D], zero padding.
cudaError_t launch_unpack_tokens(const float* src, int D, int64_t n_tok, const int64_t* tok_offsets, int B, int K,
                                 float* dst, WsHeader* hdr, cudaStream_t s);

}  // namespace fpstok
