// Packed token layout for block-diagonal attention (graphnet PR #923, "What is
// added": models/utils.py pack / unpack / build_block_mask; review thread on
// the block mask: doc_id is the event index of every packed token).
//
// Event b has v_b tokens (valid[b], else min(N_b, K)).  Its first v_b padded
// rows src[b, 0:v_b, :] are one contiguous span, and so are its packed rows
// dst[tok_offsets[b] : tok_offsets[b+1], :], so after one scan of the v_b the
// copy is a segmented memcpy: one block per event, coalesced on both sides.
#include "../../include/fpstok.h"
#include "common.cuh"
#include "internal.h"
#include "token_pack.h"

namespace fpstok {

namespace {

constexpr int kScanThreads = 1024;
constexpr int kScanPer = 4;  // consecutive events per scan thread
constexpr int kCopyThreads = 128;   // unpack: one block per event
constexpr int kPackThreads = 256;   // pack: one warp per event

// Tokens of event b: valid[b] (clamped to 0..K, a value outside is recorded),
// else min(N_b, K) from the point offsets.
__device__ __forceinline__ int64_t tokens_of(const int64_t* __restrict__ offsets, const int32_t* __restrict__ valid,
                                             int b, int K, WsHeader* hdr) {
  if (valid) {
    const int64_t v = valid[b];
    if (v < 0 || v > K) {
      record_error(hdr, kDevBadToken);
      return v < 0 ? 0 : K;
    }
    return v;
  }
  const int64_t n = offsets[b + 1] - offsets[b];
  if (n < 0) record_error(hdr, kDevBadOffsets);
  return n < 0 ? 0 : (n < K ? n : K);
}

// tok_offsets[0] = 0, tok_offsets[b+1] = tok_offsets[b] + v_b, by one CTA in
// tiles of kScanThreads * kScanPer events (kScanPer consecutive events per
// thread, so the small-event batches take one tile).  Resets the call's
// status word first (before the barrier that precedes every check).
__global__ void __launch_bounds__(kScanThreads) k_pack_scan(const int64_t* __restrict__ offsets,
                                                            const int32_t* __restrict__ valid, int B, int K,
                                                            int64_t* __restrict__ tok_offsets, WsHeader* hdr) {
  // the copy kernel, launched as a programmatic dependent, may start now: it
  // reads its source rows and then waits for this kernel's offsets
  asm volatile("griddepcontrol.launch_dependents;");
  __shared__ int64_t s_warp[kScanThreads / 32];
  __shared__ int64_t s_carry;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  if (threadIdx.x == 0) {
    s_carry = 0;
    tok_offsets[0] = 0;
    hdr->status = 0;  // this call's status word (the copy kernel records nothing)
    hdr->detail = 0;
  }
  __syncthreads();
  for (int64_t t0 = 0; t0 < B; t0 += (int64_t)kScanThreads * kScanPer) {
    const int64_t b0 = t0 + (int64_t)threadIdx.x * kScanPer;
    int64_t v[kScanPer];
    int64_t sum = 0;
#pragma unroll
    for (int q = 0; q < kScanPer; ++q) {
      v[q] = b0 + q < B ? tokens_of(offsets, valid, (int)(b0 + q), K, hdr) : 0;
      sum += v[q];
    }
    int64_t x = sum;  // inclusive scan of the thread sums: warp, then warp totals
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int64_t y = __shfl_up_sync(0xffffffffu, x, o);
      if (lane >= o) x += y;
    }
    if (lane == 31) s_warp[warp] = x;
    __syncthreads();
    if (warp == 0) {
      int64_t w = s_warp[lane];
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int64_t y = __shfl_up_sync(0xffffffffu, w, o);
        if (lane >= o) w += y;
      }
      s_warp[lane] = w;  // inclusive over warps
    }
    __syncthreads();
    int64_t run = s_carry + (warp ? s_warp[warp - 1] : 0) + x - sum;
#pragma unroll
    for (int q = 0; q < kScanPer; ++q) {
      run += v[q];
      if (b0 + q < B) tok_offsets[b0 + q + 1] = run;
    }
    __syncthreads();
    if (threadIdx.x == kScanThreads - 1) s_carry = run;
    __syncthreads();
  }
}

// One warp per event (kPackThreads / 32 events per block): dst rows
// tok_offsets[b] .. + v_b <- src[b, 0:v_b, :], doc_id over the same rows <-
// b.  v_b comes from the inputs again, so only the destination base waits on
// the scan's result: launched as the scan's programmatic dependent, each lane
// loads its first kPre elements before it waits (a no-op wait otherwise),
// and with a few blocks per SM every event's loads are in flight at once.
constexpr int kPre = 24;
__global__ void __launch_bounds__(kPackThreads) k_pack_copy(const float* __restrict__ src, int D, int K, int B,
                                                            const int64_t* __restrict__ offsets,
                                                            const int32_t* __restrict__ valid,
                                                            const int64_t* __restrict__ tok_offsets,
                                                            float* __restrict__ dst, int32_t* __restrict__ doc_id) {
  const int lane = threadIdx.x & 31;
  const int b = blockIdx.x * (kPackThreads / 32) + (threadIdx.x >> 5);
  int v = 0;
  if (b < B) {
    if (valid) {
      const int32_t c = valid[b];
      v = c < 0 ? 0 : (c > K ? K : c);
    } else {
      const int64_t n = offsets[b + 1] - offsets[b];
      v = (int)(n < 0 ? 0 : (n < K ? n : K));
    }
  }
  const float* s = src + (int64_t)b * K * D;
  const int n = v * D;
  float pre[kPre];
#pragma unroll
  for (int q = 0; q < kPre; ++q) {
    const int e = lane + q * 32;
    pre[q] = e < n ? s[e] : 0.f;
  }
  asm volatile("griddepcontrol.wait;" ::: "memory");
  if (b >= B) return;
  const int64_t base = tok_offsets[b];
  float* d = dst + base * D;
#pragma unroll
  for (int q = 0; q < kPre; ++q) {
    const int e = lane + q * 32;
    if (e < n) d[e] = pre[q];
  }
  for (int e = lane + kPre * 32; e < n; e += 32) d[e] = s[e];
  for (int j = lane; j < v; j += 32) doc_id[base + j] = b;
}

// One block per event: dst[b, 0:v_b, :] <- packed rows, dst[b, v_b:K, :] <- 0.
__global__ void __launch_bounds__(kCopyThreads) k_unpack_copy(const float* __restrict__ src, int D, int64_t n_tok,
                                                              int K, const int64_t* __restrict__ tok_offsets,
                                                              float* __restrict__ dst, WsHeader* hdr) {
  const int b = blockIdx.x;
  const int64_t base = tok_offsets[b];
  int64_t v = tok_offsets[b + 1] - base;
  if (base < 0 || v < 0 || v > K || base + v > n_tok) {
    if (threadIdx.x == 0) record_error(hdr, kDevBadOffsets);
    v = 0;  // the event's rows become padding
  }
  const float* s = src + base * D;
  float* d = dst + (int64_t)b * K * D;
  const int nv = (int)v * D, n = K * D;
  for (int e = threadIdx.x; e < n; e += kCopyThreads) d[e] = e < nv ? s[e] : 0.f;
}

}  // namespace

cudaError_t launch_pack_tokens(const float* src, int D, const int64_t* offsets, const int32_t* valid, int B, int K,
                               float* dst, int32_t* doc_id, int64_t* tok_offsets, WsHeader* hdr, cudaStream_t s) {
  count_launch();
  k_pack_scan<<<1, kScanThreads, 0, s>>>(offsets, valid, B, K, tok_offsets, hdr);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess || B == 0) return e;
  count_launch();
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)((B + kPackThreads / 32 - 1) / (kPackThreads / 32)));
  cfg.blockDim = dim3(kPackThreads);
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, k_pack_copy, src, D, K, B, offsets, valid, (const int64_t*)tok_offsets, dst,
                            doc_id);
}

cudaError_t launch_unpack_tokens(const float* src, int D, int64_t n_tok, const int64_t* tok_offsets, int B, int K,
                                 float* dst, WsHeader* hdr, cudaStream_t s) {
  if (B == 0) return cudaSuccess;
  count_launch();
  k_unpack_copy<<<B, kCopyThreads, 0, s>>>(src, D, n_tok, K, tok_offsets, dst, hdr);
  return cudaGetLastError();
}

}  // namespace fpstok
