// Backward of the per-token mean-pool: the gradient of the pooled rows with
// respect to the point features (graphnet PR #923, "What is added": the
// tokenizer runs inside the training step and its tests check gradients).
//
// The pool is linear.  Point i of token (b, j) enters pooled[b,j,:] with
// weight 1/counts[b,j], so:
//   Voronoi: grad_feats[i,:] = grad_pooled[b, token_id[i], :] / counts[b, token_id[i]]
//            -- a gather, one write per feature, no atomics;
//   kNN:     grad_feats[i,:] = sum over the rows (b, j) that gathered i of
//            grad_pooled[b,j,:] / counts[b,j] -- a scatter, accumulated in
//            float64 with red.global.add.f64 and rounded once.
// Quotients are taken in float64 and rounded once to float32 (for the
// Voronoi gather that equals a correctly rounded float32 division, which is
// what it computes).
#include "common.cuh"
#include "internal.h"
#include "pool_backward.h"

namespace fpstok {

namespace {

constexpr int kBwdThreads = 256;
constexpr int kBwdPts = 4;                      // points per thread of the Voronoi gather
constexpr int kBwdTile = kBwdThreads * kBwdPts;  // points per block
constexpr int kKnnBwdThreads = 512;
constexpr int64_t kKnnBwdSmemBytes = 104 * 1024;  // shares + per-event float64 sums of the kNN scatter

// Largest b in [lo, hi] with offsets[b] <= i (offsets non-decreasing), i.e.
// the event holding point i when i < offsets[hi + 1].
__device__ __forceinline__ int event_of(const int64_t* __restrict__ offsets, int lo, int hi, int64_t i) {
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (__ldg(offsets + mid) <= i) lo = mid;
    else hi = mid - 1;
  }
  return lo;
}

// g / c as the float64 quotient rounded once to float32.  For c < 2^24 (exact
// in float32) that is the correctly rounded float32 division: rounding the
// 53-bit quotient to 24 bits cannot differ from rounding the exact quotient
// (double rounding is harmless for division when 53 >= 2 * 24 + 2).
__device__ __forceinline__ float share_f32(float g, int c) {
  return c < (1 << 24) ? __fdiv_rn(g, (float)c) : (float)((double)g / (double)c);
}

// The gather: one block per tile of kBwdTile points, kBwdPts per thread with
// their loads issued together.  Per point its gradient row (b*K + token) and
// count go to shared memory, then one thread per output element writes the
// flat [P, F] gradient with coalesced stores.  e / F is taken as
// __umulhi(e, fdiv) with fdiv = ceil(2^32 / F) (F >= 2), exact for
// e < kBwdTile * F <= 2^16: the error e * (fdiv * F - 2^32) / 2^32 stays below 1/F.
__global__ void __launch_bounds__(kBwdThreads) k_pool_bwd_voronoi(
    const float* __restrict__ grad_pooled, int F, uint32_t fdiv, const int64_t* __restrict__ offsets, int B,
    int64_t P, int K, const int32_t* __restrict__ token_id, const int32_t* __restrict__ counts,
    float* __restrict__ grad_feats, WsHeader* hdr) {
  __shared__ int s_row[kBwdTile];  // b*K + token, -1 when the point gets no gradient
  __shared__ int s_cnt[kBwdTile];
  __shared__ int s_ev[2];
  const int64_t t0 = (int64_t)blockIdx.x * kBwdTile;
  const int n = (int)min((int64_t)kBwdTile, P - t0);
  int t[kBwdPts];
#pragma unroll
  for (int r = 0; r < kBwdPts; ++r) {  // issued before the event search
    const int p = threadIdx.x + r * kBwdThreads;
    t[r] = p < n ? token_id[t0 + p] : -1;
  }
  if (threadIdx.x < 2) s_ev[threadIdx.x] = event_of(offsets, 0, B - 1, threadIdx.x ? t0 + n - 1 : t0);
  __syncthreads();
  const int lo = s_ev[0], hi = max(s_ev[0], s_ev[1]);
  int row[kBwdPts], b[kBwdPts];
#pragma unroll
  for (int r = 0; r < kBwdPts; ++r) {
    const int p = threadIdx.x + r * kBwdThreads;
    const int64_t i = t0 + p;
    b[r] = p < n ? event_of(offsets, lo, hi, i) : lo;
    row[r] = -1;
    if (p < n) {
      if (__ldg(offsets + b[r]) > i || __ldg(offsets + b[r] + 1) <= i) record_error(hdr, kDevBadOffsets);
      else if (t[r] >= K || t[r] < -1) record_error(hdr, kDevBadToken);
      else if (t[r] >= 0) row[r] = b[r] * K + t[r];
    }
  }
#pragma unroll
  for (int r = 0; r < kBwdPts; ++r) {
    const int p = threadIdx.x + r * kBwdThreads;
    const int c = row[r] >= 0 ? counts[row[r]] : 0;
    if (p < n) {
      s_row[p] = c > 0 ? row[r] : -1;
      s_cnt[p] = c;
    }
  }
  __syncthreads();
  const uint32_t ne = (uint32_t)(n * F);
  float* out = grad_feats + t0 * F;
#pragma unroll 8
  for (uint32_t e = threadIdx.x; e < ne; e += kBwdThreads) {
    const uint32_t q = F == 1 ? e : __umulhi(e, fdiv);
    const int rw = s_row[q];
    out[e] = rw >= 0 ? share_f32(__ldg(grad_pooled + (int64_t)rw * F + (e - q * F)), s_cnt[q]) : 0.f;
  }
}

// kNN scatter: a warp per row (b, j); lane e holds entries e, e+32, ...
template <int KPL>
__global__ void __launch_bounds__(256) k_pool_bwd_knn(const float* __restrict__ grad_pooled, int F, int64_t rows,
                                                      int k, const int32_t* __restrict__ knn_idx,
                                                      const int32_t* __restrict__ counts, int64_t P,
                                                      double* __restrict__ acc, WsHeader* hdr) {
  const int lane = threadIdx.x & 31;
  const int64_t gw = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int64_t nw = ((int64_t)gridDim.x * blockDim.x) >> 5;
  for (int64_t r = gw; r < rows; r += nw) {
    const int c = counts[r];
    if (c <= 0) continue;  // warp-uniform
    int idx[KPL];
#pragma unroll
    for (int q = 0; q < KPL; ++q) {
      const int e = q * 32 + lane;
      int v = e < k ? knn_idx[r * k + e] : -1;
      if (v >= P) {
        record_error(hdr, kDevBadToken);
        v = -1;
      }
      idx[q] = v;
    }
    const float* g = grad_pooled + r * F;
    for (int f = 0; f < F; ++f) {
      const double share = (double)__ldg(g + f) / (double)c;
#pragma unroll
      for (int q = 0; q < KPL; ++q)
        if (idx[q] >= 0) atomicAdd(acc + (int64_t)idx[q] * F + f, share);
    }
  }
}

// kNN scatter with the rows grouped by event: one CTA takes all K rows of
// event b.  It first stages the K x F float64 shares grad_pooled / counts in
// shared memory (all loads issued together), then runs one thread per row
// entry.  Shares for points inside the event (when its n x F float64 sums fit
// in shared memory) are summed there and added to the global accumulators
// with one reduction per (point, feature) touched, instead of one per (row
// entry, feature); entries outside the event, and events too large for the
// shared buffer, go straight to the global accumulators.  Entry e of the
// event's K*k entries is row e / k, taken as __umulhi(e, kdiv) with
// kdiv = ceil(2^32 / k) (k >= 2; exact for e < 2^15, k <= 128).
__global__ void __launch_bounds__(kKnnBwdThreads, 2) k_pool_bwd_knn_event(
    const float* __restrict__ grad_pooled, int F, const int64_t* __restrict__ offsets, int B, int K, int k,
    uint32_t kdiv, const int32_t* __restrict__ knn_idx, const int32_t* __restrict__ counts, int64_t P,
    int smem_points, double* __restrict__ acc, WsHeader* hdr) {
  extern __shared__ double s_mem[];
  double* s_share = s_mem;                    // [K, F]; 0 rows for empty tokens
  double* s_acc = s_mem + (size_t)K * F;      // [smem_points, F]
  const int ke = K * k;
  for (int b = blockIdx.x; b < B; b += gridDim.x) {
    const int64_t off = offsets[b];
    const int64_t n = offsets[b + 1] - off;
    const bool local = n > 0 && n <= smem_points && off >= 0 && off + n <= P;  // block-uniform
    const float* g = grad_pooled + (int64_t)b * K * F;
    for (int e = threadIdx.x; e < K * F; e += blockDim.x) {
      const int c = counts[(int64_t)b * K + e / F];
      s_share[e] = c > 0 ? (double)__ldg(g + e) / (double)c : 0.0;
    }
    if (local)
      for (int e = threadIdx.x; e < (int)n * F; e += blockDim.x) s_acc[e] = 0.0;
    __syncthreads();
    const int32_t* rows = knn_idx + (int64_t)b * ke;
#pragma unroll 4
    for (int e = threadIdx.x; e < ke; e += blockDim.x) {
      int v = rows[e];
      if (v >= P) {
        record_error(hdr, kDevBadToken);
        v = -1;
      }
      if (v < 0) continue;
      const int j = k == 1 ? e : (int)__umulhi((uint32_t)e, kdiv);
      const double* sh = s_share + j * F;
      const int64_t li = v - off;
      if (local && li >= 0 && li < n) {
        double* dst = s_acc + li * F;
        for (int f = 0; f < F; ++f)
          if (sh[f] != 0.0) atomicAdd(dst + f, sh[f]);
      } else {
        double* dst = acc + (int64_t)v * F;
        for (int f = 0; f < F; ++f)
          if (sh[f] != 0.0) atomicAdd(dst + f, sh[f]);
      }
    }
    __syncthreads();
    if (local) {
      double* dst = acc + off * F;
      for (int e = threadIdx.x; e < (int)n * F; e += blockDim.x) {
        const double v = s_acc[e];
        if (v != 0.0) atomicAdd(dst + e, v);  // +0 needs no add: the accumulators start at +0
      }
    }
    __syncthreads();
  }
}

// Rounds the float64 accumulators to the float32 gradient.
__global__ void __launch_bounds__(256) k_pool_bwd_round(const double* __restrict__ acc, int64_t n,
                                                        float* __restrict__ out) {
  const int64_t stride = (int64_t)gridDim.x * blockDim.x;
  for (int64_t e = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; e < n; e += stride) out[e] = (float)acc[e];
}

int grid_for(int64_t work_items, int per_block, int blocks_per_sm) {
  const DeviceInfo& di = device_info();
  int64_t g = (work_items + per_block - 1) / per_block;
  const int64_t cap = (int64_t)di.sm_count * blocks_per_sm;
  if (g > cap) g = cap;
  return (int)(g < 1 ? 1 : g);
}

}  // namespace

cudaError_t launch_pool_bwd_voronoi(const float* grad_pooled, int F, const int64_t* offsets, int B, int64_t P,
                                    int K, const int32_t* token_id, const int32_t* counts, float* grad_feats,
                                    WsHeader* hdr, cudaStream_t s) {
  if (P == 0) return cudaSuccess;
  const uint32_t fdiv = F > 1 ? (uint32_t)((((uint64_t)1 << 32) + F - 1) / F) : 0u;
  const int64_t blocks = (P + kBwdTile - 1) / kBwdTile;
  count_launch();
  k_pool_bwd_voronoi<<<(unsigned)blocks, kBwdThreads, 0, s>>>(grad_pooled, F, fdiv, offsets, B, P, K, token_id,
                                                              counts, grad_feats, hdr);
  return cudaGetLastError();
}

cudaError_t launch_pool_bwd_knn(const float* grad_pooled, int F, const int64_t* offsets, int B, int K, int k,
                                const int32_t* knn_idx, const int32_t* counts, int64_t P, double* acc,
                                float* grad_feats, WsHeader* hdr, cudaStream_t s) {
  if (P == 0) return cudaSuccess;
  cudaError_t e = cudaMemsetAsync(acc, 0, (size_t)P * F * sizeof(double), s);
  if (e != cudaSuccess) return e;
  const int64_t rows = (int64_t)B * K;
  const int64_t share_bytes = (int64_t)K * F * sizeof(double);
  if (rows > 0 && offsets && share_bytes <= kKnnBwdSmemBytes) {
    int64_t pts = (kKnnBwdSmemBytes - share_bytes) / ((int64_t)F * sizeof(double));
    if (pts > P) pts = P;
    const size_t smem = (size_t)(share_bytes + pts * F * (int64_t)sizeof(double));
    static bool attr_set[64] = {};
    int dev = 0;
    cudaGetDevice(&dev);
    if (dev >= 0 && dev < 64 && !attr_set[dev]) {
      if ((e = cudaFuncSetAttribute(k_pool_bwd_knn_event, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                    (int)kKnnBwdSmemBytes)))
        return e;
      attr_set[dev] = true;
    }
    const uint32_t kdiv = k > 1 ? (uint32_t)((((uint64_t)1 << 32) + k - 1) / k) : 0u;
    count_launch();
    k_pool_bwd_knn_event<<<grid_for(B, 1, 2), kKnnBwdThreads, smem, s>>>(grad_pooled, F, offsets, B, K, k, kdiv,
                                                                         knn_idx, counts, P, (int)pts, acc, hdr);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
  } else if (rows > 0) {
    const int g = grid_for(rows, 8, 16);
    count_launch();
    if (k <= 32)
      k_pool_bwd_knn<1><<<g, 256, 0, s>>>(grad_pooled, F, rows, k, knn_idx, counts, P, acc, hdr);
    else if (k <= 64)
      k_pool_bwd_knn<2><<<g, 256, 0, s>>>(grad_pooled, F, rows, k, knn_idx, counts, P, acc, hdr);
    else
      k_pool_bwd_knn<4><<<g, 256, 0, s>>>(grad_pooled, F, rows, k, knn_idx, counts, P, acc, hdr);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
  }
  count_launch();
  k_pool_bwd_round<<<grid_for((int64_t)P * F, 256, 8), 256, 0, s>>>(acc, (int64_t)P * F, grad_feats);
  return cudaGetLastError();
}

}  // namespace fpstok
