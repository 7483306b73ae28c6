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
// Quotients are taken in float64 and rounded once to float32; the Voronoi
// path divides once per (token, feature) into a small table and then only
// gathers.
#include "common.cuh"
#include "internal.h"
#include "pool_backward.h"

namespace fpstok {

namespace {

constexpr int kBwdThreads = 256;
constexpr int kBwdPts = 4;                      // points per thread of the Voronoi gather
constexpr int kBwdTile = kBwdThreads * kBwdPts;  // points per block
constexpr int kKnnBwdThreads = 512;
constexpr int kFeatGroup = 8;  // features summed together per thread in the kNN scatter
constexpr int64_t kKnnBwdSmemBytes = 104 * 1024;  // shares and per-point row masks of the kNN scatter
constexpr int kBwdRowGroup = 16;  // rows of one event per warp in the kNN scatter's second phase

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

// quot[r, f] = grad_pooled[r, f] / counts[r] as the float64 quotient rounded
// once to float32, 0 for an empty row: the division happens once per
// (token, feature), and the per-point pass only gathers.  With hdr, thread 0
// first resets the call's status word; the gather, its programmatic
// dependent, may start at once and waits for this kernel before its checks.
__global__ void __launch_bounds__(256) k_pool_bwd_quot(const float* __restrict__ grad_pooled, int F, int64_t rows,
                                                       const int32_t* __restrict__ counts,
                                                       float* __restrict__ quot, WsHeader* hdr) {
  asm volatile("griddepcontrol.launch_dependents;");
  if (hdr && blockIdx.x == 0 && threadIdx.x == 0) {
    hdr->status = 0;
    hdr->detail = 0;
  }
  const int64_t n = rows * F;
  const int64_t stride = (int64_t)gridDim.x * blockDim.x;
  for (int64_t e = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; e < n; e += stride) {
    const int c = counts[e / F];
    quot[e] = c > 0 ? (float)((double)grad_pooled[e] / (double)c) : 0.f;
  }
}

// The gather: one block per tile of kBwdTile points, kBwdPts per thread with
// their loads issued together.  Per point its quotient row (b*K + token) goes
// to shared memory, then one thread per output element writes the flat
// [P, F] gradient with coalesced stores.  e / F is taken as __umulhi(e, fdiv)
// with fdiv = ceil(2^32 / F) (F >= 2): exact while e * (fdiv * F - 2^32) <
// 2^32, which holds for every e < kBwdTile * F <= 2^16.
__global__ void __launch_bounds__(kBwdThreads) k_pool_bwd_voronoi(
    const float* __restrict__ quot, int F, uint32_t fdiv, const int64_t* __restrict__ offsets, int B, int64_t P,
    int K, const int32_t* __restrict__ token_id, float* __restrict__ grad_feats, WsHeader* hdr) {
  __shared__ int s_row[kBwdTile];  // b*K + token, -1 when the point gets no gradient
  __shared__ int s_ev[2];
  const int64_t t0 = (int64_t)blockIdx.x * kBwdTile;
  const int n = (int)min((int64_t)kBwdTile, P - t0);
  int t[kBwdPts];
#pragma unroll
  for (int r = 0; r < kBwdPts; ++r) {  // issued before the event search
    const int p = threadIdx.x + r * kBwdThreads;
    t[r] = p < n ? token_id[t0 + p] : -1;
  }
  // the quotient table and the reset status word (a no-op outside a
  // programmatic dependent launch)
  asm volatile("griddepcontrol.wait;" ::: "memory");
  if (threadIdx.x < 2) s_ev[threadIdx.x] = event_of(offsets, 0, B - 1, threadIdx.x ? t0 + n - 1 : t0);
  __syncthreads();
  const int lo = s_ev[0], hi = max(s_ev[0], s_ev[1]);
#pragma unroll
  for (int r = 0; r < kBwdPts; ++r) {
    const int p = threadIdx.x + r * kBwdThreads;
    if (p < n) {
      const int64_t i = t0 + p;
      const int b = event_of(offsets, lo, hi, i);
      int row = -1;
      if (__ldg(offsets + b) > i || __ldg(offsets + b + 1) <= i) record_error(hdr, kDevBadOffsets);
      else if (t[r] >= K || t[r] < -1) record_error(hdr, kDevBadToken);
      else if (t[r] >= 0) row = b * K + t[r];
      s_row[p] = row;
    }
  }
  __syncthreads();
  const uint32_t ne = (uint32_t)(n * F);
  float* out = grad_feats + t0 * F;
#pragma unroll 8
  for (uint32_t e = threadIdx.x; e < ne; e += kBwdThreads) {
    const uint32_t q = F == 1 ? e : __umulhi(e, fdiv);
    const int rw = s_row[q];
    out[e] = rw >= 0 ? __ldg(quot + (int64_t)rw * F + (e - q * F)) : 0.f;
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

// Whether event b (n points from off) gets the per-event path: its row masks
// fit in shared memory and its points lie inside 0..P-1.
__device__ __forceinline__ bool knn_event_local(int64_t off, int64_t n, int cap_n, int64_t P) {
  return n > 0 && n <= cap_n && off >= 0 && off + n <= P;
}

// kNN scatter with the rows grouped by event.  Phase 1, one CTA per event:
// stage the K x F float64 shares grad_pooled / counts in shared memory, mark
// for each point of the event the rows that name it in a K-bit mask (shared
// atomicOr, independent of order), then let each point sum the shares of its
// marked rows in increasing row order -- the order a sequential loop over the
// rows takes -- and store the sums (plain stores: only this CTA writes these
// points of sums[]).  Entries that name a point outside their event, or a
// point already marked in the same row, are added to extra[] with float64
// atomics.  Phase 2, a warp per 16 rows of one event over the whole grid:
// the rows of events whose masks do not fit in shared memory add all their
// entries to extra[].
// The gradient is (float)(sums + extra); extra is 0 when every row names
// only its own event's points, once each, and the events fit, and then the
// result is exactly the sequential row-order sum.  Entry e of the event's
// K*k entries is row e / k = __umulhi(e, kdiv) with kdiv = ceil(2^32 / k)
// (k >= 2; exact for e < 2^15, k <= 128).  The sums run one thread per
// (point, group of up to kFeatGroup features) t: one scan of the mask feeds
// the group's independent sums; the point is t / G = __umulhi(t, gdiv),
// exact while t * (gdiv * G - 2^32) < 2^32, i.e. for every t < 2^26 (the
// shared buffer caps t near 2^21).
__global__ void __launch_bounds__(kKnnBwdThreads, 2) k_pool_bwd_knn_event(
    const float* __restrict__ grad_pooled, int F, const int64_t* __restrict__ offsets, int B, int K, int k,
    uint32_t kdiv, uint32_t gdiv, const int32_t* __restrict__ knn_idx, const int32_t* __restrict__ counts,
    int64_t P, int cap_n, double* __restrict__ sums, double* __restrict__ extra, WsHeader* hdr) {
  extern __shared__ double s_mem[];
  double* s_share = s_mem;                                                  // [K, F]; 0 rows for empty tokens
  uint32_t* s_bits = reinterpret_cast<uint32_t*>(s_share + (size_t)K * F);  // [cap_n, W] row masks
  const int W = (K + 31) >> 5;
  const int ke = K * k;
  const int G = (F + kFeatGroup - 1) / kFeatGroup;
  for (int b = blockIdx.x; b < B; b += gridDim.x) {
    const int64_t off = offsets[b];
    const int64_t n = offsets[b + 1] - off;
    if (!knn_event_local(off, n, cap_n, P)) continue;  // block-uniform; phase 2 takes it
    const float* g = grad_pooled + (int64_t)b * K * F;
    for (int e = threadIdx.x; e < K * F; e += blockDim.x) {
      const int c = counts[(int64_t)b * K + e / F];
      s_share[e] = c > 0 ? (double)__ldg(g + e) / (double)c : 0.0;
    }
    for (int i = threadIdx.x; i < (int)n * W; i += blockDim.x) s_bits[i] = 0u;
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
      const int64_t li = v - off;
      if (li >= 0 && li < n) {
        const uint32_t bit = 1u << (j & 31);
        if (!(atomicOr(s_bits + li * W + (j >> 5), bit) & bit)) continue;  // marked: summed below
      }
      const double* sh = s_share + j * F;  // outside the event, or a repeat within the row
      double* dst = extra + (int64_t)v * F;
      for (int f = 0; f < F; ++f)
        if (sh[f] != 0.0) atomicAdd(dst + f, sh[f]);
    }
    __syncthreads();
    for (int t = threadIdx.x; t < (int)n * G; t += blockDim.x) {
      const int i = G == 1 ? t : (int)__umulhi((uint32_t)t, gdiv);
      const int f0 = (t - i * G) * kFeatGroup;
      const int nf = min(kFeatGroup, F - f0);
      const uint32_t* bits = s_bits + (int64_t)i * W;
      double sum[kFeatGroup];
#pragma unroll
      for (int q = 0; q < kFeatGroup; ++q) sum[q] = 0.0;
      for (int w = 0; w < W; ++w) {
        uint32_t m = bits[w];
        while (m) {
          const int j = (w << 5) + __ffs(m) - 1;
          m &= m - 1;
          const double* sh = s_share + j * F + f0;
#pragma unroll
          for (int q = 0; q < kFeatGroup; ++q)
            if (q < nf) sum[q] += sh[q];
        }
      }
      double* dst = sums + (off + i) * F + f0;
#pragma unroll
      for (int q = 0; q < kFeatGroup; ++q)
        if (q < nf) dst[q] = sum[q];
    }
    __syncthreads();
  }
  // phase 2: rows of the events phase 1 skipped, a warp per group of
  // kBwdRowGroup rows of one event (one locality check per group)
  const int lane = threadIdx.x & 31;
  const int64_t gw = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int64_t nw = ((int64_t)gridDim.x * blockDim.x) >> 5;
  const int groups = (K + kBwdRowGroup - 1) / kBwdRowGroup;
  for (int64_t it = gw; it < (int64_t)B * groups; it += nw) {
    const int b = (int)(it / groups);
    const int j0 = (int)(it - (int64_t)b * groups) * kBwdRowGroup;
    const int64_t off = offsets[b];
    if (knn_event_local(off, offsets[b + 1] - off, cap_n, P)) continue;  // warp-uniform
    for (int j = j0; j < min(K, j0 + kBwdRowGroup); ++j) {
      const int64_t r = (int64_t)b * K + j;
      const int c = counts[r];
      if (c <= 0) continue;
      const float* g = grad_pooled + r * F;
      for (int e = lane; e < k; e += 32) {
        const int v = knn_idx[r * k + e];
        if (v >= P) record_error(hdr, kDevBadToken);
        if (v < 0 || v >= P) continue;
        double* dst = extra + (int64_t)v * F;
        for (int f = 0; f < F; ++f) {
          const double sh = (double)__ldg(g + f) / (double)c;
          if (sh != 0.0) atomicAdd(dst + f, sh);
        }
      }
    }
  }
}

// Rounds the float64 accumulators to the float32 gradient: out = (float)(a + b),
// b optional.
__global__ void __launch_bounds__(256) k_pool_bwd_round(const double* __restrict__ a, const double* __restrict__ b,
                                                        int64_t n, float* __restrict__ out) {
  const int64_t stride = (int64_t)gridDim.x * blockDim.x;
  for (int64_t e = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; e < n; e += stride)
    out[e] = (float)(b ? a[e] + b[e] : a[e]);
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
                                    int K, const int32_t* token_id, const int32_t* counts, float* quot,
                                    float* grad_feats, WsHeader* hdr, cudaStream_t s) {
  if (P == 0) return cudaSuccess;
  const int64_t rows = (int64_t)B * K;
  count_launch();
  k_pool_bwd_quot<<<grid_for(rows * F, 256, 8), 256, 0, s>>>(grad_pooled, F, rows, counts, quot, hdr);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  const uint32_t fdiv = F > 1 ? (uint32_t)((((uint64_t)1 << 32) + F - 1) / F) : 0u;
  const int64_t blocks = (P + kBwdTile - 1) / kBwdTile;
  count_launch();
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)blocks);
  cfg.blockDim = dim3(kBwdThreads);
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, k_pool_bwd_voronoi, (const float*)quot, F, fdiv, offsets, B, P, K, token_id,
                            grad_feats, hdr);
}

cudaError_t launch_pool_bwd_knn(const float* grad_pooled, int F, const int64_t* offsets, int B, int K, int k,
                                const int32_t* knn_idx, const int32_t* counts, int64_t P, double* acc,
                                float* grad_feats, WsHeader* hdr, cudaStream_t s) {
  if (P == 0) return cudaSuccess;
  const int64_t rows = (int64_t)B * K;
  const int64_t share_bytes = (int64_t)K * F * sizeof(double);
  const bool per_event = rows > 0 && offsets && share_bytes <= kKnnBwdSmemBytes / 2;
  double* extra = per_event ? acc + (size_t)P * F : nullptr;
  cudaError_t e = cudaMemsetAsync(acc, 0, (size_t)P * F * sizeof(double) * (per_event ? 2 : 1), s);
  if (e != cudaSuccess) return e;
  if (per_event) {
    // shared memory: the shares, then a K-bit row mask per point of the event
    const int64_t mask_bytes = (int64_t)((K + 31) / 32) * sizeof(uint32_t);
    int64_t cap = (kKnnBwdSmemBytes - share_bytes) / mask_bytes;
    if (cap > P) cap = P;
    const size_t smem = (size_t)(share_bytes + cap * mask_bytes);
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
    const int G = (F + kFeatGroup - 1) / kFeatGroup;
    const uint32_t gdiv = G > 1 ? (uint32_t)((((uint64_t)1 << 32) + G - 1) / G) : 0u;
    count_launch();
    k_pool_bwd_knn_event<<<grid_for(B, 1, 2), kKnnBwdThreads, smem, s>>>(
        grad_pooled, F, offsets, B, K, k, kdiv, gdiv, knn_idx, counts, P, (int)cap, acc, extra, hdr);
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
  k_pool_bwd_round<<<grid_for((int64_t)P * F, 256, 8), 256, 0, s>>>(acc, extra, (int64_t)P * F, grad_feats);
  return cudaGetLastError();
}

}  // namespace fpstok
