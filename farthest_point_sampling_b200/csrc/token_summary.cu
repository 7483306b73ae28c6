// Charge-weighted token summaries (graphnet PR #923, review thread on the
// no-charge case: the tokenizer uses the charge for weighting and for token
// summaries, unit charge without a charge column).  Per Voronoi token j of
// event b, with q = feats[:, charge_col] (or 1):
//   wsum = sum q,  wcoords = sum q * coords / wsum,  wfeats = sum q * feats / wsum,
// float64 sums, means 0 for an empty cell or wsum <= 0, each output rounded
// once to float32.
//
// k_token_sums takes the point array in tiles of kSumTile points, staging the
// tile's coordinate and feature rows in shared memory (coalesced) when they
// fit.  A tile that spans few events sorts its points by (event, token) with
// a counting sort in shared memory and adds each non-empty (token, value) sum
// to the float64 accumulators once; a tile spanning more events than its bucket
// table holds (events of a few points each) adds point by point.
// k_token_finalize sums the replicas in order, divides and rounds.
#include "../../include/fpstok.h"
#include "common.cuh"
#include "internal.h"
#include "token_summary.h"

namespace fpstok {

namespace {

constexpr int kSumThreads = 256;
constexpr int kSumPts = 4;
constexpr int kSumTile = kSumThreads * kSumPts;
constexpr int kMaxBuckets = 2048;  // (events in the tile) * K of the counting sort
// Tiles add into up to kSumMaxReplicas copies of the accumulators (tile i into
// copy i mod R), as many as fit in kSumReplicaBudget bytes: the tiles of a large
// event would otherwise all serialise on the same few accumulator lines.
constexpr int kSumMaxReplicas = 16;
constexpr int64_t kSumReplicaBudget = 32ll << 20;
constexpr int kSumStageBytes = 160 * 1024;  // dynamic shared memory for the staged tile rows

__device__ __forceinline__ int sum_event_of(const int64_t* __restrict__ offsets, int lo, int hi, int64_t i) {
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (__ldg(offsets + mid) <= i) lo = mid;
    else hi = mid - 1;
  }
  return lo;
}

// Value v of point i: q, q * coords[i, v-1] (v = 1..4), q * feats[i, v-5].
__device__ __forceinline__ double summary_value(const float* __restrict__ coords, const float* __restrict__ feats,
                                                int F, int charge_col, int64_t i, int v) {
  const double q = charge_col >= 0 ? (double)__ldg(feats + i * F + charge_col) : 1.0;
  if (v == 0) return q;
  if (v < 5) return q * (double)__ldg(coords + 4 * i + (v - 1));
  return q * (double)__ldg(feats + i * F + (v - 5));
}

// Value v of tile point p (point i): q, q * coords[i, v-1] (v = 1..4),
// q * feats[i, v-5], read from the tile's rows staged in shared memory (sc:
// [n, 4], sf: [n, F]) when staged, else from global memory.
__device__ __forceinline__ double tile_value(const float* sc, const float* sf, bool staged,
                                             const float* __restrict__ coords, const float* __restrict__ feats,
                                             int F, int charge_col, int64_t t0, int p, int v) {
  if (!staged) return summary_value(coords, feats, F, charge_col, t0 + p, v);
  const double q = charge_col >= 0 ? (double)sf[p * F + charge_col] : 1.0;
  if (v == 0) return q;
  if (v < 5) return q * (double)sc[p * 4 + (v - 1)];
  return q * (double)sf[p * F + (v - 5)];
}

__global__ void __launch_bounds__(kSumThreads) k_token_sums(const float* __restrict__ coords,
                                                            const float* __restrict__ feats, int F, int charge_col,
                                                            const int64_t* __restrict__ offsets, int B, int64_t P,
                                                            int K, const int32_t* __restrict__ token_id, int reps,
                                                            int staged, double* __restrict__ acc, WsHeader* hdr) {
  extern __shared__ float s_rows[];  // staged tile rows: coords [kSumTile, 4], then feats [kSumTile, F]
  __shared__ int s_cnt[kMaxBuckets];        // counts, then fill cursors
  __shared__ int s_start[kMaxBuckets + 1];  // exclusive scan of the counts
  __shared__ int s_perm[kSumTile];          // tile points sorted by bucket
  __shared__ int s_key[kSumTile];           // bucket of each tile point, -1 none
  __shared__ int s_ev[2];
  __shared__ int s_warp[kSumThreads / 32];
  const int V = 5 + F;
  const int tid = threadIdx.x;
  const int rep = blockIdx.x % reps;  // accumulator replica of this tile
  const int64_t t0 = (int64_t)blockIdx.x * kSumTile;
  const int n = (int)min((int64_t)kSumTile, P - t0);
  int t[kSumPts];
#pragma unroll
  for (int r = 0; r < kSumPts; ++r) {
    const int p = tid + r * kSumThreads;
    t[r] = p < n ? token_id[t0 + p] : -1;
  }
  float* sc = s_rows;
  float* sf = s_rows + 4 * kSumTile;
  if (staged) {  // coalesced copies of the tile's rows
    const float4* c4 = reinterpret_cast<const float4*>(coords) + t0;
    for (int p = tid; p < n; p += kSumThreads) reinterpret_cast<float4*>(sc)[p] = __ldg(c4 + p);
    const float* fr = feats + t0 * F;
    for (int e = tid; e < n * F; e += kSumThreads) sf[e] = __ldg(fr + e);
  }
  if (tid < 2) s_ev[tid] = sum_event_of(offsets, 0, B - 1, tid ? t0 + n - 1 : t0);
  __syncthreads();
  const int lo = s_ev[0], hi = max(s_ev[0], s_ev[1]);
  const int64_t nb64 = (int64_t)(hi - lo + 1) * K;
  const bool dense = nb64 <= kMaxBuckets;  // block-uniform
  const int NB = dense ? (int)nb64 : 0;
  for (int e = tid; e < NB; e += kSumThreads) s_cnt[e] = 0;
  __syncthreads();
#pragma unroll
  for (int r = 0; r < kSumPts; ++r) {
    const int p = tid + r * kSumThreads;
    if (p >= n) continue;
    const int64_t i = t0 + p;
    const int b = sum_event_of(offsets, lo, hi, i);
    int key = -1;
    if (__ldg(offsets + b) > i || __ldg(offsets + b + 1) <= i) record_error(hdr, kDevBadOffsets);
    else if (t[r] >= K || t[r] < -1) record_error(hdr, kDevBadToken);
    else if (t[r] >= 0) key = (b - lo) * K + t[r];
    if (key >= 0 && !dense) {  // point by point into the accumulators
      double* a = acc + (((int64_t)rep * B + b) * K + t[r]) * V;
      for (int v = 0; v < V; ++v) atomicAdd(a + v, summary_value(coords, feats, F, charge_col, i, v));
      key = -1;
    }
    s_key[p] = key;
    if (key >= 0) atomicAdd(s_cnt + key, 1);
  }
  __syncthreads();
  if (!dense) return;
  // exclusive scan of s_cnt[0..NB): contiguous chunks per thread, then warps
  {
    const int lane = tid & 31, warp = tid >> 5;
    const int ch = (NB + kSumThreads - 1) / kSumThreads;
    const int a = min(NB, tid * ch), z = min(NB, a + ch);
    int sum = 0;
    for (int e = a; e < z; ++e) sum += s_cnt[e];
    int x = sum;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, x, o);
      if (lane >= o) x += y;
    }
    if (lane == 31) s_warp[warp] = x;
    __syncthreads();
    if (warp == 0) {
      int w = lane < kSumThreads / 32 ? s_warp[lane] : 0;
      const int w0 = w;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, w, o);
        if (lane >= o) w += y;
      }
      if (lane < kSumThreads / 32) s_warp[lane] = w - w0;
    }
    __syncthreads();
    int run = s_warp[warp] + x - sum;
    for (int e = a; e < z; ++e) {
      s_start[e] = run;
      run += s_cnt[e];
    }
    if (tid == kSumThreads - 1) s_start[NB] = run;
  }
  __syncthreads();
  for (int e = tid; e < NB; e += kSumThreads) s_cnt[e] = s_start[e];
  __syncthreads();
  for (int p = tid; p < n; p += kSumThreads) {
    const int key = s_key[p];
    if (key >= 0) s_perm[atomicAdd(s_cnt + key, 1)] = p;
  }
  __syncthreads();
  // one item per (bucket, value): the bucket's points in sorted order
  for (int it = tid; it < NB * V; it += kSumThreads) {
    const int bk = it / V, v = it - bk * V;
    const int a = s_start[bk], z = s_start[bk + 1];
    if (a == z) continue;
    double sum = 0.0;  // in sorted order, four values at a time
    int m = a;
    for (; m + 4 <= z; m += 4) {
      double x[4];
#pragma unroll
      for (int u = 0; u < 4; ++u)
        x[u] = tile_value(sc, sf, staged, coords, feats, F, charge_col, t0, s_perm[m + u], v);
#pragma unroll
      for (int u = 0; u < 4; ++u) sum += x[u];
    }
    for (; m < z; ++m) sum += tile_value(sc, sf, staged, coords, feats, F, charge_col, t0, s_perm[m], v);
    const int b = lo + bk / K, j = bk - (bk / K) * K;
    atomicAdd(acc + (((int64_t)rep * B + b) * K + j) * V + v, sum);
  }
}

__global__ void __launch_bounds__(256) k_token_finalize(const double* __restrict__ acc, int reps, int F,
                                                        int64_t rows, float* __restrict__ wsum,
                                                        float* __restrict__ wcoords, float* __restrict__ wfeats) {
  const int V = 5 + F;
  const int64_t n = rows * V;
  const int64_t stride = (int64_t)gridDim.x * blockDim.x;
  for (int64_t e = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; e < n; e += stride) {
    const int64_t r = e / V;
    const int v = (int)(e - r * V);
    double W = 0.0, x = 0.0;
    for (int q = 0; q < reps; ++q) {  // replicas in order
      W += acc[(int64_t)q * n + r * V];
      x += acc[(int64_t)q * n + e];
    }
    if (v == 0) wsum[r] = (float)W;
    else if (v < 5) wcoords[r * 4 + (v - 1)] = W > 0.0 ? (float)(x / W) : 0.f;
    else wfeats[r * F + (v - 5)] = W > 0.0 ? (float)(x / W) : 0.f;
  }
}

}  // namespace

int token_summary_replicas(int B, int K, int F) {
  const int64_t one = (int64_t)B * K * (5 + F) * (int64_t)sizeof(double);
  int64_t r = one > 0 ? kSumReplicaBudget / one : kSumMaxReplicas;
  if (r > kSumMaxReplicas) r = kSumMaxReplicas;
  return r < 1 ? 1 : (int)r;
}

cudaError_t launch_token_summaries(const float* coords, const float* feats, int F, int charge_col,
                                   const int64_t* offsets, int B, int64_t P, int K, const int32_t* token_id,
                                   double* acc, float* wsum, float* wcoords, float* wfeats, WsHeader* hdr,
                                   cudaStream_t s) {
  const int64_t rows = (int64_t)B * K;
  const int V = 5 + F;
  const int reps = token_summary_replicas(B, K, F);
  cudaError_t e = cudaMemsetAsync(acc, 0, (size_t)reps * rows * V * sizeof(double), s);
  if (e != cudaSuccess) return e;
  if (P > 0) {
    // stage the tile's rows in shared memory when they fit (F up to about 36)
    const size_t rows_bytes = (size_t)kSumTile * (4 + F) * sizeof(float);
    const int staged = rows_bytes <= (size_t)kSumStageBytes;
    static bool attr_set[64] = {};
    int dev = 0;
    cudaGetDevice(&dev);
    if (dev >= 0 && dev < 64 && !attr_set[dev]) {
      if ((e = cudaFuncSetAttribute(k_token_sums, cudaFuncAttributeMaxDynamicSharedMemorySize, kSumStageBytes)))
        return e;
      attr_set[dev] = true;
    }
    count_launch();
    k_token_sums<<<(unsigned)((P + kSumTile - 1) / kSumTile), kSumThreads, staged ? rows_bytes : 0, s>>>(
        coords, feats, F, charge_col, offsets, B, P, K, token_id, reps, staged, acc, hdr);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
  }
  const DeviceInfo& di = device_info();
  int64_t g = (rows * V + 255) / 256;
  if (g > (int64_t)di.sm_count * 8) g = (int64_t)di.sm_count * 8;
  if (g < 1) g = 1;
  count_launch();
  k_token_finalize<<<(unsigned)g, 256, 0, s>>>(acc, reps, F, rows, wsum, wcoords, wfeats);
  return cudaGetLastError();
}

}  // namespace fpstok
