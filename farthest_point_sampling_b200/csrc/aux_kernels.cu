// Binning, passthrough, pooling, Lloyd refinement, nearest-centroid assignment
// and the kNN gather of the fpstok tokenizer.
//
// Per-token pooling ("pools the pulses of each token", graphnet PR #923 "Add
// Neptune point-transformer backbone", Summary), small events kept at one
// token per pulse (same page, "What is added", FPSTokenizer), nearest-centroid
// assignment and the kNN gather (components/fps.py nearest_assign and
// farthest_point_sampling_with_knn, same list), and charge-weighted Lloyd
// refinement (Neptune README, "How it works", step 1).
//
// Float sums (pool means, Lloyd weighted means) accumulate in float64 and are
// rounded once to float32.  A CTA sorts the points of its chunk by token
// (a counting sort in shared memory), then one thread per (token, value) adds
// that token's points; events spread over several chunks combine their chunk
// sums with float64 atomics in global memory.  Every term is an exact float64
// (a float32, or the product of two float32), so the result differs from a
// sequential float64 sum only by float64 rounding, far below the float32
// rounding of the final mean.
#include "common.cuh"
#include "internal.h"

namespace fpstok {

// ------------------------------------------------------------------ binning

// Size buckets of the counting sort that orders each schedule's list by
// decreasing event size (bucket = n >> shift; shift keeps cap >> shift < 256).
constexpr int kBins = 256;
constexpr int kBinCache = 8192;  // events whose size the binning kernel keeps in shared memory
__device__ __forceinline__ int sched_shift(int q) {
  return q == 0 ? 1 : (q == 1 ? 4 : (q == 2 ? 6 : (q == 3 ? 9 : 10)));
}

// One CTA: classifies every event, builds the per-schedule work lists sorted
// by decreasing size (longest chains first), the (event, chunk) items of FPS
// events, and the accumulator slots; resets the status word and the cursors.
__global__ void __launch_bounds__(1024) k_bin(const int64_t* __restrict__ offsets, int B, int64_t P,
                                               int K, const int32_t* __restrict__ start_local,
                                               int force, int chunk_all, int fused_pool, int latency_events,
                                               Workspace ws) {
  __shared__ int cnt[kNumLists];
  __shared__ int hist[kNumSchedules][kBins];
  __shared__ int n_fps;
  __shared__ int s_n[kBinCache];  // event sizes (cls in the sign: -1 - cls for non-FPS events)
  for (int i = threadIdx.x; i < kNumSchedules * kBins; i += blockDim.x) (&hist[0][0])[i] = 0;
  if (threadIdx.x < kNumLists) cnt[threadIdx.x] = 0;
  if (threadIdx.x < 8) ws.hdr->next_item[threadIdx.x] = 0;
  if (threadIdx.x == 0) {
    ws.hdr->status = 0;
    ws.hdr->detail = 0;
    n_fps = 0;
  }
  __syncthreads();
  // pass 1: classify and count FPS events (four events per thread in flight)
  constexpr int U = 4;
  for (int b0 = threadIdx.x; b0 < B; b0 += U * blockDim.x) {
    int64_t o0[U], o1[U];
    int st[U];
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int b = b0 + u * blockDim.x;
      o0[u] = o1[u] = 0;
      st[u] = 0;
      if (b < B) {
        o0[u] = offsets[b];
        o1[u] = offsets[b + 1];
        if (start_local) st[u] = start_local[b];
      }
    }
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int b = b0 + u * blockDim.x;
      if (b >= B) continue;
      int cls;
      int64_t n = 0;
      if (o0[u] < 0 || o1[u] < o0[u] || o1[u] > P) {
        record_error(ws.hdr, kDevBadOffsets);
        cls = kClsSkip;
      } else {
        if ((b == 0 && o0[u] != 0) || (b == B - 1 && o1[u] != P)) record_error(ws.hdr, kDevBadOffsets);
        n = o1[u] - o0[u];
        cls = n == 0 ? kClsEmpty : (n <= K ? kClsPass : kClsFps);
        if (cls == kClsFps) {
          if (st[u] < 0 || st[u] >= n) {
            record_error(ws.hdr, kDevBadStart);
            cls = kClsSkip;
          } else if (n > kClusterCap) {
            record_error(ws.hdr, kDevTooLarge);
            cls = kClsSkip;
          } else {
            atomicAdd(&n_fps, 1);
          }
        }
      }
      ws.cls[b] = cls;
      if (b < kBinCache) s_n[b] = cls == kClsFps || cls == kClsPass ? (int)n : -1;
    }
  }
  __syncthreads();
  const bool few = n_fps <= latency_events;
  auto schedule_of = [&](int n) {
    int q = n <= kWarpCap ? 0 : (n <= kCtaCap ? 1 : (n <= kCtaSmemCap ? 2 : (n <= kCluster8Cap ? 3 : 4)));
    if (q == 0 && few) q = 1;  // few events: lower latency per step on a whole CTA
    if (force > q) q = force > 4 ? 4 : force;
    return q;
  };
  auto size_of = [&](int b) { return b < kBinCache ? s_n[b] : (int)(offsets[b + 1] - offsets[b]); };
  // pass 2: size histogram per schedule
  for (int b = threadIdx.x; b < B; b += blockDim.x) {
    if (ws.cls[b] != kClsFps) continue;
    const int n = size_of(b);
    const int q = schedule_of(n);
    atomicAdd(&hist[q][min(n >> sched_shift(q), kBins - 1)], 1);
  }
  __syncthreads();
  // exclusive scan from the largest bucket down (one warp per schedule, 8
  // buckets per lane): list position of each bucket
  if (threadIdx.x < 32 * kNumSchedules) {
    const int q = threadIdx.x >> 5, lane = threadIdx.x & 31;
    int v[kBins / 32];
    int sum = 0;
#pragma unroll
    for (int r = 0; r < kBins / 32; ++r) {
      v[r] = hist[q][kBins - 1 - (lane * (kBins / 32) + r)];
      sum += v[r];
    }
    int x = sum;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(kFull, x, o);
      if (lane >= o) x += y;
    }
    int run = x - sum;
#pragma unroll
    for (int r = 0; r < kBins / 32; ++r) {
      hist[q][kBins - 1 - (lane * (kBins / 32) + r)] = run;
      run += v[r];
    }
    if (lane == 31) cnt[q] = run;
  }
  __syncthreads();
  // pass 3: scatter into the sorted lists; chunks and accumulator slots
  for (int b = threadIdx.x; b < B; b += blockDim.x) {
    const int cls = ws.cls[b];
    int fslot = -1, pslot = -1;
    int n = 0;
    if (cls == kClsFps || cls == kClsPass) n = size_of(b);
    if (cls == kClsFps) {
      const int q = schedule_of(n);
      int* list = q == 0 ? ws.list_warp
                         : (q == 1 ? ws.list_cta
                                   : (q == 2 ? ws.list_cta_smem : (q == 3 ? ws.list_cluster8 : ws.list_cluster16)));
      list[atomicAdd(&hist[q][min(n >> sched_shift(q), kBins - 1)], 1)] = b;
      fslot = atomicAdd(&cnt[kListFps], 1);
    }
    if (cls == kClsFps || (chunk_all && cls == kClsPass)) {
      const int nch = (n + kChunk - 1) / kChunk;
      const int base = atomicAdd(&cnt[kListChunks], nch);
      for (int c = 0; c < nch; ++c) ws.chunks[base + c] = make_int2(b, c);
      // pooling items (passthrough events of fps_tokenize are written directly;
      // events of schedules that pool in place are left out)
      if (cls == kClsFps && ((fused_pool >> schedule_of(n)) & 1)) {
        ws.fps_slot[b] = fslot;
        ws.pool_slot[b] = -1;
        continue;
      }
      const int npc = (n + kPoolChunk - 1) / kPoolChunk;
      const int pbase = atomicAdd(&cnt[kListPoolChunks], npc);
      for (int c = 0; c < npc; ++c) ws.pool_chunks[pbase + c] = make_int2(b, c);
      if (npc > 1) pslot = atomicAdd(&cnt[kListPoolSlots], 1);
    }
    ws.fps_slot[b] = fslot;
    ws.pool_slot[b] = pslot;
  }
  __syncthreads();
  if (threadIdx.x < kNumLists) ws.hdr->n_items[threadIdx.x] = cnt[threadIdx.x];
}

cudaError_t launch_bin(const Problem& pb, const Workspace& ws, int chunk_all, cudaStream_t s) {
  const DeviceInfo& di = device_info();
  count_launch();
  k_bin<<<1, 1024, 0, s>>>(pb.offsets, pb.B, pb.P, pb.K, pb.start_local, pb.force_schedule, chunk_all,
                           pb.fused_pool, kLatencyEventsPerSm * di.sm_count, ws);
  return cudaGetLastError();
}

// ------------------------------------------------------------------ passthrough

// Events with N <= K keep one token per pulse; empty and skipped events get
// empty rows; FPS events get their global accumulators cleared.  One warp per
// event, copies unrolled so that loads overlap.
__global__ void __launch_bounds__(256) k_passthrough(Problem pb, Workspace ws, int lloyd_on) {
  const int K = pb.K, F = pb.F, k = pb.k;
  const int lane = threadIdx.x & 31;
  const int gw = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int nw = (gridDim.x * blockDim.x) >> 5;
  for (int b = gw; b < pb.B; b += nw) {
    const int cls = ws.cls[b];
    if (cls == kClsFps) {
      const int ps = ws.pool_slot[b];
      if (ps >= 0) {
        for (int e = lane; e < K * F; e += 32) ws.pool_acc[(int64_t)ps * K * F + e] = 0.0;
        for (int e = lane; e < K; e += 32) ws.pool_cnt[(int64_t)ps * K + e] = 0;
        if (lane == 0) ws.pool_ticket[ps] = 0;
      }
      const int fs = ws.fps_slot[b];
      if (lloyd_on && fs >= 0) {
        for (int e = lane; e < K * 5; e += 32) {
          ws.lloyd[0][(int64_t)fs * K * 5 + e] = 0.0;
          ws.lloyd[1][(int64_t)fs * K * 5 + e] = 0.0;
        }
      }
      continue;
    }
    int64_t off = 0;
    int n = 0;
    if (cls == kClsPass) {
      off = pb.offsets[b];
      n = (int)(pb.offsets[b + 1] - off);
    }
    const float* cf = reinterpret_cast<const float*>(pb.coords) + off * 4;
    float* outc = reinterpret_cast<float*>(pb.centroids) + (int64_t)b * K * 4;
    const int nc = n * 4;
#pragma unroll 8
    for (int e = lane; e < K * 4; e += 32) outc[e] = e < nc ? cf[e] : 0.f;
    const float* fe = pb.feats + off * F;
    float* outp = pb.pooled + (int64_t)b * K * F;
    const int nf = n * F;
#pragma unroll 8
    for (int e = lane; e < K * F; e += 32) outp[e] = e < nf ? fe[e] : 0.f;
    int32_t* ci = pb.centroid_idx + (int64_t)b * K;
    int32_t* co = pb.counts + (int64_t)b * K;
#pragma unroll 4
    for (int j = lane; j < K; j += 32) {
      ci[j] = j < n ? (int32_t)(off + j) : -1;
      co[j] = j < n ? 1 : 0;
    }
    if (pb.token_id)
      for (int j = lane; j < n; j += 32) pb.token_id[off + j] = j;
    if (pb.knn_idx) {  // row j = [point j, -1, ...]; one row per lane at a time
      int32_t* outk = pb.knn_idx + (int64_t)b * K * k;
      for (int j = lane; j < K; j += 32) {
        int32_t* row = outk + (int64_t)j * k;
        row[0] = j < n ? (int32_t)(off + j) : -1;
        for (int r = 1; r < k; ++r) row[r] = -1;
      }
    }
  }
}

cudaError_t launch_passthrough(const Problem& pb, const Workspace& ws, cudaStream_t s) {
  int blocks = (pb.B + 7) / 8;
  if (blocks > 65535) blocks = 65535;
  if (blocks < 1) blocks = 1;
  count_launch();
  k_passthrough<<<blocks, 256, 0, s>>>(pb, ws, pb.lloyd_iters > 0 ? 1 : 0);
  return cudaGetLastError();
}

// ------------------------------------------------------------------ Voronoi pool

// Shared-memory layout of one chunk's counting sort.
struct SortSmem {
  int* lab;    // [kChunk] token of every point
  int* perm;   // [kChunk] point of every sorted position
  int* slab;   // [kChunk] token of every sorted position
  int* cnt;    // [256]
  int* start;  // [256]
  int* cur;    // [256]
};
__device__ __forceinline__ SortSmem sort_smem(int* base, int chunk) {
  return SortSmem{base, base + chunk, base + 2 * chunk, base + 3 * chunk, base + 3 * chunk + 256,
                  base + 3 * chunk + 512};
}
constexpr size_t sort_smem_bytes(int chunk) { return (size_t)(3 * chunk + 3 * 256) * sizeof(int); }

__device__ __forceinline__ void cta_sync() { __syncthreads(); }

constexpr int kStageMaxF = 8;  // the pool kernel stages feature rows in shared memory up to this F

// Sorts the chunk by token and adds up V values per token into acc[K * V]
// (shared float64, zeroed here): balanced over the CTA.
template <typename Val>
__device__ __forceinline__ void chunk_token_sums(const SortSmem& sm, int npts, int K, int V, double* acc, Val val) {
  const int tid = threadIdx.x, T = blockDim.x;
  for (int e = tid; e < K * V; e += T) acc[e] = 0.0;
  label_sort(sm.lab, npts, K, sm.cnt, sm.start, sm.cur, sm.perm, sm.slab, tid, T, cta_sync);
  int nsorted = 0;
  if (K > 0) nsorted = sm.start[K - 1] + sm.cnt[K - 1];
  for (int v0 = 0; v0 < V; v0 += 8)
    segment_sums(sm.perm, sm.slab, nsorted, min(8, V - v0), v0, V, acc, tid, T, val);
  __syncthreads();
}

// One CTA per (event, chunk) item: counting sort of the chunk's points by
// token, float64 sums per (token, feature) -- one thread per token when no
// token holds more than kDenseToken points of the chunk, else the balanced
// segmented sums -- then the means (single-chunk event) or float64
// accumulation in global memory with the last-arriving CTA of the event
// producing the means.  Thread j < K owns token j's outputs.
constexpr int kDenseToken = 32;

__global__ void __launch_bounds__(256) k_pool_voronoi(const float* __restrict__ feats, int F,
                                                      const int64_t* __restrict__ offsets, int K,
                                                      const int32_t* __restrict__ labels,
                                                      float* __restrict__ pooled,
                                                      int32_t* __restrict__ counts, Workspace ws) {
  extern __shared__ int smem_i[];
  const SortSmem sm = sort_smem(smem_i, kPoolChunk);
  double* acc = reinterpret_cast<double*>(smem_i + 3 * kPoolChunk + 3 * 256);  // [K * F]
  float* s_feat = reinterpret_cast<float*>(acc + K * F);  // [kPoolChunk * F] when F <= kStageMaxF
  __shared__ int s_last;
  const int nitems = ws.hdr->n_items[kListPoolChunks];
  const int T = blockDim.x, tid = threadIdx.x;
  for (int item = blockIdx.x; item < nitems; item += gridDim.x) {
    const int2 it = ws.pool_chunks[item];
    const int b = it.x;
    const int64_t off = offsets[b];
    const int n = (int)(offsets[b + 1] - off);
    const int i0 = it.y * kPoolChunk;
    const int npts = min(n, i0 + kPoolChunk) - i0;
    const int nch = (n + kPoolChunk - 1) / kPoolChunk;
    const bool staged = F <= kStageMaxF;
    const float* fe = feats + (off + i0) * F;
#pragma unroll 2
    for (int i = tid; i < npts; i += T) {
      int l = labels[off + i0 + i];
      if (l >= K) {
        record_error(ws.hdr, kDevBadToken);
        l = -1;
      }
      sm.lab[i] = l;
    }
    if (staged) {
#pragma unroll 4
      for (int e = tid; e < npts * F; e += T) s_feat[e] = __ldg(fe + e);
    }
    label_sort(sm.lab, npts, K, sm.cnt, sm.start, sm.cur, sm.perm, sm.slab, tid, T, cta_sync);
    auto val = [&](int i, int f) { return staged ? (double)s_feat[i * F + f] : (double)__ldg(fe + (int64_t)i * F + f); };
    const int cj = tid < K ? sm.cnt[tid] : 0;
    const bool dense = __syncthreads_or(cj > kDenseToken);
    if (dense) {  // balanced over the CTA, flushed into acc
      for (int e = tid; e < K * F; e += T) acc[e] = 0.0;
      __syncthreads();
      const int nsorted = sm.start[K - 1] + sm.cnt[K - 1];
      segment_sums_scan(sm.perm, sm.slab, nsorted, F, 0, F, acc, tid, T, val);
    } else if (tid < K) {  // one thread per token: its (short) run, in sorted order
      const int* pj = sm.perm + sm.start[tid];
      for (int f0 = 0; f0 < F; f0 += 8) {
        double s8[8];
#pragma unroll
        for (int v = 0; v < 8; ++v) s8[v] = 0.0;
        for (int t = 0; t < cj; ++t) {
          const int i = pj[t];
#pragma unroll
          for (int v = 0; v < 8; ++v)
            if (f0 + v < F) s8[v] += val(i, f0 + v);
        }
#pragma unroll
        for (int v = 0; v < 8; ++v)
          if (f0 + v < F) acc[tid * F + f0 + v] = s8[v];
      }
    }
    __syncthreads();
    if (nch == 1) {
      if (tid < K) {
        float* prow = pooled + ((int64_t)b * K + tid) * F;
        for (int f = 0; f < F; ++f) prow[f] = cj ? (float)(acc[tid * F + f] / (double)cj) : 0.f;
        counts[(int64_t)b * K + tid] = cj;
      }
    } else {
      const int ps = ws.pool_slot[b];
      double* gacc = ws.pool_acc + (int64_t)ps * K * F;
      int* gcnt = ws.pool_cnt + (int64_t)ps * K;
      if (tid < K && cj) {
        for (int f = 0; f < F; ++f) atomicAdd(&gacc[tid * F + f], acc[tid * F + f]);
        atomicAdd(&gcnt[tid], cj);
      }
      __threadfence();
      __syncthreads();
      if (tid == 0) s_last = atomicAdd(&ws.pool_ticket[ps], 1) == nch - 1;
      __syncthreads();
      if (s_last && tid < K) {
        __threadfence();
        const int c = __ldcg(&gcnt[tid]);
        float* prow = pooled + ((int64_t)b * K + tid) * F;
        for (int f = 0; f < F; ++f) prow[f] = c ? (float)(__ldcg(&gacc[tid * F + f]) / (double)c) : 0.f;
        counts[(int64_t)b * K + tid] = c;
      }
    }
    __syncthreads();
  }
}

static size_t pool_smem_bytes(int K, int F) {
  return sort_smem_bytes(kPoolChunk) + (size_t)K * F * sizeof(double) +
         (F <= kStageMaxF ? (size_t)kPoolChunk * F * sizeof(float) : 0);
}

cudaError_t launch_pool_voronoi(const float* feats, int F, const int64_t* offsets, int K,
                                const int32_t* labels, float* pooled, int32_t* counts,
                                const Workspace& ws, cudaStream_t s) {
  const DeviceInfo& di = device_info();
  count_launch();
  k_pool_voronoi<<<di.sm_count * 8, 256, pool_smem_bytes(K, F), s>>>(feats, F, offsets, K, labels, pooled, counts,
                                                                     ws);
  return cudaGetLastError();
}

// ------------------------------------------------------------------ nearest centroid

// Centroid slots padded to a whole number of pairs; the pad holds +inf
// coordinates, whose distance to any finite point is +inf.
__host__ __device__ constexpr int pad_pairs(int nv) { return (nv + 1) & ~1; }

__device__ __forceinline__ void load_cents_padded(const float4* __restrict__ c, int nv, Cent2* s) {
  const float inf = __int_as_float(0x7f800000);
  for (int j = threadIdx.x; j < pad_pairs(nv); j += blockDim.x)
    s[j] = cent2(j < nv ? c[j] : make_float4(inf, inf, inf, inf));
}

// Nearest centroid of this thread's 2 PR points (PR packed pairs) among the
// centroid pairs cs[0 .. 2 ng) (pads +inf).  The loop keeps, per point, the
// smallest distance and the pair g of centroids holding it: one three-input
// minimum, one compare and one select per point and pair of centroids, the
// strict '<' keeping the earliest pair on ties.  The slot inside the winning
// pair is then 2 g when the recomputed distance to centroid 2 g equals the
// minimum, else 2 g + 1.  Both passes evaluate the same float32 distance, so
// the result is exactly the lowest-slot nearest centroid.
template <int PR>
__device__ __forceinline__ void nearest_pairs(const uint64_t (&X)[PR], const uint64_t (&Y)[PR],
                                              const uint64_t (&Z)[PR], const uint64_t (&W)[PR],
                                              const Cent2* __restrict__ cs, int ng, int (&lab)[2 * PR]) {
  const uint64_t z2 = opaque_zero2();
  float best[2 * PR];
#pragma unroll
  for (int r = 0; r < 2 * PR; ++r) {
    best[r] = __int_as_float(0x7f800000);
    lab[r] = 0;
  }
#pragma unroll 1
  for (int g = 0; g < ng; ++g) {
    const Cent2 A = cs[2 * g], B = cs[2 * g + 1];
#pragma unroll
    for (int p = 0; p < PR; ++p) {
      const uint64_t da = dist2(X[p], Y[p], Z[p], W[p], A, z2);
      const uint64_t db = dist2(X[p], Y[p], Z[p], W[p], B, z2);
      const float m0 = min3f(best[2 * p], lo2(da), lo2(db));
      const float m1 = min3f(best[2 * p + 1], hi2(da), hi2(db));
      lab[2 * p] = m0 < best[2 * p] ? g : lab[2 * p];
      lab[2 * p + 1] = m1 < best[2 * p + 1] ? g : lab[2 * p + 1];
      best[2 * p] = m0;
      best[2 * p + 1] = m1;
    }
  }
#pragma unroll
  for (int r = 0; r < 2 * PR; ++r) {
    const int p = r >> 1;
    const float4 q = (r & 1) ? make_float4(hi2(X[p]), hi2(Y[p]), hi2(Z[p]), hi2(W[p]))
                             : make_float4(lo2(X[p]), lo2(Y[p]), lo2(Z[p]), lo2(W[p]));
    const Cent2 c = cs[2 * lab[r]];
    const float d = dist1(q, make_float4(lo2(c.x), lo2(c.y), lo2(c.z), lo2(c.t)));
    lab[r] = 2 * lab[r] + (d == best[r] ? 0 : 1);
  }
}

// Nearest centroid of the chunk points tid + r T (r < 2 PR NPASS) of
// `pts` (npts valid), in NPASS passes of PR pairs; emit(li, label) is called
// for every valid local point li at the end of its pass.
template <int PR, int NPASS, int T, typename Emit>
__device__ __forceinline__ void chunk_nearest(const float4* __restrict__ pts, int npts,
                                              const Cent2* __restrict__ cs, int ng, Emit emit) {
  const int tid = threadIdx.x;
#pragma unroll 1
  for (int q = 0; q < NPASS; ++q) {
    uint64_t X[PR], Y[PR], Z[PR], W[PR];
#pragma unroll
    for (int p = 0; p < PR; ++p) {
      const int ia = tid + (2 * PR * q + 2 * p) * T, ib = ia + T;
      float4 a = make_float4(0.f, 0.f, 0.f, 0.f), c = a;
      if (ia < npts) a = ldg4(pts + ia);
      if (ib < npts) c = ldg4(pts + ib);
      X[p] = pack2(a.x, c.x);
      Y[p] = pack2(a.y, c.y);
      Z[p] = pack2(a.z, c.z);
      W[p] = pack2(a.w, c.w);
    }
    int l[2 * PR];
    nearest_pairs<PR>(X, Y, Z, W, cs, ng, l);
#pragma unroll
    for (int r = 0; r < 2 * PR; ++r) {
      const int li = tid + (2 * PR * q + r) * T;
      if (li < npts) emit(li, l[r]);
    }
  }
}

constexpr int kNearestPairs = 2;  // pairs per pass: with two centroids in flight, 8 distance chains
constexpr int kNearestPasses = kChunk / (2 * kNearestPairs * 256);
static_assert(kNearestPasses * 2 * kNearestPairs * 256 == kChunk, "whole passes per chunk");

// Standalone nearest-centroid assignment over (event, chunk) items.
constexpr int kAssignThreads = 256;

__global__ void __launch_bounds__(kAssignThreads, 3) k_assign(const float4* __restrict__ coords,
                                                           const int64_t* __restrict__ offsets, int K,
                                                           const float4* __restrict__ centroids,
                                                           const int32_t* __restrict__ valid,
                                                           int32_t* __restrict__ token_id, Workspace ws) {
  constexpr int T = kAssignThreads;
  extern __shared__ Cent2 s_cent[];  // [pad_pairs(K)]
  const int tid = threadIdx.x;
  const int nitems = ws.hdr->n_items[kListChunks];
  for (int item = blockIdx.x; item < nitems; item += gridDim.x) {
    const int2 it = ws.chunks[item];
    const int b = it.x;
    const int64_t off = offsets[b];
    const int n = (int)(offsets[b + 1] - off);
    int nv = valid ? valid[b] : min(n, K);
    if (nv < 0 || nv > K) {
      record_error(ws.hdr, kDevBadToken);
      nv = 0;
    }
    load_cents_padded(centroids + (int64_t)b * K, nv, s_cent);
    __syncthreads();
    const int i0 = it.y * kChunk, npts = min(n, i0 + kChunk) - i0;
    int32_t* out = token_id + off + i0;
    chunk_nearest<kNearestPairs, kNearestPasses, T>(coords + off + i0, npts, s_cent, pad_pairs(nv) / 2,
                                                    [&](int li, int l) { out[li] = nv > 0 ? l : -1; });
    __syncthreads();
  }
}

// ------------------------------------------------------------------ Lloyd

__device__ __forceinline__ float charge_of(const float* fe, int F, int charge_col, int i) {
  return charge_col < 0 ? 1.0f : __ldg(fe + (int64_t)i * F + charge_col);
}

// Lloyd sums of one chunk whose labels, points and charges are in shared
// memory: W_j = sum q and S_j = sum q p per token, added to `out` (float64,
// [K][5], global).
__device__ __forceinline__ void lloyd_chunk_sums(const SortSmem& sm, const float4* s_p, const float* s_q, int npts,
                                                 int K, double* acc, double* out) {
  chunk_token_sums(sm, npts, K, 5, acc, [&](int i, int v) {
    const double q = (double)s_q[i];
    if (v == 0) return q;
    const float4 p = s_p[i];
    return q * (double)(v == 1 ? p.x : (v == 2 ? p.y : (v == 3 ? p.z : p.w)));
  });
  for (int e = threadIdx.x; e < K * 5; e += blockDim.x)
    if (sm.cnt[e / 5]) atomicAdd(&out[e], acc[e]);
}

constexpr size_t kLloydSmemBytes =
    sort_smem_bytes(kChunk) + (size_t)kChunk * (sizeof(float4) + sizeof(float)) + 256 * 5 * sizeof(double);

// Cell sums of the current labels.
__global__ void __launch_bounds__(256) k_lloyd_sums(const float4* __restrict__ coords,
                                                    const float* __restrict__ feats, int F,
                                                    int charge_col, const int64_t* __restrict__ offsets,
                                                    int K, const int32_t* __restrict__ labels,
                                                    Workspace ws, double* __restrict__ out) {
  extern __shared__ int smem_i[];
  const SortSmem sm = sort_smem(smem_i, kChunk);
  float4* s_p = reinterpret_cast<float4*>(smem_i + 3 * kChunk + 3 * 256);
  float* s_q = reinterpret_cast<float*>(s_p + kChunk);
  double* acc = reinterpret_cast<double*>(s_q + kChunk);  // [K * 5]
  const int nitems = ws.hdr->n_items[kListChunks];
  for (int item = blockIdx.x; item < nitems; item += gridDim.x) {
    const int2 it = ws.chunks[item];
    const int b = it.x;
    const int fs = ws.fps_slot[b];
    if (fs < 0) continue;  // uniform across the CTA
    const int64_t off = offsets[b];
    const int n = (int)(offsets[b + 1] - off);
    const int i0 = it.y * kChunk, npts = min(n, i0 + kChunk) - i0;
    const float4* pts = coords + off + i0;
    const float* fe = feats ? feats + (off + i0) * F : nullptr;
#pragma unroll 4
    for (int i = threadIdx.x; i < npts; i += blockDim.x) {
      int l = labels[off + i0 + i];
      if ((unsigned)l >= (unsigned)K) {
        record_error(ws.hdr, kDevBadToken);
        l = -1;
      }
      sm.lab[i] = l;
      s_p[i] = ldg4(pts + i);
      s_q[i] = charge_of(fe, F, charge_col, i);
    }
    lloyd_chunk_sums(sm, s_p, s_q, npts, K, acc, out + (int64_t)fs * K * 5);
    __syncthreads();
  }
}

// One Lloyd iteration per (event, chunk) item: the centroids from the cell
// sums `in` (an empty cell or a zero weight keeps its centroid), the nearest
// of them for the chunk's points (eight per thread, in two passes) and,
// unless this is the last iteration (next == nullptr), the chunk's cell sums
// of the new labels added into `next`.  Also clears `clear`, which the
// following iteration accumulates into.
constexpr int kLloydThreads = 256;
constexpr int kLloydPts = kChunk / kLloydThreads;  // points per thread
static_assert(kLloydPts == 2 * kNearestPairs * kNearestPasses, "chunk_nearest covers the chunk");

static size_t lloyd_step_smem_bytes(int K) {
  return (size_t)(2 * kChunk + 3 * 256) * sizeof(int) + (size_t)kChunk * (sizeof(float4) + sizeof(float)) +
         (size_t)K * 5 * sizeof(double) + (size_t)pad_pairs(K) * sizeof(Cent2);
}

__global__ void __launch_bounds__(kLloydThreads, 3) k_lloyd_step(const float4* __restrict__ coords,
                                                                 const float* __restrict__ feats, int F,
                                                                 int charge_col,
                                                                 const int64_t* __restrict__ offsets, int K,
                                                                 int32_t* __restrict__ labels,
                                                                 float4* __restrict__ centroids, Workspace ws,
                                                                 const double* __restrict__ in,
                                                                 double* __restrict__ next,
                                                                 double* __restrict__ clear, int64_t clear_n) {
  constexpr int T = kLloydThreads;
  extern __shared__ int smem_i[];
  int* perm = smem_i;              // [kChunk]
  int* slab = perm + kChunk;       // [kChunk]
  int* cnt = slab + kChunk;        // [256]
  int* start = cnt + 256;          // [256]
  int* cur = start + 256;          // [256]
  float4* s_p = reinterpret_cast<float4*>(cur + 256);  // [kChunk]
  float* s_q = reinterpret_cast<float*>(s_p + kChunk);  // [kChunk]
  double* acc = reinterpret_cast<double*>(s_q + kChunk);  // [K * 5]
  Cent2* s_cent = reinterpret_cast<Cent2*>(acc + K * 5);  // [K]
  const int tid = threadIdx.x;
  for (int64_t e = (int64_t)blockIdx.x * T + tid; e < clear_n; e += (int64_t)gridDim.x * T) clear[e] = 0.0;
  const int nitems = ws.hdr->n_items[kListChunks];
  for (int item = blockIdx.x; item < nitems; item += gridDim.x) {
    const int2 it = ws.chunks[item];
    const int b = it.x;
    const int fs = ws.fps_slot[b];
    if (fs < 0) continue;  // uniform across the CTA
    const int64_t off = offsets[b];
    const int n = (int)(offsets[b + 1] - off);
    const double* sb = in + (int64_t)fs * K * 5;
    for (int j = tid; j < K; j += T) {
      const double W = __ldcg(&sb[j * 5]);
      float4 c = centroids[(int64_t)b * K + j];
      if (W > 0.0) {
        c.x = (float)(__ldcg(&sb[j * 5 + 1]) / W);
        c.y = (float)(__ldcg(&sb[j * 5 + 2]) / W);
        c.z = (float)(__ldcg(&sb[j * 5 + 3]) / W);
        c.w = (float)(__ldcg(&sb[j * 5 + 4]) / W);
      }
      s_cent[j] = cent2(c);
      if (it.y == 0) centroids[(int64_t)b * K + j] = c;  // every chunk computes the same values
    }
    if (tid == 0 && (K & 1)) {
      const float inf = __int_as_float(0x7f800000);
      s_cent[K] = cent2(make_float4(inf, inf, inf, inf));
    }
    if (next) {
      for (int j = tid; j < K; j += T) cnt[j] = 0;
      for (int e = tid; e < K * 5; e += T) acc[e] = 0.0;
    }
    __syncthreads();
    const int i0 = it.y * kChunk, npts = min(n, i0 + kChunk) - i0;
    const float4* pts = coords + off + i0;
    int32_t* lab_out = labels + off + i0;
    const float* fe = feats ? feats + (off + i0) * F : nullptr;
    chunk_nearest<kNearestPairs, kNearestPasses, T>(pts, npts, s_cent, pad_pairs(K) / 2, [&](int li, int l) {
      lab_out[li] = l;
      if (next) {
        s_p[li] = ldg4(pts + li);  // read a moment ago: a cache hit
        s_q[li] = charge_of(fe, F, charge_col, li);
        atomicAdd(&cnt[l], 1);
      }
    });
    if (next) {  // counting sort by label (this thread's own labels, read back), then the cell sums
      __syncthreads();
      if (tid < 32) count_scan(cnt, start, cur, K, tid);
      __syncthreads();
#pragma unroll
      for (int r = 0; r < kLloydPts; ++r) {
        const int li = tid + r * T;
        if (li < npts) {
          const int l = lab_out[li];
          const int pos = atomicAdd(&cur[l], 1);
          perm[pos] = li;
          slab[pos] = l;
        }
      }
      __syncthreads();
      segment_sums(perm, slab, npts, 5, 0, 5, acc, tid, T, [&](int i, int v) {
        const double q = (double)s_q[i];
        if (v == 0) return q;
        const float4 p = s_p[i];
        return q * (double)(v == 1 ? p.x : (v == 2 ? p.y : (v == 3 ? p.z : p.w)));
      });
      __syncthreads();
      double* out = next + (int64_t)fs * K * 5;
      for (int e = tid; e < K * 5; e += T)
        if (cnt[e / 5]) atomicAdd(&out[e], acc[e]);
    }
    __syncthreads();
  }
}

// Lloyd refinement: cell sums of the incoming labels into buffer 0, then
// iteration t updates from buffer t % 3, accumulates the next sums into
// (t + 1) % 3 unless it is the last one, and clears (t + 2) % 3 when
// iteration t + 1 will accumulate into it (buffers 0 and 1 start zeroed).
cudaError_t launch_lloyd(const Problem& pb, const Workspace& ws, int32_t* labels, cudaStream_t s) {
  const DeviceInfo& di = device_info();
  const int K = pb.K;
  const float* feats = pb.charge_col >= 0 ? pb.feats : nullptr;
  const int64_t per = (int64_t)K * 5;
  cudaError_t e;
  count_launch();
  k_lloyd_sums<<<di.sm_count * 2, 256, kLloydSmemBytes, s>>>(pb.coords, feats, pb.F, pb.charge_col, pb.offsets,
                                                             K, labels, ws, ws.lloyd[0]);
  if ((e = cudaGetLastError())) return e;
  const size_t sm_step = lloyd_step_smem_bytes(K);
  for (int t = 0; t < pb.lloyd_iters; ++t) {
    const bool last = t == pb.lloyd_iters - 1;
    double* clear = (t + 1 < pb.lloyd_iters - 1) ? ws.lloyd[(t + 2) % 3] : nullptr;
    count_launch();
    k_lloyd_step<<<di.sm_count * 3, kLloydThreads, sm_step, s>>>(
        pb.coords, feats, pb.F, pb.charge_col, pb.offsets, K, labels, pb.centroids, ws, ws.lloyd[t % 3],
        last ? nullptr : ws.lloyd[(t + 1) % 3], clear, clear ? (int64_t)ws.fps_slots * per : 0);
    if ((e = cudaGetLastError())) return e;
  }
  return cudaSuccess;
}

// Shared-memory limits of the auxiliary kernels, set once per device for the
// largest K and F the ABI accepts.
cudaError_t prepare_aux_kernels() {
  cudaError_t e;
  if ((e = cudaFuncSetAttribute(k_lloyd_sums, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kLloydSmemBytes)))
    return e;
  if ((e = cudaFuncSetAttribute(k_lloyd_step, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                (int)lloyd_step_smem_bytes(256))))
    return e;
  const size_t pool_max = pool_smem_bytes(256, 64) > pool_smem_bytes(256, kStageMaxF)
                              ? pool_smem_bytes(256, 64)
                              : pool_smem_bytes(256, kStageMaxF);
  if ((e = cudaFuncSetAttribute(k_pool_voronoi, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)pool_max)))
    return e;
  return cudaSuccess;
}

// ------------------------------------------------------------------ kNN

// Mean of the features of the valid entries of one kNN row (warp-cooperative;
// each lane contributes the entries it holds).  Lane 0 writes the results.
template <int KPL>
__device__ __forceinline__ void knn_row_pool(const float* __restrict__ feats, int F, const int* gidx,
                                             float* __restrict__ pooled_row, int32_t* count_out) {
  const int lane = threadIdx.x & 31;
  int c = 0;
#pragma unroll
  for (int q = 0; q < KPL; ++q) c += gidx[q] >= 0;
  c = __reduce_add_sync(kFull, c);
  for (int f = 0; f < F; ++f) {
    double s = 0.0;
#pragma unroll
    for (int q = 0; q < KPL; ++q)
      if (gidx[q] >= 0) s += (double)feats[(int64_t)gidx[q] * F + f];
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(kFull, s, o);
    if (lane == 0) pooled_row[f] = c ? (float)(s / (double)c) : 0.f;
  }
  if (lane == 0) *count_out = c;
}

// Compare-exchange of a bitonic network step across the warp: the lane
// keeps the smaller key when it is the lower lane of an ascending pair (or
// the upper lane of a descending one), else the larger.
__device__ __forceinline__ uint64_t cmpx64(uint64_t v, int lane, int stride, bool ascending) {
  const uint64_t o = __shfl_xor_sync(kFull, v, stride);
  const bool keep_min = ((lane & stride) == 0) == ascending;
  const bool o_less = o < v;
  return keep_min == o_less ? o : v;
}

// Ascending bitonic sort of one 64-bit key per lane (lane e ends with the
// e-th smallest).
__device__ __forceinline__ uint64_t warp_sort64(uint64_t v, int lane) {
#pragma unroll
  for (int size = 2; size <= 32; size <<= 1)
#pragma unroll
    for (int stride = size >> 1; stride > 0; stride >>= 1) v = cmpx64(v, lane, stride, (lane & size) == 0);
  return v;
}

// The 32 smallest keys of two ascending warp lists, ascending: the
// element-wise minimum of one list and the other reversed is a bitonic
// sequence holding them, which one half-cleaner cascade sorts.
__device__ __forceinline__ uint64_t warp_merge64(uint64_t a, uint64_t b, int lane) {
  const uint64_t r = __shfl_sync(kFull, b, 31 - lane);
  uint64_t v = a < r ? a : r;
#pragma unroll
  for (int stride = 16; stride > 0; stride >>= 1) v = cmpx64(v, lane, stride, true);
  return v;
}

// A 32-point chunk with more passing keys than this is sorted and merged
// into the list at once; fewer are inserted one by one.
constexpr int kKnnInsertMax = 4;

// Row order of the kNN kernel inside fps_tokenize: the FPS events of the
// binning kernel's schedule lists, largest schedule first (each list is
// sorted by decreasing size), so that the longest rows start first.
struct KnnOrder {
  const int* list[kNumSchedules];  // list[q] = the list of schedule kNumSchedules - 1 - q
  int on;
};

__device__ __forceinline__ int ordered_event(const WsHeader* hdr, const KnnOrder& o, int e) {
#pragma unroll
  for (int q = 0; q < kNumSchedules; ++q) {
    const int nq = hdr->n_items[kNumSchedules - 1 - q];
    if (e < nq) return o.list[q][e];
    e -= nq;
  }
  return -1;
}

// One warp per (event, centroid) row: the k smallest (d, index) keys of the
// event, kept sorted across the warp (element e at lane e % 32, slot e / 32).
template <int KPL>
__global__ void __launch_bounds__(256) k_knn(const float4* __restrict__ coords,
                                             const int64_t* __restrict__ offsets, int B,
                                             const float4* __restrict__ centroids,
                                             const int32_t* __restrict__ valid, int K, int k,
                                             int32_t* __restrict__ knn_idx,
                                             const float* __restrict__ feats, int F,
                                             float* __restrict__ pooled, int32_t* __restrict__ counts,
                                             KnnOrder ord, WsHeader* hdr) {
  const int lane = threadIdx.x & 31;
  const int gw = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int nw = (gridDim.x * blockDim.x) >> 5;
  int n_ev = B;
  if (ord.on) {
    n_ev = 0;
#pragma unroll
    for (int q = 0; q < kNumSchedules; ++q) n_ev += hdr->n_items[q];
  }
  const int64_t rows = (int64_t)n_ev * K;
  const int kq = (k - 1) >> 5, kl = (k - 1) & 31;
  for (int64_t r = gw; r < rows; r += nw) {
    const int e = (int)(r / K), j = (int)(r - (int64_t)e * K);
    const int b = ord.on ? ordered_event(hdr, ord, e) : e;
    const int64_t orow = (int64_t)b * K + j;  // output row
    const int64_t o0 = offsets[b], o1 = offsets[b + 1];
    int n = 0, nv = 0;
    if (o0 >= 0 && o1 >= o0) {
      n = (int)(o1 - o0);
      nv = valid ? valid[b] : min(n, K);
      if (nv < 0 || nv > K) {
        if (lane == 0) record_error(hdr, kDevBadToken);
        nv = 0;
      }
    } else if (lane == 0) {
      record_error(hdr, kDevBadOffsets);
    }
    uint64_t L[KPL];
#pragma unroll
    for (int q = 0; q < KPL; ++q) L[q] = ~0ull;
    if (j < nv) {
      const float4 c = centroids[orow];
      const float4* pts = coords + o0;
      uint64_t thr = ~0ull;
      constexpr int U = 4;  // 32-point chunks loaded per iteration
      for (int base = 0; base < n; base += 32 * U) {
        float4 pt[U];
#pragma unroll
        for (int u = 0; u < U; ++u) {
          const int i = base + u * 32 + lane;
          pt[u] = i < n ? ldg4(pts + i) : make_float4(0.f, 0.f, 0.f, 0.f);
        }
#pragma unroll
        for (int u = 0; u < U; ++u) {
          const int i = base + u * 32 + lane;
          const uint64_t key =
              i < n ? (((uint64_t)__float_as_uint(dist1(pt[u], c)) << 32) | (uint32_t)i) : ~0ull;
          unsigned mask = __ballot_sync(kFull, key < thr);
          if constexpr (KPL == 1) {
            if (__popc(mask) > kKnnInsertMax) {  // many candidates: sort them and merge
              L[0] = warp_merge64(L[0], warp_sort64(key < thr ? key : ~0ull, lane), lane);
              thr = __shfl_sync(kFull, L[0], kl);
              mask = 0;
            }
          }
          while (mask) {
            const int src = __ffs(mask) - 1;
            mask &= mask - 1;
            const uint64_t v = __shfl_sync(kFull, key, src);
            if (v >= thr) continue;
            int pos = 0;
#pragma unroll
            for (int q = 0; q < KPL; ++q) pos += __popc(__ballot_sync(kFull, L[q] < v));
#pragma unroll
            for (int q = KPL - 1; q >= 0; --q) {
              uint64_t up = __shfl_up_sync(kFull, L[q], 1);
              if (q > 0) {
                const uint64_t carry = __shfl_sync(kFull, L[q - 1], 31);
                if (lane == 0) up = carry;
              }
              const int e2 = q * 32 + lane;
              if (e2 > pos) L[q] = up;
              else if (e2 == pos) L[q] = v;
            }
            uint64_t t = 0;
#pragma unroll
            for (int q = 0; q < KPL; ++q)
              if (q == kq) t = L[q];
            thr = __shfl_sync(kFull, t, kl);
          }
        }
      }
    }
    int gidx[KPL];
#pragma unroll
    for (int q = 0; q < KPL; ++q) {
      const int e2 = q * 32 + lane;
      gidx[q] = (e2 < k && L[q] != ~0ull) ? (int)(o0 + (int64_t)(uint32_t)L[q]) : -1;
      if (e2 < k) knn_idx[orow * k + e2] = gidx[q];
    }
    if (pooled) knn_row_pool<KPL>(feats, F, gidx, pooled + orow * F, counts + orow);
  }
}

cudaError_t launch_knn(const float4* coords, const int64_t* offsets, int B, const float4* centroids,
                       const int32_t* valid_tokens, int K, int k, int32_t* knn_idx, const float* feats,
                       int F, float* pooled, int32_t* counts, const Workspace* ws, WsHeader* hdr,
                       cudaStream_t s) {
  const DeviceInfo& di = device_info();
  const int64_t rows = (int64_t)B * K;
  int64_t blocks = (rows + 7) / 8;
  const int64_t cap = (int64_t)di.sm_count * 16;
  if (blocks > cap) blocks = cap;
  if (blocks < 1) blocks = 1;
  KnnOrder ord{};
  if (ws) {
    ord.on = 1;
    ord.list[0] = ws->list_cluster16;
    ord.list[1] = ws->list_cluster8;
    ord.list[2] = ws->list_cta_smem;
    ord.list[3] = ws->list_cta;
    ord.list[4] = ws->list_warp;
  }
  count_launch();
  if (k <= 32)
    k_knn<1><<<(int)blocks, 256, 0, s>>>(coords, offsets, B, centroids, valid_tokens, K, k, knn_idx,
                                         feats, F, pooled, counts, ord, hdr);
  else if (k <= 64)
    k_knn<2><<<(int)blocks, 256, 0, s>>>(coords, offsets, B, centroids, valid_tokens, K, k, knn_idx,
                                         feats, F, pooled, counts, ord, hdr);
  else
    k_knn<4><<<(int)blocks, 256, 0, s>>>(coords, offsets, B, centroids, valid_tokens, K, k, knn_idx,
                                         feats, F, pooled, counts, ord, hdr);
  return cudaGetLastError();
}

// Standalone kNN pooling over given rows.
template <int KPL>
__global__ void __launch_bounds__(256) k_pool_knn(const float* __restrict__ feats, int F, int64_t rows,
                                                  int k, const int32_t* __restrict__ knn_idx, int64_t P,
                                                  float* __restrict__ pooled, int32_t* __restrict__ counts,
                                                  WsHeader* hdr) {
  const int lane = threadIdx.x & 31;
  const int gw = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int nw = (gridDim.x * blockDim.x) >> 5;
  for (int64_t r = gw; r < rows; r += nw) {
    int gidx[KPL];
#pragma unroll
    for (int q = 0; q < KPL; ++q) {
      const int e = q * 32 + lane;
      int v = e < k ? knn_idx[r * k + e] : -1;
      if (v >= P) {
        record_error(hdr, kDevBadToken);
        v = -1;
      }
      gidx[q] = v;
    }
    knn_row_pool<KPL>(feats, F, gidx, pooled + r * F, counts + r);
  }
}

cudaError_t launch_pool_knn(const float* feats, int F, int B, int K, int k, const int32_t* knn_idx,
                            int64_t P, float* pooled, int32_t* counts, WsHeader* hdr, cudaStream_t s) {
  const DeviceInfo& di = device_info();
  const int64_t rows = (int64_t)B * K;
  int64_t blocks = (rows + 7) / 8;
  const int64_t cap = (int64_t)di.sm_count * 16;
  if (blocks > cap) blocks = cap;
  if (blocks < 1) blocks = 1;
  count_launch();
  if (k <= 32)
    k_pool_knn<1><<<(int)blocks, 256, 0, s>>>(feats, F, rows, k, knn_idx, P, pooled, counts, hdr);
  else if (k <= 64)
    k_pool_knn<2><<<(int)blocks, 256, 0, s>>>(feats, F, rows, k, knn_idx, P, pooled, counts, hdr);
  else
    k_pool_knn<4><<<(int)blocks, 256, 0, s>>>(feats, F, rows, k, knn_idx, P, pooled, counts, hdr);
  return cudaGetLastError();
}

cudaError_t launch_assign(const float4* coords, const int64_t* offsets, const float4* centroids,
                          const int32_t* valid_tokens, int K, int32_t* token_id, const Workspace& ws,
                          cudaStream_t s) {
  const DeviceInfo& di = device_info();
  const size_t sm = (size_t)pad_pairs(K) * sizeof(Cent2);
  count_launch();
  k_assign<<<di.sm_count * 4, 256, sm, s>>>(coords, offsets, K, centroids, valid_tokens, token_id, ws);
  return cudaGetLastError();
}

}  // namespace fpstok
