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

// Exclusive prefix sum of v over the CTA and (in `total`) the CTA's sum;
// tmp: 32 ints of shared memory.  Every thread of the CTA must call it.
__device__ __forceinline__ int cta_exclusive_scan(int v, int* tmp, int& total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = blockDim.x >> 5;
  int x = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(kFull, x, o);
    if (lane >= o) x += y;
  }
  if (lane == 31) tmp[warp] = x;
  __syncthreads();
  if (warp == 0) {
    int w = lane < nw ? tmp[lane] : 0;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(kFull, w, o);
      if (lane >= o) w += y;
    }
    tmp[lane] = w;  // inclusive over the warps
  }
  __syncthreads();
  const int before = warp > 0 ? tmp[warp - 1] : 0;
  total = tmp[nw - 1];
  __syncthreads();  // tmp may be reused
  return before + x - v;
}

// 64-bit form of cta_exclusive_scan (tmp: 32 x 64 bits of shared memory).
__device__ __forceinline__ unsigned long long cta_exclusive_scan64(unsigned long long v, unsigned long long* tmp,
                                                                   unsigned long long& total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = blockDim.x >> 5;
  unsigned long long x = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const unsigned long long y = __shfl_up_sync(kFull, x, o);
    if (lane >= o) x += y;
  }
  if (lane == 31) tmp[warp] = x;
  __syncthreads();
  if (warp == 0) {
    unsigned long long w = lane < nw ? tmp[lane] : 0ull;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const unsigned long long y = __shfl_up_sync(kFull, w, o);
      if (lane >= o) w += y;
    }
    tmp[lane] = w;
  }
  __syncthreads();
  const unsigned long long before = warp > 0 ? tmp[warp - 1] : 0ull;
  total = tmp[nw - 1];
  __syncthreads();
  return before + x - v;
}

// Writes the work items (b, c * step), c < count, of every lane's event with
// the whole warp: the events that have items are taken in turn and every
// lane writes a share of each (all lanes call it).
__device__ __forceinline__ void warp_fill_items(int2* dst, int base, int count, int b, int step) {
  const int lane = threadIdx.x & 31;
  unsigned m = __ballot_sync(kFull, count > 0);
  while (m) {
    const int src = __ffs(m) - 1;
    m &= m - 1;
    const int sb = __shfl_sync(kFull, base, src), sc = __shfl_sync(kFull, count, src);
    const int se = __shfl_sync(kFull, b, src);
    for (int c = lane; c < sc; c += 32) dst[sb + c] = make_int2(se, c * step);
  }
}

// One CTA: classifies every event, builds the per-schedule work lists sorted
// by decreasing size (longest chains first), the (event, chunk) items of FPS
// events, and the accumulator slots; resets the status word and the cursors.
// Threads of the one binning CTA: its passes are chains of CTA barriers, and
// a barrier of fewer warps is cheaper.
#ifndef FPS_BIN_THREADS
#define FPS_BIN_THREADS 1024
#endif
constexpr int kBinThreads = FPS_BIN_THREADS;

__global__ void __launch_bounds__(kBinThreads) k_bin(const int64_t* __restrict__ offsets, int B, int64_t P,
                                               int K, const int32_t* __restrict__ start_local,
                                               int force, int chunk_all, int fused_pool, int latency_events,
                                               int mid_cluster_events, int need_passes, Workspace ws) {
  // a kernel launched after this one as a programmatic dependent may start
  // now; it waits for this kernel's completion before it reads the lists
  asm volatile("griddepcontrol.launch_dependents;");
  __shared__ int cnt[kNumLists];
  __shared__ int hist[kNumSchedules][kBins];
  __shared__ int n_fps, n_mid, n_warp;
  __shared__ int s_n[kBinCache];              // event sizes (-1 for events that are neither FPS nor passthrough)
  __shared__ signed char s_cls[kBinCache];    // event classes, so later passes need no global re-reads
  for (int i = threadIdx.x; i < kNumSchedules * kBins; i += blockDim.x) (&hist[0][0])[i] = 0;
  if (threadIdx.x < kNumLists) cnt[threadIdx.x] = 0;
  if (threadIdx.x < 8) ws.hdr->next_item[threadIdx.x] = 0;
  if (threadIdx.x == 0) {
    ws.hdr->status = 0;
    ws.hdr->detail = 0;
    n_fps = 0;
    n_mid = 0;
    n_warp = 0;
  }
  __syncthreads();
  // pass 1: classify and count FPS events (four events per thread in flight;
  // counts kept per thread and added once per warp after the loop), and
  // histogram their sizes under the schedule they get when neither the
  // few-events nor the few-mid-size rule applies (pass 2 redoes it if one does)
  constexpr int U = 4;
  int my_fps = 0, my_mid = 0, my_warp = 0;
  auto plain_schedule_of = [&](int n) {
    int q = n <= kWarpCap ? 0 : (n <= kCtaCap ? 1 : (n <= kCtaSmemCap ? 2 : (n <= kCluster8Cap ? 3 : 4)));
    if (force > q) q = force > 4 ? 4 : force;
    return q;
  };
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
            ++my_fps;
            if (n > kCtaCap && n <= kCtaSmemCap) ++my_mid;
            const int q = plain_schedule_of((int)n);
            if (q == 0) ++my_warp;
            atomicAdd(&hist[q][min((int)n >> sched_shift(q), kBins - 1)], 1);
          }
        }
      }
      ws.cls[b] = cls;
      if (b < kBinCache) {
        s_n[b] = cls == kClsFps || cls == kClsPass ? (int)n : -1;
        s_cls[b] = (signed char)cls;
      }
    }
  }
  my_fps = __reduce_add_sync(kFull, my_fps);
  my_mid = __reduce_add_sync(kFull, my_mid);
  my_warp = __reduce_add_sync(kFull, my_warp);
  if ((threadIdx.x & 31) == 0) {
    if (my_fps) atomicAdd(&n_fps, my_fps);
    if (my_mid) atomicAdd(&n_mid, my_mid);
    if (my_warp) atomicAdd(&n_warp, my_warp);
  }
  __syncthreads();
  const bool few = n_fps <= latency_events;
  // few mid-size events: an 8-CTA cluster each (one pair per thread, the
  // step bound by the cluster exchange) instead of one CTA reading 10+
  // pairs per thread from shared memory; only under automatic scheduling
  const bool few_mid = force < 0 && n_mid <= mid_cluster_events;
  auto schedule_of = [&](int n) {
    int q = n <= kWarpCap ? 0 : (n <= kCtaCap ? 1 : (n <= kCtaSmemCap ? 2 : (n <= kCluster8Cap ? 3 : 4)));
    if (q == 0 && few) q = 1;  // few events: lower latency per step on a whole CTA
    if (q == 2 && few_mid) q = 3;
    if (force > q) q = force > 4 ? 4 : force;
    return q;
  };
  auto size_of = [&](int b) { return b < kBinCache ? s_n[b] : (int)(offsets[b + 1] - offsets[b]); };
  auto cls_of = [&](int b) { return b < kBinCache ? (int)s_cls[b] : ws.cls[b]; };
  // pass 2 (only when a rule above moves events): size histogram per schedule
  if ((few && n_warp > 0) || (few_mid && n_mid > 0)) {
    for (int i = threadIdx.x; i < kNumSchedules * kBins; i += blockDim.x) (&hist[0][0])[i] = 0;
    __syncthreads();
    for (int b = threadIdx.x; b < B; b += blockDim.x) {
      if (cls_of(b) != kClsFps) continue;
      const int n = size_of(b);
      const int q = schedule_of(n);
      atomicAdd(&hist[q][min(n >> sched_shift(q), kBins - 1)], 1);
    }
    __syncthreads();
  }
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
  // pass 3: scatter into the sorted lists; FPS slots, pooling items and
  // accumulator slots.  Each 1024-event round reserves its slots with one
  // CTA scan of the four counts packed into 64 bits (FPS slot 12 bits, pooled
  // event 12, replica slots 16, pool chunks 20: a round's totals fit), and
  // the warps write the pooling items cooperatively.
  __shared__ unsigned long long s_tmp64[32];
  int c_fps = 0, c_events = 0, c_slots = 0, c_chunks = 0;
  // Without Lloyd, assignment passes or any event pooled outside its FPS
  // kernel, nothing reads the slots and items: the lists alone are written.
  bool need_items = need_passes != 0;
  for (int q = 0; q < kNumSchedules; ++q)
    if (cnt[q] > 0 && !((fused_pool >> q) & 1)) need_items = true;
  if (!need_items) {
    for (int b = threadIdx.x; b < B; b += blockDim.x) {
      if (cls_of(b) != kClsFps) continue;
      const int n = size_of(b);
      const int q = schedule_of(n);
      int* list = q == 0 ? ws.list_warp
                         : (q == 1 ? ws.list_cta
                                   : (q == 2 ? ws.list_cta_smem : (q == 3 ? ws.list_cluster8 : ws.list_cluster16)));
      list[atomicAdd(&hist[q][min(n >> sched_shift(q), kBins - 1)], 1)] = b;
    }
    c_fps = n_fps;
  }
  for (int b0 = 0; need_items && b0 < B; b0 += blockDim.x) {
    const int b = b0 + threadIdx.x;
    const int cls = b < B ? cls_of(b) : kClsSkip;
    int n = 0;
    if (cls == kClsFps || cls == kClsPass) n = size_of(b);
    const int q = cls == kClsFps ? schedule_of(n) : 0;
    if (cls == kClsFps) {
      int* list = q == 0 ? ws.list_warp
                         : (q == 1 ? ws.list_cta
                                   : (q == 2 ? ws.list_cta_smem : (q == 3 ? ws.list_cluster8 : ws.list_cluster16)));
      list[atomicAdd(&hist[q][min(n >> sched_shift(q), kBins - 1)], 1)] = b;
    }
    // pooling items (passthrough events of fps_tokenize are written directly;
    // events of schedules that pool in place are left out)
    const bool pooled_here = (cls == kClsFps && !((fused_pool >> q) & 1)) || (chunk_all && cls == kClsPass);
    const int npc = pooled_here ? (n + kPoolChunk - 1) / kPoolChunk : 0;
    const int nrep = npc > 1 ? min(kPoolReplicas, npc) : 0;
    const unsigned long long v = (unsigned long long)npc | ((unsigned long long)nrep << 20) |
                                 ((unsigned long long)(npc > 1 ? 1 : 0) << 36) |
                                 ((unsigned long long)(cls == kClsFps ? 1 : 0) << 48);
    unsigned long long tot;
    const unsigned long long pre = cta_exclusive_scan64(v, s_tmp64, tot);
    const int pbase = c_chunks + (int)(pre & 0xFFFFFull);
    const int pslot = c_slots + (int)((pre >> 20) & 0xFFFFull);
    const int pev = c_events + (int)((pre >> 36) & 0xFFFull);
    const int fslot = c_fps + (int)((pre >> 48) & 0xFFFull);
    warp_fill_items(ws.pool_chunks, pbase, npc, b, 1);
    if (npc > 1) ws.pool_event[pev] = b;
    if (b < B) {
      ws.fps_slot[b] = cls == kClsFps ? fslot : -1;
      ws.pool_slot[b] = npc > 1 ? pslot : -1;
    }
    c_chunks += (int)(tot & 0xFFFFFull);
    c_slots += (int)((tot >> 20) & 0xFFFFull);
    c_events += (int)((tot >> 36) & 0xFFFull);
    c_fps += (int)((tot >> 48) & 0xFFFull);
  }
  if (threadIdx.x == 0) {
    cnt[kListFps] = c_fps;
    cnt[kListPoolChunks] = c_chunks;
    cnt[kListPoolSlots] = c_slots;
    cnt[kListPoolEvents] = c_events;
  }

  __syncthreads();
  // pass 4 (need_passes): the nearest-centroid passes of the chunked events (FPS events,
  // and the passthrough ones with chunk_all) in batch order: event b with n_b
  // points contributes passes (b, 0), (b, kPass), ... -- ceil(n_b / kPass)
  // of them, consecutive -- so that a CTA given a contiguous range of passes
  // mostly stays on one event.
  __shared__ int s_tmp[32];
  int carry = 0;
  for (int b0 = 0; need_passes && b0 < B; b0 += blockDim.x) {
    const int b = b0 + threadIdx.x;
    int n = 0;
    if (b < B) {
      const int cls = cls_of(b);
      if (cls == kClsFps || (chunk_all && cls == kClsPass)) n = size_of(b);
    }
    const int np = (n + kPass - 1) / kPass;
    int tot;
    const int base = carry + cta_exclusive_scan(np, s_tmp, tot);
    warp_fill_items(ws.passes, base, np, b, kPass);
    carry += tot;
  }
  if (threadIdx.x == 0) cnt[kListChunks] = carry;
  __syncthreads();
  if (threadIdx.x < kNumLists) ws.hdr->n_items[threadIdx.x] = cnt[threadIdx.x];
}

cudaError_t launch_bin(const Problem& pb, const Workspace& ws, int chunk_all, cudaStream_t s) {
  const DeviceInfo& di = device_info();
  count_launch();
  const int need_passes = chunk_all || pb.lloyd_iters > 0;
  k_bin<<<1, kBinThreads, 0, s>>>(pb.offsets, pb.B, pb.P, pb.K, pb.start_local, pb.force_schedule, chunk_all,
                           pb.fused_pool, kLatencyEventsPerSm * di.sm_count, di.sm_count / 8, need_passes, ws);
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
    const float* fe = pb.feats + off * F;
    float* outp = pb.pooled + (int64_t)b * K * F;
    const int nf = n * F;
    // both rows' loads of a round are issued before its stores, so that an
    // event costs about one memory round trip (K = 128, F <= 6: one round)
    constexpr int R = 24;  // elements per lane and row per round
    const int tc = K * 4, tp = K * F;
    for (int r0 = 0; r0 < tc || r0 < tp; r0 += 32 * R) {
      float vc[R], vp[R];
#pragma unroll
      for (int u = 0; u < R; ++u) {
        const int e = r0 + lane + 32 * u;
        vc[u] = e < nc ? cf[e] : 0.f;
        vp[u] = e < nf ? fe[e] : 0.f;
      }
#pragma unroll
      for (int u = 0; u < R; ++u) {
        const int e = r0 + lane + 32 * u;
        if (e < tc) outc[e] = vc[u];
        if (e < tp) outp[e] = vp[u];
      }
    }
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
  int* lab;    // [chunk] token of every point
  int* perm;   // [chunk] point of every sorted position
  int* slab;   // [chunk] token of every sorted position
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
      // chunk c adds into replica c % nrep: fewer updates per address
      const int ps = ws.pool_slot[b] + it.y % min(kPoolReplicas, nch);
      double* gacc = ws.pool_acc + (int64_t)ps * K * F;
      int* gcnt = ws.pool_cnt + (int64_t)ps * K;
      if (tid < K && cj) {  // reductions only; k_pool_finalize forms the means
        for (int f = 0; f < F; ++f) atomicAdd(&gacc[tid * F + f], acc[tid * F + f]);
        atomicAdd(&gcnt[tid], cj);
      }
    }
    __syncthreads();
  }
}

// Means of the events pooled over several chunks, from the float64 sums and
// counts of their accumulator replicas in global memory: one thread per
// (event, token), the replica loads of a value issued together.
__global__ void __launch_bounds__(256) k_pool_finalize(const int64_t* __restrict__ offsets,
                                                       float* __restrict__ pooled, int32_t* __restrict__ counts,
                                                       int K, int F, Workspace ws) {
  const int64_t total = (int64_t)ws.hdr->n_items[kListPoolEvents] * K;
  for (int64_t t = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; t < total; t += (int64_t)gridDim.x * blockDim.x) {
    const int e = (int)(t / K), j = (int)(t - (int64_t)e * K);
    const int b = ws.pool_event[e];
    const int ps = ws.pool_slot[b];
    const int n = (int)(offsets[b + 1] - offsets[b]);
    const int nrep = min(kPoolReplicas, (n + kPoolChunk - 1) / kPoolChunk);
    int c = 0;
#pragma unroll
    for (int r = 0; r < kPoolReplicas; ++r)
      if (r < nrep) c += ws.pool_cnt[(int64_t)(ps + r) * K + j];
    float* prow = pooled + ((int64_t)b * K + j) * F;
    for (int f = 0; f < F; ++f) {
      double sum = 0.0;
#pragma unroll
      for (int r = 0; r < kPoolReplicas; ++r)
        if (r < nrep) sum += ws.pool_acc[((int64_t)(ps + r) * K + j) * F + f];
      prow[f] = c ? (float)(sum / (double)c) : 0.f;
    }
    counts[(int64_t)b * K + j] = c;
  }
}

// Clears the pooling accumulator slots the binning kernel handed out.
__global__ void __launch_bounds__(256) k_pool_clear(int K, int F, Workspace ws) {
  const int64_t ns = ws.hdr->n_items[kListPoolSlots];
  const int64_t na = ns * K * F, nc = ns * K;
  const int64_t stride = (int64_t)gridDim.x * blockDim.x;
  for (int64_t e = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; e < na; e += stride) ws.pool_acc[e] = 0.0;
  for (int64_t e = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; e < nc; e += stride) ws.pool_cnt[e] = 0;
}

cudaError_t launch_pool_clear(const Problem& pb, const Workspace& ws, cudaStream_t s) {
  const DeviceInfo& di = device_info();
  count_launch();
  k_pool_clear<<<di.sm_count * 2, 256, 0, s>>>(pb.K, pb.F, ws);
  return cudaGetLastError();
}

static size_t pool_smem_bytes(int K, int F) {
  return sort_smem_bytes(kPoolChunk) + (size_t)K * F * sizeof(double) +
         (F <= kStageMaxF ? (size_t)kPoolChunk * F * sizeof(float) : 0);
}

cudaError_t launch_pool_voronoi(const float* feats, int F, const int64_t* offsets, int B, int K,
                                const int32_t* labels, float* pooled, int32_t* counts,
                                const Workspace& ws, cudaStream_t s) {
  const DeviceInfo& di = device_info();
  count_launch();
  k_pool_voronoi<<<di.sm_count * 8, 256, pool_smem_bytes(K, F), s>>>(feats, F, offsets, K, labels, pooled, counts,
                                                                     ws);
  cudaError_t e = cudaGetLastError();
  if (e) return e;
  return launch_pool_finalize(offsets, K, F, pooled, counts, ws, s);
}

cudaError_t launch_pool_finalize(const int64_t* offsets, int K, int F, float* pooled, int32_t* counts,
                                 const Workspace& ws, cudaStream_t s) {
  const DeviceInfo& di = device_info();
  count_launch();
  k_pool_finalize<<<di.sm_count * 2, 256, 0, s>>>(offsets, pooled, counts, K, F, ws);
  return cudaGetLastError();
}

// ------------------------------------------------------------------ nearest centroid

// Centroid slots padded to a whole number of pairs; the pad holds +inf
// coordinates, whose distance to any finite point is +inf.
__host__ __device__ constexpr int pad_pairs(int nv) { return (nv + 1) & ~1; }

__device__ __forceinline__ void load_cents_padded(const float4* __restrict__ c, int nv, Cent2* s, float4 w) {
  const float inf = __int_as_float(0x7f800000);
  for (int j = threadIdx.x; j < pad_pairs(nv); j += blockDim.x)
    s[j] = cent2(j < nv ? scale4(c[j], w) : make_float4(inf, inf, inf, inf));
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
                                              const Cent2* __restrict__ cs, int ng, float4 w, Emit emit) {
  const int tid = threadIdx.x;
#pragma unroll 1
  for (int q = 0; q < NPASS; ++q) {
    uint64_t X[PR], Y[PR], Z[PR], W[PR];
#pragma unroll
    for (int p = 0; p < PR; ++p) {
      const int ia = tid + (2 * PR * q + 2 * p) * T, ib = ia + T;
      float4 a = make_float4(0.f, 0.f, 0.f, 0.f), c = a;
      if (ia < npts) a = scale4(ldg4(pts + ia), w);
      if (ib < npts) c = scale4(ldg4(pts + ib), w);
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

constexpr int kNearestPairs = 2;  // pairs per thread: with two centroids in flight, 8 distance chains
static_assert(2 * kNearestPairs * 256 == kPass, "one nearest pass covers kPass points with 256 threads");

// The Lloyd and assignment kernels run the pass list: CTA g takes the
// contiguous range of ceil(Q / grid) passes starting at g ceil(Q / grid)
// (Q passes in all), so that every CTA does the same number of equal-cost
// passes and moves to a new event only where the list does.
__device__ __forceinline__ void pass_range(const Workspace& ws, int& q0, int& q1) {
  const int Q = ws.hdr->n_items[kListChunks];
  const int per = (Q + gridDim.x - 1) / gridDim.x;
  q0 = min(Q, blockIdx.x * per);
  q1 = min(Q, q0 + per);
}

// Standalone nearest-centroid assignment.
constexpr int kAssignThreads = 256;

__global__ void __launch_bounds__(kAssignThreads, kPassCtasPerSm) k_assign(const float4* __restrict__ coords,
                                                              const int64_t* __restrict__ offsets, int K,
                                                              const float4* __restrict__ centroids,
                                                              const int32_t* __restrict__ valid,
                                                              int32_t* __restrict__ token_id, Workspace ws,
                                                              float4 w) {
  constexpr int T = kAssignThreads;
  extern __shared__ Cent2 s_cent[];  // [pad_pairs(K)]
  int q0, q1;
  pass_range(ws, q0, q1);
  int cur = -1, nv = 0;
  for (int q = q0; q < q1; ++q) {
    const int2 it = ws.passes[q];
    const int b = it.x, i0 = it.y;
    const int64_t off = offsets[b];
    const int n = (int)(offsets[b + 1] - off);
    if (b != cur) {  // uniform: every thread reads the same pass
      __syncthreads();
      nv = valid ? valid[b] : min(n, K);
      if (nv < 0 || nv > K) {
        record_error(ws.hdr, kDevBadToken);
        nv = 0;
      }
      load_cents_padded(centroids + (int64_t)b * K, nv, s_cent, w);
      __syncthreads();
      cur = b;
    }
    int32_t* out = token_id + off + i0;
    const int v = nv;
    chunk_nearest<kNearestPairs, 1, T>(coords + off + i0, min(n - i0, kPass), s_cent, pad_pairs(nv) / 2, w,
                                       [&](int li, int l) { out[li] = v > 0 ? l : -1; });
  }
}

// ------------------------------------------------------------------ Lloyd

__device__ __forceinline__ float charge_of(const float* fe, int F, int charge_col, int i) {
  return charge_col < 0 ? 1.0f : __ldg(fe + (int64_t)i * F + charge_col);
}

constexpr int kLloydThreads = 256;
constexpr int kLloydPts = kPass / kLloydThreads;  // points per thread
static_assert(kLloydPts == 2 * kNearestPairs, "chunk_nearest covers a pass");

// Shared memory of the cell-sum kernel: the counting sort of one piece by
// label, its points and charges, and the per-token sums.
struct LloydSmem {
  int* perm;     // [kPass]
  int* slab;     // [kPass]
  int* cnt;      // [256]
  int* start;    // [256]
  int* cur;      // [256]
  float4* s_p;   // [kPass]
  float* s_q;    // [kPass]
  double* acc;   // [K * 5]
};
static size_t lloyd_smem_bytes(int K) {
  return (size_t)(2 * kPass + 3 * 256) * sizeof(int) + (size_t)kPass * (sizeof(float4) + sizeof(float)) +
         (size_t)K * 5 * sizeof(double);
}
// The update kernel keeps its centroids after that region, 16-byte aligned.
__host__ __device__ constexpr size_t lloyd_cent_offset(int K) {
  return ((size_t)(2 * kPass + 3 * 256) * sizeof(int) + (size_t)kPass * (sizeof(float4) + sizeof(float)) +
          (size_t)K * 5 * sizeof(double) + 15) & ~(size_t)15;
}
__device__ __forceinline__ LloydSmem lloyd_smem(char* base) {
  LloydSmem m;
  m.perm = reinterpret_cast<int*>(base);
  m.slab = m.perm + kPass;
  m.cnt = m.slab + kPass;
  m.start = m.cnt + 256;
  m.cur = m.start + 256;
  m.s_p = reinterpret_cast<float4*>(m.cur + 256);
  m.s_q = reinterpret_cast<float*>(m.s_p + kPass);
  m.acc = reinterpret_cast<double*>(m.s_q + kPass);
  return m;
}

// Cell sums W_j = sum q and S_j = sum q p (float64) of one piece -- points
// tid + r T, r < kLloydPts, of `pts`, labels `lab`, charges from `fe` --
// added into out[K][5]: all loads issued first, a counting sort by label in
// shared memory, balanced per-token sums, one float64 reduction per value of
// every non-empty cell.  Labels outside [0, K) are reported and left out.
__device__ __forceinline__ void lloyd_piece_sums(const float4* __restrict__ pts, const float* __restrict__ fe,
                                        int F, int charge_col, const int32_t* lab, int npts, int K,
                                                 const LloydSmem& sm, double* __restrict__ out, WsHeader* hdr) {
  constexpr int T = kLloydThreads;
  const int tid = threadIdx.x;
  for (int j = tid; j < K; j += T) sm.cnt[j] = 0;
  for (int e = tid; e < K * 5; e += T) sm.acc[e] = 0.0;
  __syncthreads();
  int l[kLloydPts];
  float4 p[kLloydPts];
  float q[kLloydPts];
#pragma unroll
  for (int r = 0; r < kLloydPts; ++r) {
    const int li = tid + r * T;
    l[r] = -1;
    if (li < npts) {
      l[r] = lab[li];
      p[r] = ldg4(pts + li);
      q[r] = charge_of(fe, F, charge_col, li);
    }
  }
#pragma unroll
  for (int r = 0; r < kLloydPts; ++r) {
    const int li = tid + r * T;
    if (li < npts) {
      if ((unsigned)l[r] >= (unsigned)K) {
        record_error(hdr, kDevBadToken);
        l[r] = -1;
        continue;
      }
      sm.s_p[li] = p[r];
      sm.s_q[li] = q[r];
      atomicAdd(&sm.cnt[l[r]], 1);
    }
  }
  __syncthreads();
  if (tid < 32) count_scan(sm.cnt, sm.start, sm.cur, K, tid);
  __syncthreads();
#pragma unroll
  for (int r = 0; r < kLloydPts; ++r) {
    if (l[r] >= 0) {
      const int pos = atomicAdd(&sm.cur[l[r]], 1);
      sm.perm[pos] = tid + r * T;
      sm.slab[pos] = l[r];
    }
  }
  __syncthreads();
  const int nsorted = sm.start[K - 1] + sm.cnt[K - 1];
  segment_sums(sm.perm, sm.slab, nsorted, 5, 0, 5, sm.acc, tid, T, [&](int i, int v) {
    const double qq = (double)sm.s_q[i];
    if (v == 0) return qq;
    const float4 pp = sm.s_p[i];
    return qq * (double)(v == 1 ? pp.x : (v == 2 ? pp.y : (v == 3 ? pp.z : pp.w)));
  });
  __syncthreads();
  for (int e = tid; e < K * 5; e += T)
    if (sm.cnt[e / 5]) atomicAdd(&out[e], sm.acc[e]);
}

// Where the last Lloyd iteration writes the token means (Voronoi mode of
// the tokenizer): feats == nullptr when it does not pool.
struct LloydPool {
  const float* feats;
  float* pooled;
  int32_t* counts;
};

// Token means of one pass in the last Lloyd iteration: the pass's points
// sorted by their final label, float64 sums of their feature rows per token
// in groups of up to 5 features (the accumulator of the cell sums), then the
// means and counts of an event pooled in one piece written directly
// (gacc == nullptr), or the sums and counts added into the event's
// accumulator replica, whose means k_pool_finalize forms.  Each thread reads
// back the labels it wrote for its own points.
__device__ __forceinline__ void lloyd_piece_pool(const float* __restrict__ fe, int F, const int32_t* lab, int npts,
                                                 int K, const LloydSmem& sm, float* __restrict__ prow,
                                                 int32_t* __restrict__ crow, double* __restrict__ gacc,
                                                 int* __restrict__ gcnt) {
  constexpr int T = kLloydThreads;
  const int tid = threadIdx.x;
  for (int j = tid; j < K; j += T) sm.cnt[j] = 0;
  __syncthreads();
  int l[kLloydPts];
#pragma unroll
  for (int r = 0; r < kLloydPts; ++r) {
    const int li = tid + r * T;
    l[r] = li < npts ? lab[li] : -1;
    if ((unsigned)l[r] >= (unsigned)K) l[r] = -1;  // never: the labels were just written
    if (l[r] >= 0) atomicAdd(&sm.cnt[l[r]], 1);
  }
  __syncthreads();
  if (tid < 32) count_scan(sm.cnt, sm.start, sm.cur, K, tid);
  __syncthreads();
#pragma unroll
  for (int r = 0; r < kLloydPts; ++r) {
    if (l[r] >= 0) {
      const int pos = atomicAdd(&sm.cur[l[r]], 1);
      sm.perm[pos] = tid + r * T;
      sm.slab[pos] = l[r];
    }
  }
  __syncthreads();
  const int nsorted = sm.start[K - 1] + sm.cnt[K - 1];
  for (int g0 = 0; g0 < F; g0 += 5) {
    const int V = min(5, F - g0);
    for (int e = tid; e < K * 5; e += T) sm.acc[e] = 0.0;
    __syncthreads();
    segment_sums(sm.perm, sm.slab, nsorted, V, 0, 5, sm.acc, tid, T,
                 [&](int i, int v) { return (double)__ldg(fe + (int64_t)i * F + g0 + v); });
    __syncthreads();
    for (int e = tid; e < K * 5; e += T) {
      const int j = e / 5, v = e - 5 * j;
      if (v >= V) continue;
      const int c = sm.cnt[j];
      if (!gacc) prow[j * F + g0 + v] = c ? (float)(sm.acc[e] / (double)c) : 0.f;
      else if (c) atomicAdd(&gacc[j * F + g0 + v], sm.acc[e]);
    }
    if (g0 == 0)
      for (int j = tid; j < K; j += T) {
        if (!gacc) crow[j] = sm.cnt[j];
        else if (sm.cnt[j]) atomicAdd(&gcnt[j], sm.cnt[j]);
      }
    __syncthreads();
  }
}

// Cell sums of the current labels.
__global__ void __launch_bounds__(kLloydThreads, kPassCtasPerSm) k_lloyd_sums(const float4* __restrict__ coords,
                                                                 const float* __restrict__ feats, int F,
                                                                 int charge_col,
                                                                 const int64_t* __restrict__ offsets, int K,
                                                                 const int32_t* __restrict__ labels,
                                                                 Workspace ws, double* __restrict__ out) {
  extern __shared__ __align__(16) char smem_c[];
  const LloydSmem sm = lloyd_smem(smem_c);
  int q0, q1;
  pass_range(ws, q0, q1);
  for (int q = q0; q < q1; ++q) {
    const int2 it = ws.passes[q];
    const int b = it.x, i0 = it.y;
    const int fs = ws.fps_slot[b];
    if (fs < 0) continue;  // uniform across the CTA
    const int64_t off = offsets[b] + i0;
    const int npts = min((int)(offsets[b + 1] - offsets[b]) - i0, kPass);
    lloyd_piece_sums(coords + off, feats ? feats + off * F : nullptr, F, charge_col, labels + off, npts, K, sm,
                     out + (int64_t)fs * K * 5, ws.hdr);
    __syncthreads();
  }
}

// One Lloyd iteration: the centroids from the cell sums `in` (an empty cell
// or a zero weight keeps its centroid), the nearest of them for every point
// of the pass and, unless this is the last iteration (next == nullptr), the
// pass's cell sums of the new labels added into `next`.  Also clears `clear`,
// the buffer the following iteration accumulates into.
__global__ void __launch_bounds__(kLloydThreads, kPassCtasPerSm) k_lloyd_step(const float4* __restrict__ coords,
                                                                 const float* __restrict__ feats, int F,
                                                                 int charge_col,
                                                                 const int64_t* __restrict__ offsets, int K,
                                                                 int32_t* __restrict__ labels,
                                                                 float4* __restrict__ centroids, Workspace ws,
                                                                 const double* __restrict__ in,
                                                                 double* __restrict__ next,
                                                                 double* __restrict__ clear, int64_t clear_n,
                                                                 float4 w, LloydPool pool) {
  constexpr int T = kLloydThreads;
  extern __shared__ __align__(16) char smem_c[];
  const LloydSmem sm = lloyd_smem(smem_c);
  Cent2* s_cent = reinterpret_cast<Cent2*>(smem_c + lloyd_cent_offset(K));  // [pad_pairs(K)]
  const int tid = threadIdx.x;
  for (int64_t e = (int64_t)blockIdx.x * T + tid; e < clear_n; e += (int64_t)gridDim.x * T) clear[e] = 0.0;
  int q0, q1;
  pass_range(ws, q0, q1);
  int cur = -1;
  for (int q = q0; q < q1; ++q) {
    const int2 it = ws.passes[q];
    const int b = it.x, i0 = it.y;
    const int fs = ws.fps_slot[b];
    if (fs < 0) continue;  // uniform across the CTA
    if (b != cur) {  // the event's updated centroids
      __syncthreads();
      const double* sb = in + (int64_t)fs * K * 5;
      const bool writer = i0 == 0;  // the event's first pass writes them back (all passes compute the same)
      for (int j = tid; j < K; j += T) {
        const double W = __ldcg(&sb[j * 5]);
        float4 c = centroids[(int64_t)b * K + j];
        if (W > 0.0) {
          c.x = (float)(__ldcg(&sb[j * 5 + 1]) / W);
          c.y = (float)(__ldcg(&sb[j * 5 + 2]) / W);
          c.z = (float)(__ldcg(&sb[j * 5 + 3]) / W);
          c.w = (float)(__ldcg(&sb[j * 5 + 4]) / W);
        }
        s_cent[j] = cent2(scale4(c, w));  // the means stay in the caller's units
        if (writer) centroids[(int64_t)b * K + j] = c;
      }
      if (tid == 0 && (K & 1)) {
        const float inf = __int_as_float(0x7f800000);
        s_cent[K] = cent2(make_float4(inf, inf, inf, inf));
      }
      __syncthreads();
      cur = b;
    }
    const int64_t off = offsets[b] + i0;
    const int npts = min((int)(offsets[b + 1] - offsets[b]) - i0, kPass);
    int32_t* lab_out = labels + off;
    chunk_nearest<kNearestPairs, 1, T>(coords + off, npts, s_cent, pad_pairs(K) / 2, w,
                                       [&](int li, int l) { lab_out[li] = l; });
    if (next) {  // this thread's own labels, read back
      lloyd_piece_sums(coords + off, feats ? feats + off * F : nullptr, F, charge_col, lab_out, npts, K, sm,
                       next + (int64_t)fs * K * 5, ws.hdr);
      __syncthreads();  // the next pass re-zeroes the sums
    } else if (pool.feats) {  // the last iteration: the pass's token means (replica piece % nrep)
      const int ps = ws.pool_slot[b];
      double* gacc = nullptr;
      int* gcnt = nullptr;
      if (ps >= 0) {
        const int n = (int)(offsets[b + 1] - offsets[b]);
        const int nrep = min(kPoolReplicas, (n + kPoolChunk - 1) / kPoolChunk);
        const int slot = ps + (i0 / kPass) % nrep;
        gacc = ws.pool_acc + (int64_t)slot * K * F;
        gcnt = ws.pool_cnt + (int64_t)slot * K;
      }
      lloyd_piece_pool(pool.feats + off * F, F, lab_out, npts, K, sm, pool.pooled + (int64_t)b * K * F,
                       pool.counts + (int64_t)b * K, gacc, gcnt);
      __syncthreads();
    }
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
  const int grid = di.sm_count * kPassCtasPerSm;
  cudaError_t e;
  count_launch();
  k_lloyd_sums<<<grid, kLloydThreads, lloyd_smem_bytes(K), s>>>(pb.coords, feats, pb.F, pb.charge_col, pb.offsets,
                                                                 K, labels, ws, ws.lloyd[0]);
  if ((e = cudaGetLastError())) return e;
  const size_t sm_step = lloyd_cent_offset(K) + (size_t)pad_pairs(K) * sizeof(Cent2);
  for (int t = 0; t < pb.lloyd_iters; ++t) {
    const bool last = t == pb.lloyd_iters - 1;
    double* clear = (t + 1 < pb.lloyd_iters - 1) ? ws.lloyd[(t + 2) % 3] : nullptr;
    count_launch();
    const LloydPool pool = {last && lloyd_pools(pb) ? pb.feats : nullptr, pb.pooled, pb.counts};
    k_lloyd_step<<<grid, kLloydThreads, sm_step, s>>>(pb.coords, feats, pb.F, pb.charge_col, pb.offsets, K, labels,
                                                      pb.centroids, ws, ws.lloyd[t % 3],
                                                      last ? nullptr : ws.lloyd[(t + 1) % 3], clear,
                                                      clear ? (int64_t)ws.fps_slots * per : 0, pb.w, pool);
    if ((e = cudaGetLastError())) return e;
  }
  return cudaSuccess;
}

// Shared-memory limits of the auxiliary kernels, set once per device for the
// largest K and F the ABI accepts.
cudaError_t prepare_aux_kernels() {
  cudaError_t e;
  if ((e = cudaFuncSetAttribute(k_lloyd_sums, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                (int)lloyd_smem_bytes(256))))
    return e;
  if ((e = cudaFuncSetAttribute(k_lloyd_step, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                (int)(lloyd_cent_offset(256) + (size_t)pad_pairs(256) * sizeof(Cent2)))))
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


// Row order of the kNN kernel inside fps_tokenize: the FPS events of the
// binning kernel's schedule lists, largest schedule first (each list is
// sorted by decreasing size), so that the longest rows start first.
struct KnnOrder {
  const int* list[kNumSchedules];  // the lists, largest schedule first
  int count_id[kNumSchedules];     // their n_items entries
  int nlists;                      // 0: every event of the batch, in batch order
};

__device__ __forceinline__ int ordered_event(const WsHeader* hdr, const KnnOrder& o, int e) {
#pragma unroll
  for (int q = 0; q < kNumSchedules; ++q) {
    if (q >= o.nlists) break;
    const int nq = hdr->n_items[o.count_id[q]];
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
                                             KnnOrder ord, WsHeader* hdr, float4 w, int scaled) {
  const int lane = threadIdx.x & 31;
  const int gw = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int nw = (gridDim.x * blockDim.x) >> 5;
  __shared__ uint64_t s_stage[256 / 32][32];  // per-warp staging slots (k <= 32)
  uint64_t* stage = s_stage[threadIdx.x >> 5];
  int n_ev = B;
  if (ord.nlists) {
    n_ev = 0;
    for (int q = 0; q < ord.nlists; ++q) n_ev += hdr->n_items[ord.count_id[q]];
  }
  const int64_t rows = (int64_t)n_ev * K;
  const int kq = (k - 1) >> 5, kl = (k - 1) & 31;
  for (int64_t r = gw; r < rows; r += nw) {
    const int e = (int)(r / K), j = (int)(r - (int64_t)e * K);
    const int b = ord.nlists ? ordered_event(hdr, ord, e) : e;
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
      const float4 c = scale4(centroids[orow], w);
      const float4* pts = coords + o0;
      uint64_t thr = ~0ull;
      int ns = 0;  // staged candidates (k <= 32)
      constexpr int U = 4;  // 32-point chunks loaded per iteration
      for (int base = 0; base < n; base += 32 * U) {
        float4 pt[U];
#pragma unroll
        for (int u = 0; u < U; ++u) {
          const int i = base + u * 32 + lane;
          pt[u] = i < n ? ldg4(pts + i) : make_float4(0.f, 0.f, 0.f, 0.f);
        }
        if (scaled) {  // uniform: unscaled calls skip the multiplies
#pragma unroll
          for (int u = 0; u < U; ++u) pt[u] = scale4(pt[u], w);
        }
#pragma unroll
        for (int u = 0; u < U; ++u) {
          const int i = base + u * 32 + lane;
          const uint64_t key =
              i < n ? (((uint64_t)__float_as_uint(dist1(pt[u], c)) << 32) | (uint32_t)i) : ~0ull;
          if constexpr (KPL == 1) {
            // candidates below the threshold go to the warp's staging slots; a
            // chunk that would overflow them first sorts the staged keys and
            // merges them into the list (refreshing the threshold)
            bool pass = key < thr;
            unsigned mask = __ballot_sync(kFull, pass);
            int cnt = __popc(mask);
            if (ns + cnt > 32) {
              __syncwarp();
              const uint64_t sv = lane < ns ? stage[lane] : ~0ull;
              L[0] = warp_merge64(L[0], warp_sort64(sv, lane), lane);
              thr = __shfl_sync(kFull, L[0], kl);
              ns = 0;
              pass = key < thr;
              mask = __ballot_sync(kFull, pass);
              cnt = __popc(mask);
              __syncwarp();
            }
            if (pass) stage[ns + __popc(mask & ((1u << lane) - 1u))] = key;
            ns += cnt;
          } else {
          unsigned mask = __ballot_sync(kFull, key < thr);
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
      if constexpr (KPL == 1) {
        if (ns > 0) {  // the last staged candidates
          __syncwarp();
          const uint64_t sv = lane < ns ? stage[lane] : ~0ull;
          L[0] = warp_merge64(L[0], warp_sort64(sv, lane), lane);
          __syncwarp();
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
                       cudaStream_t s, float4 w, int scaled, int only_schedule) {
  const DeviceInfo& di = device_info();
  // one block per 8 rows (one row per warp), not a persistent grid: short
  // blocks let the schedulers interleave the per-schedule kNN launches by
  // stream priority (rows past the device's count exit at once)
  const int64_t rows = (int64_t)B * K;
  int64_t blocks = (rows + 7) / 8;
  const int64_t cap = (int64_t)1 << 24;
  if (blocks > cap) blocks = cap;
  if (blocks < 1) blocks = 1;
  KnnOrder ord{};
  if (ws) {
    const int* lists[kNumSchedules] = {ws->list_warp, ws->list_cta, ws->list_cta_smem, ws->list_cluster8,
                                       ws->list_cluster16};
    for (int q = kNumSchedules - 1; q >= 0; --q) {
      if (only_schedule >= 0 && q != only_schedule) continue;
      ord.list[ord.nlists] = lists[q];
      ord.count_id[ord.nlists] = q;  // the schedule lists are n_items[0 .. kNumSchedules)
      ++ord.nlists;
    }
  }
  count_launch();
  if (k <= 32)
    k_knn<1><<<(int)blocks, 256, 0, s>>>(coords, offsets, B, centroids, valid_tokens, K, k, knn_idx,
                                         feats, F, pooled, counts, ord, hdr, w, scaled);
  else if (k <= 64)
    k_knn<2><<<(int)blocks, 256, 0, s>>>(coords, offsets, B, centroids, valid_tokens, K, k, knn_idx,
                                         feats, F, pooled, counts, ord, hdr, w, scaled);
  else
    k_knn<4><<<(int)blocks, 256, 0, s>>>(coords, offsets, B, centroids, valid_tokens, K, k, knn_idx,
                                         feats, F, pooled, counts, ord, hdr, w, scaled);
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
                          cudaStream_t s, float4 w) {
  const DeviceInfo& di = device_info();
  const size_t sm = (size_t)pad_pairs(K) * sizeof(Cent2);
  count_launch();
  k_assign<<<di.sm_count * kPassCtasPerSm, kAssignThreads, sm, s>>>(coords, offsets, K, centroids, valid_tokens,
                                                                token_id, ws, w);
  return cudaGetLastError();
}

}  // namespace fpstok
