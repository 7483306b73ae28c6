// Farthest point sampling fused with the Voronoi labels, five schedules.
//
// Tokenization per the Neptune README ("How it works", step 1): farthest-point
// sampling of every event down to K centroids with nearest-centroid (Voronoi)
// assignment of each pulse.  The loop for one event with N > K points:
//
//   c_0 = start;  dist_i = +inf
//   for s = 0 .. K-1:
//     for every point i: d = d(i, c_s); if d < dist_i: dist_i = d, label_i = s
//     if s < K-1: c_{s+1} = arg-max_i dist_i, lowest index on ties
//                 (when the maximum is 0, the lowest-index unselected point)
//
// Already-selected points have dist 0, so for a positive maximum the arg-max
// over all points equals the arg-max over unselected points; the zero case is
// resolved from a per-thread bit mask of selected slots.  The final pass with
// c_{K-1} only updates labels.  Because min() is exact and the strict '<'
// keeps the earliest slot, label_i equals the nearest centroid with the
// lowest slot on ties, i.e. the plain Voronoi assignment.
//
// Schedules (chosen per event by the binning kernel; they run concurrently,
// the block schedules on helper streams forked from the caller's stream):
//   warp        N <= 448     one warp per event, points in registers (lane l
//                            owns points l + 32 j); arg-max by two redux.sync.
//   CTA         N <= 2560    one 256-thread CTA per event, points in
//                            registers; warp winners exchanged through shared
//                            memory, one barrier per step.  Also takes the
//                            warp-class events when there are few events.
//   CTA-smem    N <= 12288   one 256-thread CTA per event, points in shared
//                            memory as packed f32x2 pairs.
//   cluster-8   N <= 98304   an 8-CTA cluster per event (same layout): warp 0
//   cluster-16  N <= 196608  of every CTA posts the CTA's winner into a slot
//                            of every CTA's shared memory with st.async, which
//                            signals that CTA's mbarrier; a bounded wait on it,
//                            no cluster barrier per step.
// Each event runs a step loop compiled for its exact number of point pairs
// (one dispatch per event; in the warp schedule an out-of-line function per
// pair count), and work items are claimed from a counter in decreasing size
// order so that the longest chains start first.  The warp and register-CTA
// schedules also pool their events' token means in place.
#include <cooperative_groups.h>

#include <mutex>

#include "common.cuh"
#include "internal.h"

namespace cg = cooperative_groups;

namespace fpstok {

__device__ __forceinline__ unsigned low_bits(int n) { return n >= 32 ? 0xffffffffu : ((1u << n) - 1u); }

// Dispatches CALL(N) for the compile-time N that equals the runtime np
// (N <= kMaxPairs).
#define FPS_CASE(N, CALL) \
  case N:                 \
    if constexpr ((N) <= kMaxPairs) { CALL(N); } break;
#define FPS_DISPATCH_7(np, CALL) \
  switch (np) { FPS_CASE(1, CALL) FPS_CASE(2, CALL) FPS_CASE(3, CALL) FPS_CASE(4, CALL) FPS_CASE(5, CALL) \
                FPS_CASE(6, CALL) FPS_CASE(7, CALL) default : break; }

// Where an FPS kernel writes the token means of the events it pools itself
// (no Lloyd follows): feats == nullptr means the pool kernel does it.
struct PoolOut {
  const float* feats;
  int F;
  float* pooled;
  int32_t* counts;
};

// Asks L2 to fetch the event's feature rows [lo, lo + bytes) while the FPS
// loop runs, so that the pooling at its end reads them from L2.  The range
// is shrunk inward to 16-byte boundaries (it never leaves the rows) and
// split into 16 KiB bulk prefetches, one per calling `part` < nparts.
__device__ __forceinline__ void prefetch_rows_l2(const float* lo, size_t bytes, int part, int nparts) {
  uintptr_t a = (reinterpret_cast<uintptr_t>(lo) + 15) & ~(uintptr_t)15;
  const uintptr_t end = (reinterpret_cast<uintptr_t>(lo) + bytes) & ~(uintptr_t)15;
  constexpr uintptr_t kPiece = 16384;
  for (uintptr_t p = a + (uintptr_t)part * kPiece; p < end; p += (uintptr_t)nparts * kPiece) {
    const uint32_t len = (uint32_t)((end - p) < kPiece ? (end - p) : kPiece);
    asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(p), "r"(len) : "memory");
  }
}

// Layout of the warp schedule's per-warp shared memory: the event's points
// (float4, the caller's units), then the list of chosen local indices (the
// step's centroid is recorded by one lane; positions and global indices are
// written once at the end).  The points region is reused by the fused
// pooling afterwards.
typedef float4 WarpPt;
constexpr int kWarpPtBytes = (int)sizeof(WarpPt);
constexpr int kWarpListInts = FPS_MAX_K_DEV;  // chosen local indices, one per step
// Shared memory of one warp: the event copy and the list, then room for the
// pooling's staged feature rows (the whole region is reused by it).
constexpr int kWarpRegionBytes = 15360;
static_assert(64 * kWarpPairs * kWarpPtBytes + kWarpListInts * 4 <= kWarpRegionBytes, "event copy and list fit");
static_assert(8 * FPS_MAX_K_DEV + 4 * kWarpCap <= kWarpRegionBytes, "one staged feature per pass fits");

// The packed centroid of a stored point (scaled per step when SCALED).
template <bool SCALED>
__device__ __forceinline__ Cent2 warp_pt_cent(const WarpPt& p, float4 w) {
  return cent2(SCALED ? scale4(p, w) : p);
}

// Running-min / label update of the two points of one packed pair.
__device__ __forceinline__ void relax2(uint64_t d, float& d0, float& d1, int& l0, int& l1, int s) {
  relax(lo2(d), d0, l0, s);
  relax(hi2(d), d1, l1, s);
}

// One FPS event on one warp, NP point pairs per lane (lane l owns points
// l + 32 j, slot j = 2 p + h of pair p and half h); SCALED: the per-axis
// scale is applied (a separate instantiation, so the common loop has no
// branch for it).
template <int NP, bool SCALED>
__device__ __noinline__ void warp_event(const float4* __restrict__ pts, int n, int c, int K, int64_t off,
                                           int lane, WarpPt* s_pts, int* s_c, int32_t* __restrict__ cidx,
                                           float4* __restrict__ cpos, int32_t* __restrict__ tok, int64_t b,
                                           const PoolOut& po, float4 w, int* claim_ctr, int claim_base,
                                           int& next) {
  if (po.feats && lane < 4) prefetch_rows_l2(po.feats + off * po.F, (size_t)n * po.F * sizeof(float), lane, 4);
  const uint64_t z2 = opaque_zero2();
  uint64_t X[NP], Y[NP], Z[NP], T[NP];
  float dist[2 * NP];
  int lab[2 * NP];
  unsigned empty = 0;  // bit j: slot j holds no point
#pragma unroll
  for (int p = 0; p < NP; ++p) {
    const int i0 = 64 * p + lane, i1 = i0 + 32;
    float4 a = make_float4(0.f, 0.f, 0.f, 0.f), b = a;
    if (i0 < n) a = ldg4(pts + i0);
    if (i1 < n) b = ldg4(pts + i1);
    if (i0 < n) s_pts[i0] = a;  // caller's units: centroid outputs (scaled per step when needed)
    if (i1 < n) s_pts[i1] = b;
    if (SCALED) {
      a = scale4(a, w);
      b = scale4(b, w);
    }
    X[p] = pack2(a.x, b.x);
    Y[p] = pack2(a.y, b.y);
    Z[p] = pack2(a.z, b.z);
    T[p] = pack2(a.w, b.w);
    if (i0 >= n) empty |= 1u << (2 * p);
    if (i1 >= n) empty |= 1u << (2 * p + 1);
  }
  auto reset = [&]() {
#pragma unroll
    for (int j = 0; j < 2 * NP; ++j) {
      dist[j] = (empty >> j) & 1u ? kEmptySlot : __int_as_float(0x7f800000);
      lab[j] = 0;
    }
  };
  // One step: update with c_s = c, then c = the arg-max (lowest index among
  // equal maxima); returns the maximum's key.
  auto step = [&](int s) -> int {
    if (lane == 0) s_c[s] = c;
    const Cent2 C = warp_pt_cent<SCALED>(s_pts[c], w);
    float pm[NP];
#pragma unroll
    for (int p = 0; p < NP; ++p) {
      const uint64_t d = dist2(X[p], Y[p], Z[p], T[p], C, z2);
      relax2(d, dist[2 * p], dist[2 * p + 1], lab[2 * p], lab[2 * p + 1], s);
      pm[p] = fmaxf(dist[2 * p], dist[2 * p + 1]);
    }
    const int M = __reduce_max_sync(kFull, fkey(lane_max<NP>(pm)));
    const int slot = lane_first_slot<NP>(pm, dist, M);  // lowest slot of this lane holding the maximum
    c = (int)__reduce_min_sync(kFull, slot < 0 ? 0xffffffffu : (unsigned)(slot * 32 + lane));
    return M;
  };
  reset();
  __syncwarp();
  // steps 0 .. K-2 without an exit test: a zero maximum (every unselected
  // point duplicates a chosen one, so the arg-max may return a chosen point)
  // is only recorded, and such an event is run again from the start below,
  // leaving at its first zero maximum.  The chosen index stays a point of the
  // event either way (empty slots never hold the maximum).
  const int c_first = c;
  bool zero = false;
  for (int s = 0; s < K - 1; ++s) zero |= step(s) == 0;
  int s = K - 1;
  if (zero) {
    reset();
    c = c_first;
    for (s = 0; s < K - 1; ++s)
      if (step(s) == 0) break;
  }
  // only duplicates of chosen points remain: each next centroid is the
  // lowest-index unselected point (steps s + 1 .. K - 2; step s's update is done)
  if (s < K - 1) {
    __syncwarp();
    unsigned taken = empty;
    for (int t = 0; t <= s; ++t) {
      const int ct = s_c[t];
      if ((ct & 31) == lane) taken |= 1u << (ct >> 5);
    }
    for (;;) {
      const unsigned free_slots = ~taken & low_bits(2 * NP);
      c = (int)__reduce_min_sync(kFull, free_slots ? (unsigned)((__ffs(free_slots) - 1) * 32 + lane) : 0xffffffffu);
      if ((c & 31) == lane) taken |= 1u << (c >> 5);
      if (++s == K - 1) break;
      if (lane == 0) s_c[s] = c;
      const Cent2 C = warp_pt_cent<SCALED>(s_pts[c], w);
#pragma unroll
      for (int p = 0; p < NP; ++p) {
        const uint64_t d = dist2(X[p], Y[p], Z[p], T[p], C, z2);
        relax2(d, dist[2 * p], dist[2 * p + 1], lab[2 * p], lab[2 * p + 1], s);
      }
    }
  }
  {  // step K-1: the last centroid only updates the labels
    if (lane == 0) s_c[K - 1] = c;
    const Cent2 C = warp_pt_cent<SCALED>(s_pts[c], w);
#pragma unroll
    for (int p = 0; p < NP; ++p) {
      const uint64_t d = dist2(X[p], Y[p], Z[p], T[p], C, z2);
      relax2(d, dist[2 * p], dist[2 * p + 1], lab[2 * p], lab[2 * p + 1], K - 1);
    }
  }
  // the next item is claimed here, so that the atomic's round trip overlaps the writes and the pooling below
  if (lane == 0) next = claim_base + atomicAdd(claim_ctr, 1);
  __syncwarp();
  for (int j = lane; j < K; j += 32) {  // the event's centroids, once
    const int cj = s_c[j];
    cidx[j] = (int32_t)(off + cj);
    cpos[j] = s_pts[cj];
  }
  if (tok) {
#pragma unroll
    for (int j = 0; j < 2 * NP; ++j) {
      const int i = j * 32 + lane;
      if (i < n) tok[i] = lab[j];
    }
  }
  if (po.feats) {
    // Token means.  Every point's rank inside its token (one shared atomic
    // each) and the token starts by a scan of the counts.  When the event's
    // whole feature block fits beside them, it is copied into shared memory
    // by asynchronous copies (16-byte pieces, in flight during the sort), and
    // lane t sums token t's rows, found through the sorted point list, in
    // float64.  Otherwise, per pass of at most 8 features, the lanes copy
    // their points' rows into shared memory in token order and lane t sums
    // token t's contiguous rows.
    const int F = po.F;
    __syncwarp();
    int* cnt = reinterpret_cast<int*>(s_pts);  // [K] counts, then [K] starts, then the rest
    int* start = cnt + K;
    const float* fe = po.feats + off * F;
    const int pad = (int)((reinterpret_cast<uintptr_t>(fe) >> 2) & 3);  // floats before a 16-byte boundary
    const int head = (4 - pad) & 3;
    const size_t list_bytes = ((size_t)(2 * K + n) * 4 + 15) & ~(size_t)15;
    const bool whole = list_bytes + (size_t)(pad + n * F) * 4 <= (size_t)kWarpRegionBytes;
    int* perm = start + K;                                                 // [n] points in token order
    float* sfb = reinterpret_cast<float*>(reinterpret_cast<unsigned char*>(cnt) + list_bytes);
    if (whole) {  // element e of the block lands at sfb[pad + e]: 16-byte pieces stay aligned on both sides
      const int total = n * F;
      const int h = min(head, total);
      const uint32_t s0 = (uint32_t)__cvta_generic_to_shared(sfb) + 4u * (uint32_t)pad;
      if (lane < h)
        asm volatile("cp.async.ca.shared.global [%0], [%1], 4;" ::"r"(s0 + 4u * lane), "l"(fe + lane) : "memory");
      const int nb = (total - h) >> 2;
      for (int k = lane; k < nb; k += 32)
        asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(s0 + 4u * (uint32_t)(h + 4 * k)),
                     "l"(fe + h + 4 * k)
                     : "memory");
      for (int e = h + 4 * nb + lane; e < total; e += 32)
        asm volatile("cp.async.ca.shared.global [%0], [%1], 4;" ::"r"(s0 + 4u * (uint32_t)e), "l"(fe + e) : "memory");
      asm volatile("cp.async.commit_group;" ::: "memory");
    }
    for (int j = lane; j < K; j += 32) cnt[j] = 0;
    __syncwarp();
    int pos[2 * NP];
#pragma unroll
    for (int j = 0; j < 2 * NP; ++j) pos[j] = j * 32 + lane < n ? atomicAdd(&cnt[lab[j]], 1) : 0;
    __syncwarp();
    count_scan(cnt, start, start, K, lane);
    __syncwarp();
#pragma unroll
    for (int j = 0; j < 2 * NP; ++j)
      if (j * 32 + lane < n) pos[j] += start[lab[j]];
    if (whole) {
#pragma unroll
      for (int j = 0; j < 2 * NP; ++j)
        if (j * 32 + lane < n) perm[pos[j]] = j * 32 + lane;
      asm volatile("cp.async.wait_group 0;" ::: "memory");
      __syncwarp();
      const float* rows = sfb + pad;
      for (int t = lane; t < K; t += 32) {
        const int c2 = cnt[t];
        const int* pj = perm + start[t];
        float* prow = po.pooled + (b * K + t) * F;
        for (int f0 = 0; f0 < F; f0 += 8) {
          double a[8];
#pragma unroll
          for (int f = 0; f < 8; ++f) a[f] = 0.0;
          for (int q = 0; q < c2; ++q) {
            const float* src = rows + pj[q] * F + f0;
#pragma unroll
            for (int f = 0; f < 8; ++f)
              if (f0 + f < F) a[f] += (double)src[f];
          }
          // the mean as the sum times the float64 reciprocal of the count
          // (within an ulp of the float64 quotient)
          const double inv = c2 ? 1.0 / (double)c2 : 0.0;
#pragma unroll
          for (int f = 0; f < 8; ++f)
            if (f0 + f < F) prow[f0 + f] = (float)(a[f] * inv);
        }
        po.counts[b * K + t] = c2;
      }
      __syncwarp();
    } else {
      float* sf = reinterpret_cast<float*>(start + K);
      const int fcap = (kWarpRegionBytes - 8 * K) / (4 * n);  // features one pass can stage (>= 1)
      const int FC = min(min(F, 8), fcap);
      for (int f0 = 0; f0 < F; f0 += FC) {
        const int fc = min(FC, F - f0);
#pragma unroll
        for (int j = 0; j < 2 * NP; ++j) {
          const int i = j * 32 + lane;
          if (i < n) {
            const float* row = fe + (int64_t)i * F + f0;
            float* dst = sf + pos[j] * fc;
#pragma unroll
            for (int f = 0; f < 8; ++f)
              if (f < fc) dst[f] = __ldg(row + f);
          }
        }
        __syncwarp();
        for (int t = lane; t < K; t += 32) {
          const int c2 = cnt[t];
          const float* src = sf + start[t] * fc;
          double a[8];
#pragma unroll
          for (int f = 0; f < 8; ++f) a[f] = 0.0;
          for (int q = 0; q < c2; ++q, src += fc) {
#pragma unroll
            for (int f = 0; f < 8; ++f)
              if (f < fc) a[f] += (double)src[f];
          }
          float* prow = po.pooled + (b * K + t) * F + f0;
          const double inv = c2 ? 1.0 / (double)c2 : 0.0;
#pragma unroll
          for (int f = 0; f < 8; ++f)
            if (f < fc) prow[f] = (float)(a[f] * inv);
          if (f0 == 0) po.counts[b * K + t] = c2;
        }
        __syncwarp();
      }
    }
  }
  __syncwarp();  // the next event overwrites this warp's copy
}

// Resident 128-thread blocks per SM of the warp schedule (its register budget).
#ifndef FPS_WARP_MIN_BLOCKS
#define FPS_WARP_MIN_BLOCKS 3
#endif

template <int NPMAX>
__global__ void __launch_bounds__(128, FPS_WARP_MIN_BLOCKS) k_fps_warp(const float4* __restrict__ coords,
                                                     const int64_t* __restrict__ offsets,
                                                     const int32_t* __restrict__ start_local,
                                                     const int* __restrict__ list, WsHeader* hdr, int K,
                                                     int32_t* __restrict__ centroid_idx,
                                                     int32_t* __restrict__ token_id,
                                                     float4* __restrict__ centroids, PoolOut po, float4 w,
                                                     int scaled) {
  constexpr int kMaxPairs = NPMAX;
  static_assert(2 * NPMAX <= 32, "selected-slot mask is 32 bits");
  // Launched as a programmatic dependent of the binning kernel: the CTAs
  // start while it runs and wait here for its lists (a no-op otherwise).
  asm volatile("griddepcontrol.wait;" ::: "memory");
  extern __shared__ __align__(16) unsigned char s_warp_all[];
  const int lane = threadIdx.x & 31;
  unsigned char* mine = s_warp_all + (size_t)(threadIdx.x >> 5) * kWarpRegionBytes;
  WarpPt* s_pts = reinterpret_cast<WarpPt*>(mine);                      // this warp's event copy
  int* s_c = reinterpret_cast<int*>(mine + 64 * NPMAX * kWarpPtBytes);  // its chosen local indices
  const int count = hdr->n_items[kListWarp];
  // the first item of every warp is its global warp index; later ones come
  // from the shared cursor, offset by the number of warps
  const int nwarps = gridDim.x * (blockDim.x >> 5);
  int* ctr = &hdr->next_item[kListWarp];
  int item = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  while (item < count) {
    const int b = list[item];
    const int64_t off = offsets[b];
    const int n = (int)(offsets[b + 1] - off);
    const int c0 = start_local ? start_local[b] : 0;
    int32_t* tok = token_id ? token_id + off : nullptr;
#define WARP_CALL(N)                                                                                   \
  if (scaled)                                                                                          \
    warp_event<N, true>(coords + off, n, c0, K, off, lane, s_pts, s_c, centroid_idx + (int64_t)b * K,  \
                        centroids + (int64_t)b * K, tok, b, po, w, ctr, nwarps, next);                 \
  else                                                                                                 \
    warp_event<N, false>(coords + off, n, c0, K, off, lane, s_pts, s_c, centroid_idx + (int64_t)b * K, \
                         centroids + (int64_t)b * K, tok, b, po, w, ctr, nwarps, next)
    int next = -1;
    FPS_DISPATCH_7((n + 63) >> 6, WARP_CALL)
#undef WARP_CALL
    if (lane == 0 && next < 0) next = nwarps + atomicAdd(ctr, 1);
    item = __shfl_sync(kFull, next, 0);
  }
}

// ------------------------------------------------------------------ CTA, points in registers

// Claims the next item of `list_id` for the whole CTA (thread 0 draws, the
// others read it after the barrier).
__device__ __forceinline__ int claim_cta(WsHeader* hdr, int list_id, int* slot) {
  __syncthreads();
  if (threadIdx.x == 0) *slot = atomicAdd(&hdr->next_item[list_id], 1);
  __syncthreads();
  return *slot;
}

template <int NP, int NT, int kMaxPairsCta>
__device__ __forceinline__ void cta_event(const float4* __restrict__ pts, int n, int c, int K, int64_t off,
                                          DupPoint* s_dup, int2* xk, int& round, int32_t* __restrict__ cidx,
                                          float4* __restrict__ cpos, int32_t* __restrict__ tok, int64_t b,
                                          const PoolOut& po, float4 w, int scaled) {
  constexpr int NW = NT / 32;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  if (po.feats && tid < 32) prefetch_rows_l2(po.feats + off * po.F, (size_t)n * po.F * sizeof(float), tid, 32);
  const uint64_t z2 = opaque_zero2();
  uint64_t X[NP], Y[NP], Z[NP], T[NP];
  float dist[2 * NP];
  int lab[2 * NP];
  unsigned taken = 0;  // bit j: slot j (point NT j + tid) is selected or empty
#pragma unroll
  for (int p = 0; p < NP; ++p) {
    const int i0 = 2 * NT * p + tid, i1 = i0 + NT;
    float4 a = make_float4(0.f, 0.f, 0.f, 0.f), b = a;
    if (i0 < n) a = ldg4(pts + i0);
    if (i1 < n) b = ldg4(pts + i1);
    if (i0 < n) s_dup[i0] = dup_point(a);  // caller's units (scaled per step when needed)
    if (i1 < n) s_dup[i1] = dup_point(b);
    if (scaled) {
      a = scale4(a, w);
      b = scale4(b, w);
    }
    X[p] = pack2(a.x, b.x);
    Y[p] = pack2(a.y, b.y);
    Z[p] = pack2(a.z, b.z);
    T[p] = pack2(a.w, b.w);
    dist[2 * p] = i0 < n ? __int_as_float(0x7f800000) : kEmptySlot;
    dist[2 * p + 1] = i1 < n ? __int_as_float(0x7f800000) : kEmptySlot;
    lab[2 * p] = 0;
    lab[2 * p + 1] = 0;
    if (i0 >= n) taken |= 1u << (2 * p);
    if (i1 >= n) taken |= 1u << (2 * p + 1);
  }
  __syncthreads();

  // one exchange round: every warp posts (key, index), all warps reduce them
  auto exchange = [&](int wkey, unsigned widx, int& M, unsigned& idx) {
    if (lane == 0) xk[(round & 1) * NW + warp] = make_int2(wkey, (int)widx);
    __syncthreads();
    const int2 v = lane < NW ? xk[(round & 1) * NW + lane] : make_int2(-0x7fffffff - 1, -1);
    warp_argmax(v.x, (unsigned)v.y, M, idx);
    ++round;
  };

  for (int s = 0; s < K; ++s) {
    const DupPoint cp = s_dup[c];
    if (tid == 0) {
      cidx[s] = (int32_t)(off + c);
      cpos[s] = dup_to_float4(cp);
    }
    if (c % NT == tid) taken |= 1u << (c / NT);
    const Cent2 C = scaled ? cent2(scale4(dup_to_float4(cp), w)) : cent2_dup(cp);
    float pm[NP];
#pragma unroll
    for (int p = 0; p < NP; ++p) {
      const uint64_t d = dist2(X[p], Y[p], Z[p], T[p], C, z2);
      relax(lo2(d), dist[2 * p], lab[2 * p], s);
      relax(hi2(d), dist[2 * p + 1], lab[2 * p + 1], s);
      pm[p] = fmaxf(dist[2 * p], dist[2 * p + 1]);
    }
    if (s == K - 1) break;
    const int wM = __reduce_max_sync(kFull, fkey(lane_max<NP>(pm)));
    const int slot = lane_first_slot<NP>(pm, dist, wM);
    const unsigned widx = __reduce_min_sync(kFull, slot < 0 ? 0xffffffffu : (unsigned)(slot * NT + tid));
    int M;
    unsigned idx;
    exchange(wM, widx, M, idx);
    if (M == 0) {  // only duplicates of chosen points remain
      const unsigned free_slots = ~taken & low_bits(2 * NP);
      const unsigned mine = free_slots ? (unsigned)((__ffs(free_slots) - 1) * NT + tid) : 0xffffffffu;
      const unsigned wmin = __reduce_min_sync(kFull, mine);
      exchange(wmin != 0xffffffffu ? 1 : 0, wmin, M, idx);
    }
    c = (int)idx;
  }
  if (tok) {
#pragma unroll
    for (int j = 0; j < 2 * NP; ++j) {
      const int i = j * NT + tid;
      if (i < n) tok[i] = lab[j];
    }
  }
  if (po.feats) {  // token means: sort by token, then one thread per (token, feature) over its run
    constexpr int NMAX = 2 * NT * kMaxPairsCta;
    const int F = po.F;
    __syncthreads();
    int* s_lab = reinterpret_cast<int*>(s_dup);
    int* perm = s_lab + NMAX;
    int* slab = perm + NMAX;
    int* cnt = slab + NMAX;  // cnt, start, cur: 3 x 256
    float* s_feat = reinterpret_cast<float*>(cnt + 768);  // [n * F]
#pragma unroll
    for (int j = 0; j < 2 * NP; ++j) {
      const int i = j * NT + tid;
      if (i < n) s_lab[i] = lab[j];
    }
    // feature rows into shared memory by asynchronous copies, in flight while
    // the labels are sorted; each thread waits for its own before the barrier
    const float* fe = po.feats + off * F;
    const uint32_t s_feat0 = (uint32_t)__cvta_generic_to_shared(s_feat);
#pragma unroll 8
    for (int e = tid; e < n * F; e += NT)
      asm volatile("cp.async.ca.shared.global [%0], [%1], 4;" ::"r"(s_feat0 + 4u * (uint32_t)e), "l"(fe + e)
                   : "memory");
    asm volatile("cp.async.commit_group;" ::: "memory");
    label_sort(s_lab, n, K, cnt, cnt + 256, cnt + 512, perm, slab, tid, NT, [] { __syncthreads(); });
    asm volatile("cp.async.wait_group 0;" ::: "memory");
    __syncthreads();
    // the token's points are perm[start .. start + c): four independent float64
    // partial sums per value, then the mean; no atomics, no accumulator array
    const int* start = cnt + 256;
    for (int q = tid; q < K * F; q += NT) {
      const int j = q / F, f = q - j * F;
      const int c = cnt[j];
      const int* pj = perm + start[j];
      double s0 = 0.0, s1 = 0.0, s2 = 0.0, s3 = 0.0;
      int t = 0;
      for (; t + 4 <= c; t += 4) {
        s0 += (double)s_feat[pj[t] * F + f];
        s1 += (double)s_feat[pj[t + 1] * F + f];
        s2 += (double)s_feat[pj[t + 2] * F + f];
        s3 += (double)s_feat[pj[t + 3] * F + f];
      }
      for (; t < c; ++t) s0 += (double)s_feat[pj[t] * F + f];
      po.pooled[(b * K + j) * F + f] = c ? (float)(((s0 + s1) + (s2 + s3)) / (double)c) : 0.f;
      if (f == 0) po.counts[b * K + j] = c;
    }
  }
}

template <int PR>
__global__ void __launch_bounds__(kCtaThreads, 1) k_fps_cta(const float4* __restrict__ coords,
                                                            const int64_t* __restrict__ offsets,
                                                            const int32_t* __restrict__ start_local,
                                                            const int* __restrict__ list, WsHeader* hdr, int K,
                                                            int32_t* __restrict__ centroid_idx,
                                                            int32_t* __restrict__ token_id,
                                                            float4* __restrict__ centroids, PoolOut po,
                                                            float4 w, int scaled) {
  constexpr int kMaxPairs = PR;
  constexpr int NT = kCtaThreads, NW = NT / 32;
  static_assert(2 * PR <= 32, "selected-slot mask is 32 bits");
  // as the warp schedule: a programmatic dependent of the binning when it is
  // the only FPS schedule (a no-op wait otherwise)
  asm volatile("griddepcontrol.wait;" ::: "memory");
  extern __shared__ DupPoint s_dup[];  // [2 * NT * PR] event copy for centroid look-up
  __shared__ int2 xk[2 * NW];           // (key, index) per warp, double-buffered
  __shared__ int s_item;
  const int count = hdr->n_items[kListCta];
  int round = 0;
  for (;;) {
    const int item = claim_cta(hdr, kListCta, &s_item);
    if (item >= count) break;
    const int b = list[item];
    const int64_t off = offsets[b];
    const int n = (int)(offsets[b + 1] - off);
    const int c0 = start_local ? start_local[b] : 0;
    int32_t* tok = token_id ? token_id + off : nullptr;
#define CTA_CALL(N)                                                                                     \
  cta_event<N, NT, PR>(coords + off, n, c0, K, off, s_dup, xk, round, centroid_idx + (int64_t)b * K,    \
                       centroids + (int64_t)b * K, tok, b, po, w, scaled)
    FPS_DISPATCH_7((n + 2 * NT - 1) / (2 * NT), CTA_CALL)
#undef CTA_CALL
  }
}

// ------------------------------------------------------------------ CTA / cluster, points in shared memory

// DSMEM exchange primitives of the cluster schedules: stores into a peer's
// shared memory that signal the peer's mbarrier with their byte count, and a
// bounded wait on the local mbarrier.
__device__ __forceinline__ uint32_t smem_addr(const void* p) {
  return (uint32_t)__cvta_generic_to_shared(p);
}
__device__ __forceinline__ uint32_t peer_addr(uint32_t local, int rank) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(local), "r"(rank));
  return r;
}
__device__ __forceinline__ void mbar_init(uint32_t bar, int count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}
__device__ __forceinline__ void mbar_arrive_expect(uint32_t bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes) : "memory");
}
__device__ __forceinline__ void st_async_v4(uint32_t addr, int a, int b, int c, int d, uint32_t bar) {
  asm volatile("st.async.shared::cluster.mbarrier::complete_tx::bytes.v4.b32 [%0], {%1, %2, %3, %4}, [%5];" ::"r"(addr),
               "r"(a), "r"(b), "r"(c), "r"(d), "r"(bar)
               : "memory");
}
__device__ __forceinline__ void st_async_v2(uint32_t addr, int a, int b, uint32_t bar) {
  asm volatile("st.async.shared::cluster.mbarrier::complete_tx::bytes.v2.b32 [%0], {%1, %2}, [%3];" ::"r"(addr), "r"(a),
               "r"(b), "r"(bar)
               : "memory");
}
__device__ __forceinline__ bool mbar_try_wait(uint32_t bar, uint32_t parity) {
  uint32_t done;
  asm volatile(
      "{ .reg .pred p; mbarrier.try_wait.parity.acquire.cluster.shared::cta.b64 p, [%1], %2; selp.u32 %0, 1, 0, p; }"
      : "=r"(done)
      : "r"(bar), "r"(parity)
      : "memory");
  return done != 0;
}
// try_wait already suspends in hardware between polls; this many polls is
// far beyond any real exchange (microseconds), and ends a wait that a fault
// elsewhere would otherwise leave spinning.  It is a launch argument, so that
// a test can make it short (fps_set_exchange_test).
constexpr int kExchangeSpinLimit = 1 << 20;

// Launch arguments of the cluster exchange: the poll limit of each wait and,
// for tests, a CTA rank that skips its post in the first exchange of every
// event (-1: none), which makes every wait of that round run out.
struct ExchangeCfg {
  int spin_limit;
  int skip_rank;
};

// Slot of one posted candidate: (key, index, x, y) and (z, t).
struct __align__(16) ExSlot {
  int4 a;
  int2 b;
  int2 pad;
};
constexpr uint32_t kExSlotBytes = 24;  // bytes each post carries (16 + 8)

template <int CL, int NT>
struct BlockShared {
  static constexpr int NW = NT / 32;
  static constexpr int E = CL * NW;  // posted entries per exchange round
};

// Point pairs per thread the shared-memory schedules also keep in registers
// for an event of NP pairs per thread: the running minima, labels and pair
// maxima (5 registers per pair) come first, the cached coordinates (8 per
// pair) take what is left of the 255-register budget of a 256-thread block
// (the budget is set where ptxas reports no spills); the other pairs are read
// from shared memory every step.
__host__ __device__ constexpr int block_reg_pairs(int np) {
  return np < (140 - 5 * np) / 8 ? np : ((140 - 5 * np) / 8 > 0 ? (140 - 5 * np) / 8 : 0);
}

// Returns true when an exchange wait ran out (the CTA left the step loop and
// wrote nothing more for this event).
template <int NP, int CL, int NT>
__device__ __forceinline__ bool block_event(const float4* __restrict__ pts, int n, int c, int K, int64_t off,
                                            int rank, ulonglong2* sXY, ulonglong2* sZT, int2* xkey, float4* xpos,
                                            ExSlot* xslot, uint64_t* xbar, ExSlot* xbc, WsHeader* hdr, int& round,
                                            const ExchangeCfg& xcfg, int32_t* __restrict__ cidx,
                                            float4* __restrict__ cpos, int32_t* __restrict__ tok, float4 w,
                                            int scaled) {
  constexpr int NW = NT / 32;
  constexpr int E = CL * NW;
  constexpr int G = CL * NT;
  static_assert(CL > 1 || E <= 32, "one warp reads the CTA's warp winners");
  static_assert(CL == 1 || CL <= 32, "one lane posts to each CTA of the cluster");
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int g = rank * NT + tid;

  // One exchange of (key, index, position) candidates: the event's winner --
  // largest key, then lowest index -- in M, idx, pos on every thread.
  // Clusters: the CTA's warp winners meet in shared memory (one barrier);
  // warp 0 reduces them and sends the CTA winner into slot `rank` of every
  // CTA of the cluster with st.async, which signals the receiving CTA's
  // mbarrier with its bytes; lane 0 of warp 0 waits (bounded) for the CL
  // posts, warp 0 reduces them and broadcasts the winner with the outcome of
  // the wait through shared memory (a second barrier), so that every thread
  // of the CTA takes the same path.  No cluster barrier and no release fence.
  // Rounds alternate between two slot sets and mbarriers (round & 1; phase
  // parity (round >> 1) & 1): a CTA cannot post round r + 2 before every peer
  // has posted round r + 1, which each does after reading round r.  Posts
  // arriving before the local arm are counted in the same phase (it cannot
  // complete before the local arrival).  Returns false when the wait ran
  // out: every thread of the CTA leaves the event.
  auto exchange = [&](int key, unsigned idx_in, float4 pos_in, bool first, int& M, unsigned& idx,
                      float4& pos) -> bool {
    bool ok = true;
    if constexpr (CL > 1) {
      int2* lkey = xkey + (round & 1) * NW;
      float4* lpos = xpos + (round & 1) * NW;
      const int p = round & 1;
      const uint32_t parity = (uint32_t)(round >> 1) & 1u;
      ExSlot* slots = xslot + p * CL;
      ExSlot* bcs = reinterpret_cast<ExSlot*>(xpos + 2 * NW) + p;
      const uint32_t bar = smem_addr(&xbar[p]);
      ++round;
      if (lane == 0) {
        lkey[warp] = make_int2(key, (int)idx_in);
        lpos[warp] = pos_in;
      }
      __syncthreads();
      if (warp == 0) {
        if (lane == 0) mbar_arrive_expect(bar, CL * kExSlotBytes);
        const int2 v = lane < NW ? lkey[lane] : make_int2(-0x7fffffff - 1, -1);
        int cM;
        unsigned cI;
        warp_argmax(v.x, (unsigned)v.y, cM, cI);
        const unsigned who = __ballot_sync(kFull, lane < NW && v.x == cM && (unsigned)v.y == cI);
        const float4 cp = lpos[__ffs(who) - 1];
        const bool post = !(first && rank == xcfg.skip_rank);
        if (lane < CL && post) {
          const uint32_t ra = peer_addr(smem_addr(&slots[rank]), lane);
          const uint32_t rb = peer_addr(bar, lane);
          st_async_v4(ra, cM, (int)cI, __float_as_int(cp.x), __float_as_int(cp.y), rb);
          st_async_v2(ra + 16, __float_as_int(cp.z), __float_as_int(cp.w), rb);
        }
        bool got = false;
        if (lane == 0)
          for (int it = 0; it < xcfg.spin_limit && !got; ++it) got = mbar_try_wait(bar, parity);
        got = __shfl_sync(kFull, got ? 1 : 0, 0) != 0;
        int2 w2 = make_int2(-0x7fffffff - 1, -1);
        if (got && lane < CL) {
          const int4 a = slots[lane].a;
          w2 = make_int2(a.x, a.y);
        }
        int wM;
        unsigned wI;
        warp_argmax(w2.x, (unsigned)w2.y, wM, wI);
        const unsigned wwho = __ballot_sync(kFull, lane < CL && w2.x == wM && (unsigned)w2.y == wI);
        if (lane == 0) {
          ExSlot bc;
          bc.a = make_int4(wM, (int)wI, 0, 0);
          bc.b = make_int2(0, 0);
          bc.pad = make_int2(got ? 1 : 0, 0);
          if (got) {
            const ExSlot& x = slots[__ffs(wwho) - 1];
            bc.a.z = x.a.z;
            bc.a.w = x.a.w;
            bc.b = x.b;
          } else {
            bc.a = make_int4(-1, 0, 0, 0);
            record_error(hdr, kDevExchangeTimeout);
          }
          *bcs = bc;
        }
      }
      __syncthreads();
      const ExSlot bc = *bcs;
      M = bc.a.x;
      idx = (unsigned)bc.a.y;
      pos = make_float4(__int_as_float(bc.a.z), __int_as_float(bc.a.w), __int_as_float(bc.b.x),
                        __int_as_float(bc.b.y));
      ok = bc.pad.x != 0;
      return ok;
    } else {
      (void)first;
      const int base = (round & 1) * E;
      if (lane == 0) {
        xkey[base + warp] = make_int2(key, (int)idx_in);
        xpos[base + warp] = pos_in;
      }
      __syncthreads();
      const int2 v = lane < E ? xkey[base + lane] : make_int2(-0x7fffffff - 1, -1);
      warp_argmax(v.x, (unsigned)v.y, M, idx);
      const unsigned who = __ballot_sync(kFull, lane < E && v.x == M && (unsigned)v.y == idx);
      pos = xpos[base + __ffs(who) - 1];
    }
    ++round;
    return ok;
  };
  auto local_pos = [&](unsigned idx) {
    const int gi = (int)(idx % (unsigned)G);
    const int j = (int)(idx / (unsigned)G);
    const int t = gi - rank * NT;
    const ulonglong2 xy = sXY[(j >> 1) * NT + t];
    const ulonglong2 zt = sZT[(j >> 1) * NT + t];
    return (j & 1) ? make_float4(hi2(xy.x), hi2(xy.y), hi2(zt.x), hi2(zt.y))
                   : make_float4(lo2(xy.x), lo2(xy.y), lo2(zt.x), lo2(zt.y));
  };

  constexpr int RP = block_reg_pairs(NP);
  const uint64_t z2 = opaque_zero2();
  float dist[2 * NP];
  int lab[2 * NP];
  uint64_t RX[RP], RY[RP], RZ[RP], RT[RP];  // register copies of the first RP pairs
  unsigned long long taken = 0;
#pragma unroll
  for (int p = 0; p < NP; ++p) {
    const int i0 = g + G * (2 * p), i1 = i0 + G;
    float4 a = make_float4(0.f, 0.f, 0.f, 0.f), b = a;
    if (i0 < n) a = ldg4(pts + i0);
    if (i1 < n) b = ldg4(pts + i1);
    if (scaled) {  // the distance reads scaled copies; positions handed out are the caller's
      a = scale4(a, w);
      b = scale4(b, w);
    }
    sXY[p * NT + tid] = make_ulonglong2(pack2(a.x, b.x), pack2(a.y, b.y));
    sZT[p * NT + tid] = make_ulonglong2(pack2(a.z, b.z), pack2(a.w, b.w));
    if (p < RP) {
      RX[p] = pack2(a.x, b.x);
      RY[p] = pack2(a.y, b.y);
      RZ[p] = pack2(a.z, b.z);
      RT[p] = pack2(a.w, b.w);
    }
    dist[2 * p] = i0 < n ? __int_as_float(0x7f800000) : kEmptySlot;
    dist[2 * p + 1] = i1 < n ? __int_as_float(0x7f800000) : kEmptySlot;
    lab[2 * p] = 0;
    lab[2 * p + 1] = 0;
    if (i0 >= n) taken |= 1ull << (2 * p);
    if (i1 >= n) taken |= 1ull << (2 * p + 1);
  }

  __syncthreads();  // every thread's pairs are in shared memory before any warp reads a winner's position
  float4 cc = ldg4(pts + c);  // the current centroid, scaled like the points
  if (scaled) cc = scale4(cc, w);
  for (int s = 0; s < K; ++s) {
    if (rank == 0 && tid == 0) {
      cidx[s] = (int32_t)(off + c);
      cpos[s] = scaled ? ldg4(pts + c) : cc;
    }
    if (c % G == g) taken |= 1ull << (c / G);
    const Cent2 C = cent2(cc);
    float pm[NP];
#pragma unroll
    for (int p = 0; p < NP; ++p) {
      uint64_t d;
      if (p < RP) {
        d = dist2(RX[p], RY[p], RZ[p], RT[p], C, z2);
      } else {
        const ulonglong2 xy = sXY[p * NT + tid];
        const ulonglong2 zt = sZT[p * NT + tid];
        d = dist2(xy.x, xy.y, zt.x, zt.y, C, z2);
      }
      relax(lo2(d), dist[2 * p], lab[2 * p], s);
      relax(hi2(d), dist[2 * p + 1], lab[2 * p + 1], s);
      pm[p] = fmaxf(dist[2 * p], dist[2 * p + 1]);
    }
    if (s == K - 1) break;
    const int wM = __reduce_max_sync(kFull, fkey(lane_max<NP>(pm)));
    const int slot = lane_first_slot<NP>(pm, dist, wM);
    const unsigned widx = __reduce_min_sync(kFull, slot < 0 ? 0xffffffffu : (unsigned)(g + G * slot));
    float4 wpos = make_float4(0.f, 0.f, 0.f, 0.f);
    if (wM >= 0) wpos = local_pos(widx);
    int M;
    unsigned idx;
    if (!exchange(wM, widx, wpos, s == 0, M, idx, cc)) return true;
    if (M == 0) {  // only duplicates of chosen points remain
      const unsigned long long mask = 2 * NP >= 64 ? ~0ull : ((1ull << (2 * NP)) - 1ull);
      const unsigned long long free_slots = ~taken & mask;
      unsigned cand = 0xffffffffu;
      if (free_slots) cand = (unsigned)(g + G * (__ffsll((long long)free_slots) - 1));
      const unsigned wmin = __reduce_min_sync(kFull, cand);
      float4 p = make_float4(0.f, 0.f, 0.f, 0.f);
      if (wmin != 0xffffffffu) p = local_pos(wmin);
      // keys: 1 for a real candidate, 0 for none; ties resolve to the lowest index
      if (!exchange(wmin != 0xffffffffu ? 1 : 0, wmin, p, false, M, idx, cc)) return true;
    }
    c = (int)idx;
  }
  if (tok) {
#pragma unroll
    for (int j = 0; j < 2 * NP; ++j) {
      const int i = g + G * j;
      if (i < n) tok[i] = lab[j];
    }
  }
  return false;
}

// Pair counts compiled for the shared-memory schedules; an event uses the
// smallest one that covers it (extra pairs hold no points).
#define FPS_BLOCK_BUCKETS(np, CALL)                                                                     \
  if ((np) <= 2) { CALL(2); } else if ((np) <= 4) { CALL(4); } else if ((np) <= 6) { CALL(6); }          \
  else if ((np) <= 8) { CALL(8); } else if ((np) <= 10) { CALL(10); } else if ((np) <= 12) { CALL(12); } \
  else if ((np) <= 14) { CALL(14); } else if ((np) <= 16) { CALL(16); } else if ((np) <= 18) { CALL(18); } \
  else if ((np) <= 20) { CALL(20); } else if ((np) <= 22) { CALL(22); } else { CALL(24); }

template <int CL, int NT, int PS>
__global__ void __launch_bounds__(NT, 1) k_fps_block(const float4* __restrict__ coords,
                                                     const int64_t* __restrict__ offsets,
                                                     const int32_t* __restrict__ start_local,
                                                     const int* __restrict__ list, WsHeader* hdr,
                                                     int list_id, int K,
                                                     int32_t* __restrict__ centroid_idx,
                                                     int32_t* __restrict__ token_id,
                                                     float4* __restrict__ centroids, ExchangeCfg xcfg,
                                                     float4 w, int scaled) {
  static_assert(2 * PS <= 64, "selected-slot mask is 64 bits");
  static_assert(PS == 24, "pair buckets of FPS_BLOCK_BUCKETS");
  constexpr int E = BlockShared<CL, NT>::E;
  constexpr int G = CL * NT;
  extern __shared__ __align__(16) unsigned char smem_raw[];
  ulonglong2* sXY = reinterpret_cast<ulonglong2*>(smem_raw);  // [PS][NT] packed (x, y)
  ulonglong2* sZT = sXY + PS * NT;                            // [PS][NT] packed (z, t)
  int2* xkey = reinterpret_cast<int2*>(sZT + PS * NT);        // [2][E] (key, index)
  float4* xpos = reinterpret_cast<float4*>(xkey + 2 * E);     // [2][E] candidate position
  ExSlot* xslot = reinterpret_cast<ExSlot*>(xpos + 2 * E);    // [2][CL] posted CTA winners (clusters)
  ExSlot* xbc = xslot + 2 * CL;                                // spare (the broadcast lives in xpos)
  uint64_t* xbar = reinterpret_cast<uint64_t*>(xbc + 2);       // [2] exchange mbarriers
  __shared__ int s_item;
  __shared__ int s_abort;  // an exchange wait of this CTA ran out (sticky for the launch)

  int rank = 0;
  if constexpr (CL > 1) {
    rank = (int)cg::this_cluster().block_rank();
    if (threadIdx.x == 0) {
      s_abort = 0;
      mbar_init(smem_addr(&xbar[0]), 1);  // armed once per round, by warp 0
      mbar_init(smem_addr(&xbar[1]), 1);
      asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    cg::this_cluster().sync();  // every CTA is running, its barriers initialised, before DSMEM use
  }
  const int count = hdr->n_items[list_id];
  int round = 0;
  for (;;) {
    // the cluster's first CTA claims an item and hands it to the others
    if constexpr (CL > 1) {
      if (rank == 0 && threadIdx.x == 0) {
        const int it = atomicAdd(&hdr->next_item[list_id], 1);
        cg::cluster_group cl = cg::this_cluster();
        for (int r = 0; r < CL; ++r) *cl.map_shared_rank(&s_item, r) = it;
      }
      cg::this_cluster().sync();
    } else {
      __syncthreads();
      if (threadIdx.x == 0) s_item = atomicAdd(&hdr->next_item[list_id], 1);
      __syncthreads();
    }
    const int item = s_item;
    if (item >= count) break;
    const int b = list[item];
    const int64_t off = offsets[b];
    const int n = (int)(offsets[b + 1] - off);
    const int c0 = start_local ? start_local[b] : 0;
    int32_t* tok = token_id ? token_id + off : nullptr;
    const int np = (n + 2 * G - 1) / (2 * G);
    bool aborted = false;
#define BLOCK_CALL(N)                                                                                         \
  aborted = block_event<N, CL, NT>(coords + off, n, c0, K, off, rank, sXY, sZT, xkey, xpos, xslot, xbar, xbc, \
                                   hdr, round, xcfg, centroid_idx + (int64_t)b * K, centroids + (int64_t)b * K, \
                                   tok, w, scaled)
    FPS_BLOCK_BUCKETS(np, BLOCK_CALL)
#undef BLOCK_CALL
    if constexpr (CL > 1) {
      if (aborted && threadIdx.x == 0) s_abort = 1;  // the whole CTA left the event
      cg::this_cluster().sync();  // s_item is rewritten for the next claim; abort flags are final
      // A wait that ran out leaves its mbarrier phase incomplete, so no CTA of
      // the cluster may run another event: every CTA reads every peer's flag
      // (the same values after the barrier) and the cluster stops together.
      int any = 0;
      if (threadIdx.x < CL) any = *cg::this_cluster().map_shared_rank(&s_abort, (unsigned)threadIdx.x);
      if (__syncthreads_or(any)) break;
    }
  }
  if constexpr (CL > 1) cg::this_cluster().sync();  // no CTA leaves while peers may post into it
}

#undef FPS_BLOCK_BUCKETS
#undef FPS_DISPATCH_7
#undef FPS_CASE

// ------------------------------------------------------------------ launch

constexpr int kWarpBlock = 128;
constexpr size_t kWarpSmem = (size_t)(kWarpBlock / 32) * kWarpRegionBytes;
constexpr size_t kCtaSmem = kCtaSmemBytes;
static_assert((size_t)2 * kCtaThreads * kCtaPairs * sizeof(DupPoint) <= kCtaSmem, "event copy fits");

size_t warp_region_bytes() { return (size_t)kWarpRegionBytes; }
size_t cta_region_bytes() { return kCtaSmem; }

template <int CL>
constexpr size_t block_smem_bytes() {
  return (size_t)2 * kBlockPairs * kBlockThreads * sizeof(ulonglong2) +
         (size_t)2 * BlockShared<CL, kBlockThreads>::E * (sizeof(int2) + sizeof(float4)) +
         (size_t)2 * CL * sizeof(ExSlot) + 2 * sizeof(ExSlot) + 2 * sizeof(uint64_t);
}

template <int CL>
static cudaError_t prepare_block_kernel(int* max_active_clusters) {
  auto kern = k_fps_block<CL, kBlockThreads, kBlockPairs>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)block_smem_bytes<CL>());
  if (e != cudaSuccess) return e;
  if (CL > 8 && (e = cudaFuncSetAttribute(kern, cudaFuncAttributeNonPortableClusterSizeAllowed, 1)))
    return e;
  if (CL == 1) return cudaSuccess;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(CL);
  cfg.blockDim = dim3(kBlockThreads);
  cfg.dynamicSmemBytes = block_smem_bytes<CL>();
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = CL;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaOccupancyMaxActiveClusters(max_active_clusters, kern, &cfg);
}

// Exchange settings of the next launches: the default poll limit and no
// skipped post, unless a test set others (fps_set_exchange_test).
static ExchangeCfg g_exchange_cfg = {kExchangeSpinLimit, -1};
static std::mutex g_exchange_mu;
static ExchangeCfg exchange_cfg() {
  std::lock_guard<std::mutex> lock(g_exchange_mu);
  return g_exchange_cfg;
}

void set_exchange_test(int spin_limit, int skip_rank) {
  std::lock_guard<std::mutex> lock(g_exchange_mu);
  g_exchange_cfg.spin_limit = spin_limit > 0 ? spin_limit : kExchangeSpinLimit;
  g_exchange_cfg.skip_rank = skip_rank;
}

template <int CL>
static cudaError_t launch_block(const Problem& pb, const Workspace& ws, int list_id, const int* list,
                                int n_groups, cudaStream_t s) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((n_groups > 0 ? n_groups : 1) * CL);
  cfg.blockDim = dim3(kBlockThreads);
  cfg.dynamicSmemBytes = block_smem_bytes<CL>();
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  int na = 0;
  if (CL > 1) {
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = CL;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    na = 1;
  }
  cfg.attrs = attr;
  cfg.numAttrs = na;
  count_launch();
  return cudaLaunchKernelEx(&cfg, k_fps_block<CL, kBlockThreads, kBlockPairs>, pb.coords, pb.offsets,
                            pb.start_local, list, ws.hdr, list_id, pb.K, pb.centroid_idx, pb.token_id,
                            pb.centroids, exchange_cfg(), pb.w, pb.scaled);
}

// Per-device state: occupancy figures and the helper streams / events that
// let the schedules run concurrently.
constexpr int kHelpers = kNumSchedules + 1;  // one per schedule (high priority) and the passthrough kernel
struct DeviceCtx {
  DeviceInfo info;
  cudaStream_t helper[kHelpers];
  cudaEvent_t fork, join[kHelpers];
  std::mutex launch_mu;
  bool prepared;
};

constexpr int kMaxDevices = 64;
static DeviceCtx g_ctx[kMaxDevices];
static std::mutex g_prepare_mu;

static int current_device() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return -1;
  return dev;
}

// One-time set-up per device: kernel attributes, occupancy figures, helper
// streams and fork/join events.
static cudaError_t prepare(int dev) {
  std::lock_guard<std::mutex> lock(g_prepare_mu);
  DeviceCtx& ctx = g_ctx[dev];
  if (ctx.prepared) return cudaSuccess;
  DeviceInfo info = {};
  cudaError_t e = cudaDeviceGetAttribute(&info.sm_count, cudaDevAttrMultiProcessorCount, dev);
  if (e != cudaSuccess) return e;
  if ((e = cudaFuncSetAttribute(k_fps_warp<kWarpPairs>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                (int)kWarpSmem)))
    return e;
  if ((e = cudaFuncSetAttribute(k_fps_cta<kCtaPairs>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                (int)kCtaSmem)))
    return e;
  e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&info.warp_blocks_per_sm, k_fps_warp<kWarpPairs>,
                                                    kWarpBlock, kWarpSmem);
  if (e != cudaSuccess) return e;
  int unused = 0;
  if ((e = prepare_block_kernel<1>(&unused)) != cudaSuccess) return e;
  if ((e = prepare_block_kernel<8>(&info.cluster8_max_active)) != cudaSuccess) return e;
  if ((e = prepare_block_kernel<16>(&info.cluster16_max_active)) != cudaSuccess) return e;
  if ((e = prepare_aux_kernels()) != cudaSuccess) return e;
  // FPS schedules (the critical path) on high priorities -- the larger the
  // schedule's events, the higher, so that its work (and in kNN mode its
  // rows) is scheduled first -- and the passthrough kernel, which only has
  // to finish before pooling, on the lowest
  int least = 0, greatest = 0;
  if ((e = cudaDeviceGetStreamPriorityRange(&least, &greatest))) return e;
  for (int i = 0; i < kHelpers; ++i) {
    int prio = greatest + (kNumSchedules - 1 - i);  // numerically smaller = higher
    if (prio > least) prio = least;
    if (i == kHelpers - 1) prio = least;
    if ((e = cudaStreamCreateWithPriority(&ctx.helper[i], cudaStreamNonBlocking, prio))) return e;
    if ((e = cudaEventCreateWithFlags(&ctx.join[i], cudaEventDisableTiming))) return e;
  }
  if ((e = cudaEventCreateWithFlags(&ctx.fork, cudaEventDisableTiming))) return e;
  info.ready = true;
  ctx.info = info;
  ctx.prepared = true;
  return cudaSuccess;
}

static const DeviceInfo g_none = {};

const DeviceInfo& device_info() {
  const int dev = current_device();
  if (dev < 0 || prepare(dev) != cudaSuccess) return g_none;
  return g_ctx[dev].info;
}

cudaError_t launch_fps(const Problem& pb, const Problem& pt, const Workspace& ws, cudaStream_t s, StageMark mark) {
  const int dev = current_device();
  if (dev < 0) return cudaErrorInvalidDevice;
  cudaError_t e = prepare(dev);
  if (e != cudaSuccess) return e;
  DeviceCtx& ctx = g_ctx[dev];
  const DeviceInfo& di = ctx.info;
  // Launch a schedule unless the size hint rules out every event it could
  // get: schedule q receives events above lower[q] (above K when forced; the
  // CTA schedule also takes small events when there are few of them).
  const int hint = pb.max_event_hint;
  const int f = pb.force_schedule;
  const bool maybe_few = pb.B <= kLatencyEventsPerSm * di.sm_count;  // small events may move to the CTA
  // (the 8-CTA cluster also takes mid-size events when there are few of them)
  const int lower[kNumSchedules] = {pb.K, maybe_few ? pb.K : kWarpCap, kCtaCap, f < 0 ? kCtaCap : kCtaSmemCap,
                                    kCluster8Cap};
  bool run[kNumSchedules];
  for (int q = 0; q < kNumSchedules; ++q) {
    const int lo = f >= q ? pb.K : lower[q];
    const bool allowed = f < 0 || q == kNumSchedules - 1 || f <= q;
    run[q] = allowed && (hint == 0 || hint > lo);
  }
  // at most one event per SM: every warp-class event runs on the CTA schedule
  if (f < 0 && maybe_few) run[0] = false;
  int n_run = 0;
  for (int q = 0; q < kNumSchedules; ++q) n_run += run[q] ? 1 : 0;


  const PoolOut none = {nullptr, 0, nullptr, nullptr};
  const PoolOut pool = {pb.feats, pb.F, pb.pooled, pb.counts};
  const PoolOut po_warp = (pb.fused_pool & 1) ? pool : none;
  const PoolOut po_cta = (pb.fused_pool & 2) ? pool : none;

  const bool knn_per_schedule = knn_with_fps(pb);
  std::lock_guard<std::mutex> lock(ctx.launch_mu);  // the fork/join events are shared per device
  if ((e = cudaEventRecord(ctx.fork, s))) return e;
  for (int q = 0; q < kNumSchedules; ++q) {
    if (!run[q]) continue;
    // When the warp or the register-CTA schedule is the only FPS schedule, it
    // follows the binning kernel on the caller's stream as a programmatic
    // dependent launch (its CTAs are placed while the binning runs);
    // otherwise every schedule runs on its own stream, so that no schedule's
    // CTAs take the SMs ahead of another's longest events.
    const bool chained = n_run == 1 && q <= 1;
    cudaStream_t hs = chained ? s : ctx.helper[q];
    if (!chained && (e = cudaStreamWaitEvent(hs, ctx.fork, 0))) return e;
    mark(1 + q, 0, hs);
    switch (q) {
      case 0: {
        const int blocks = di.sm_count * (di.warp_blocks_per_sm > 0 ? di.warp_blocks_per_sm : 1);
        count_launch();
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3(blocks);
        cfg.blockDim = dim3(kWarpBlock);
        cfg.dynamicSmemBytes = kWarpSmem;
        cfg.stream = hs;
        cudaLaunchAttribute attr[1];
        attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
        attr[0].val.programmaticStreamSerializationAllowed = 1;
        cfg.attrs = attr;
        cfg.numAttrs = chained ? 1 : 0;
        e = cudaLaunchKernelEx(&cfg, k_fps_warp<kWarpPairs>, pb.coords, pb.offsets, pb.start_local,
                               (const int*)ws.list_warp, ws.hdr, pb.K, pb.centroid_idx, pb.token_id, pb.centroids,
                               po_warp, pb.w, pb.scaled);
        break;
      }
      case 1: {
        count_launch();
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3(di.sm_count);
        cfg.blockDim = dim3(kCtaThreads);
        cfg.dynamicSmemBytes = kCtaSmem;
        cfg.stream = hs;
        cudaLaunchAttribute attr[1];
        attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
        attr[0].val.programmaticStreamSerializationAllowed = 1;
        cfg.attrs = attr;
        cfg.numAttrs = chained ? 1 : 0;
        e = cudaLaunchKernelEx(&cfg, k_fps_cta<kCtaPairs>, pb.coords, pb.offsets, pb.start_local,
                               (const int*)ws.list_cta, ws.hdr, pb.K, pb.centroid_idx, pb.token_id, pb.centroids,
                               po_cta, pb.w, pb.scaled);
        break;
      }
      case 2:
        e = launch_block<1>(pb, ws, kListCtaSmem, ws.list_cta_smem, di.sm_count, hs);
        break;
      case 3:
        e = launch_block<8>(pb, ws, kListCluster8, ws.list_cluster8, di.cluster8_max_active, hs);
        break;
      default:
        e = launch_block<16>(pb, ws, kListCluster16, ws.list_cluster16, di.cluster16_max_active, hs);
        break;
    }
    if (e != cudaSuccess) return e;
    // kNN mode without Lloyd: this schedule's kNN rows follow on its own
    // stream, overlapping the other schedules' FPS (its stage includes them)
    if (knn_per_schedule &&
        (e = launch_knn(pb.coords, pb.offsets, pb.B, pb.centroids, nullptr, pb.K, pb.k, pb.knn_idx, pb.feats, pb.F,
                        pb.pooled, pb.counts, &ws, ws.hdr, hs, pb.w, pb.scaled, q)))
      return e;
    mark(1 + q, 1, hs);
    if (!chained && (e = cudaEventRecord(ctx.join[q], hs))) return e;
  }
  {  // passthrough rows and accumulator clearing overlap the FPS kernels (enqueued last, lowest priority)
    cudaStream_t hs = ctx.helper[kHelpers - 1];
    if ((e = cudaStreamWaitEvent(hs, ctx.fork, 0))) return e;
    mark(kStagePassthrough, 0, hs);
    // Voronoi mode: the accumulators of a later pooling pass (the last Lloyd
    // step, or the pool kernel) start cleared; none follows when every event
    // is pooled in place
    if (pb.assign_mode == 0 && (pb.lloyd_iters > 0 || pool_kernel_needed(pb)) &&
        (e = launch_pool_clear(pb, ws, hs)))
      return e;
    if ((e = launch_passthrough(pt, ws, hs))) return e;
    mark(kStagePassthrough, 1, hs);
    if ((e = cudaEventRecord(ctx.join[kHelpers - 1], hs))) return e;
  }
  for (int q = 0; q < kNumSchedules; ++q)
    if (run[q] && !(n_run == 1 && q <= 1) && (e = cudaStreamWaitEvent(s, ctx.join[q], 0))) return e;
  return cudaStreamWaitEvent(s, ctx.join[kHelpers - 1], 0);
}

}  // namespace fpstok
