// Farthest point sampling fused with the Voronoi labels, four schedules.
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
// Schedules (chosen per event by the binning kernel; all run concurrently,
// the three block schedules on helper streams forked from the caller's):
//   warp      N <= 448      one warp per event; points in registers (lane l
//                           owns points l + 32 j); arg-max with two redux.sync.
//   CTA       N <= 2560     one 128-thread CTA per event; points in registers;
//                           warp results exchanged through shared memory,
//                           one barrier per step.
//   CTA-smem  N <= 12288    one 256-thread CTA per event; points in shared
//                           memory as packed f32x2 pairs; distances and labels
//                           in registers.
//   cluster   N <= 196608   a 16-CTA thread-block cluster per event (same
//                           layout); every warp posts its candidate into every
//                           CTA's shared memory over DSMEM; one
//                           barrier.cluster per step.
// Every step touches exactly the occupied point pairs: the unrolled per-pair
// code is entered through a switch on the pair count (no per-pair guards).
#include <cooperative_groups.h>

#include <mutex>

#include "common.cuh"
#include "internal.h"

namespace cg = cooperative_groups;

namespace fpstok {

// Runs BODY(p) for p = np-1 down to 0 (np <= 24): the switch enters the
// unrolled sequence at the right place.  BODY(p) is compiled only for
// p < kMaxPairs, a constexpr in the calling scope.
#define FPS_CASE(p, BODY) \
  case (p) + 1:           \
    if constexpr ((p) < kMaxPairs) { BODY(p) } [[fallthrough]];
#define FPS_FALL(np, BODY)                                                                                   \
  switch (np) {                                                                                              \
    FPS_CASE(23, BODY) FPS_CASE(22, BODY) FPS_CASE(21, BODY) FPS_CASE(20, BODY) FPS_CASE(19, BODY)          \
    FPS_CASE(18, BODY) FPS_CASE(17, BODY) FPS_CASE(16, BODY) FPS_CASE(15, BODY) FPS_CASE(14, BODY)          \
    FPS_CASE(13, BODY) FPS_CASE(12, BODY) FPS_CASE(11, BODY) FPS_CASE(10, BODY) FPS_CASE(9, BODY)           \
    FPS_CASE(8, BODY) FPS_CASE(7, BODY) FPS_CASE(6, BODY) FPS_CASE(5, BODY) FPS_CASE(4, BODY)               \
    FPS_CASE(3, BODY) FPS_CASE(2, BODY) FPS_CASE(1, BODY) FPS_CASE(0, BODY) default : break;                \
  }

__device__ __forceinline__ unsigned low_bits(int n) { return n >= 32 ? 0xffffffffu : ((1u << n) - 1u); }

// ------------------------------------------------------------------ warp

template <int NP>
__global__ void __launch_bounds__(128, 3) k_fps_warp(const float4* __restrict__ coords,
                                                     const int64_t* __restrict__ offsets,
                                                     const int32_t* __restrict__ start_local,
                                                     const int* __restrict__ list, WsHeader* hdr, int K,
                                                     int32_t* __restrict__ centroid_idx,
                                                     int32_t* __restrict__ token_id,
                                                     float4* __restrict__ centroids) {
  constexpr int kMaxPairs = NP;
  static_assert(2 * NP <= 32, "selected-slot mask is 32 bits");
  extern __shared__ DupPoint s_dup_all[];
  const int lane = threadIdx.x & 31;
  DupPoint* s_dup = s_dup_all + (threadIdx.x >> 5) * (64 * NP);  // this warp's event copy
  const int gw = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int nw = (gridDim.x * blockDim.x) >> 5;
  const int count = hdr->n_items[kListWarp];

  for (int w = gw; w < count; w += nw) {
    const int b = list[w];
    const int64_t off = offsets[b];
    const int n = (int)(offsets[b + 1] - off);
    const int npairs = (n + 63) >> 6;
    const float4* pts = coords + off;

    uint64_t X[NP], Y[NP], Z[NP], T[NP];
    float dist[2 * NP];
    int lab[2 * NP];
    unsigned taken = 0;  // bit j: slot j (point 32 j + lane) is selected or empty
#pragma unroll
    for (int p = 0; p < NP; ++p) {
      const int i0 = 64 * p + lane, i1 = i0 + 32;
      float4 a = make_float4(0.f, 0.f, 0.f, 0.f), c = a;
      if (p < npairs) {
        if (i0 < n) a = ldg4(pts + i0);
        if (i1 < n) c = ldg4(pts + i1);
        if (i0 < n) s_dup[i0] = dup_point(a);
        if (i1 < n) s_dup[i1] = dup_point(c);
      }
      X[p] = pack2(a.x, c.x);
      Y[p] = pack2(a.y, c.y);
      Z[p] = pack2(a.z, c.z);
      T[p] = pack2(a.w, c.w);
      dist[2 * p] = i0 < n ? __int_as_float(0x7f800000) : kEmptySlot;
      dist[2 * p + 1] = i1 < n ? __int_as_float(0x7f800000) : kEmptySlot;
      lab[2 * p] = 0;
      lab[2 * p + 1] = 0;
      if (i0 >= n) taken |= 1u << (2 * p);
      if (i1 >= n) taken |= 1u << (2 * p + 1);
    }
    __syncwarp();

    int c = start_local ? start_local[b] : 0;
    for (int s = 0; s < K; ++s) {
      const DupPoint cp = s_dup[c];
      if (lane == 0) {
        centroid_idx[(int64_t)b * K + s] = (int32_t)(off + c);
        centroids[(int64_t)b * K + s] = dup_to_float4(cp);
      }
      if ((c & 31) == lane) taken |= 1u << (c >> 5);
      const Cent2 C = cent2_dup(cp);
      float m0 = kEmptySlot, m1 = kEmptySlot;
#define W_UPD(p)                                                  \
  {                                                               \
    const uint64_t d = dist2(X[p], Y[p], Z[p], T[p], C);          \
    relax(lo2(d), dist[2 * (p)], lab[2 * (p)], s);                \
    relax(hi2(d), dist[2 * (p) + 1], lab[2 * (p) + 1], s);        \
    if ((p) & 1)                                                  \
      m1 = max3f(m1, dist[2 * (p)], dist[2 * (p) + 1]);           \
    else                                                          \
      m0 = max3f(m0, dist[2 * (p)], dist[2 * (p) + 1]);           \
  }
      FPS_FALL(npairs, W_UPD)
#undef W_UPD
      if (s == K - 1) break;
      const int key = fkey(fmaxf(m0, m1));
      const int M = __reduce_max_sync(kFull, key);
      unsigned cand = 0xffffffffu;
      if (key == M) {
#define W_SCAN(p)                                                                         \
  {                                                                                       \
    if (fkey(dist[2 * (p) + 1]) == M) cand = (unsigned)((2 * (p) + 1) * 32 + lane);       \
    if (fkey(dist[2 * (p)]) == M) cand = (unsigned)((2 * (p)) * 32 + lane);               \
  }
        FPS_FALL(npairs, W_SCAN)
#undef W_SCAN
      }
      unsigned idx = __reduce_min_sync(kFull, cand);
      if (M == 0) {  // only duplicates of chosen points remain
        const unsigned free_slots = ~taken & low_bits(2 * npairs);
        cand = free_slots ? (unsigned)((__ffs(free_slots) - 1) * 32 + lane) : 0xffffffffu;
        idx = __reduce_min_sync(kFull, cand);
      }
      c = (int)idx;
    }
    if (token_id) {
#pragma unroll
      for (int j = 0; j < 2 * NP; ++j) {
        const int i = j * 32 + lane;
        if (i < n) token_id[off + i] = lab[j];
      }
    }
    __syncwarp();  // the next event overwrites this warp's copy
  }
}

// ------------------------------------------------------------------ CTA, points in registers

template <int PR>
__global__ void __launch_bounds__(128, 1) k_fps_cta(const float4* __restrict__ coords,
                                                    const int64_t* __restrict__ offsets,
                                                    const int32_t* __restrict__ start_local,
                                                    const int* __restrict__ list, WsHeader* hdr, int K,
                                                    int32_t* __restrict__ centroid_idx,
                                                    int32_t* __restrict__ token_id,
                                                    float4* __restrict__ centroids) {
  constexpr int kMaxPairs = PR;
  constexpr int NT = 128, NW = 4;
  static_assert(2 * PR <= 32, "selected-slot mask is 32 bits");
  extern __shared__ DupPoint s_dup[];  // [256 * PR] event copy for centroid look-up
  __shared__ int2 xk[2 * NW];           // (key, index) per warp, double-buffered
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int count = hdr->n_items[kListCta];
  int round = 0;

  auto exchange = [&](int wkey, unsigned widx, int& M, unsigned& idx) {
    if (lane == 0) xk[(round & 1) * NW + warp] = make_int2(wkey, (int)widx);
    __syncthreads();
    const int2 v = lane < NW ? xk[(round & 1) * NW + lane] : make_int2(-0x7fffffff - 1, -1);
    warp_argmax(v.x, (unsigned)v.y, M, idx);
    ++round;
  };

  for (int item = blockIdx.x; item < count; item += gridDim.x) {
    const int b = list[item];
    const int64_t off = offsets[b];
    const int n = (int)(offsets[b + 1] - off);
    const int npairs = (n + 2 * NT - 1) / (2 * NT);
    const float4* pts = coords + off;

    uint64_t X[PR], Y[PR], Z[PR], T[PR];
    float dist[2 * PR];
    int lab[2 * PR];
    unsigned taken = 0;  // bit j: slot j (point NT j + tid) is selected or empty
#pragma unroll
    for (int p = 0; p < PR; ++p) {
      const int i0 = 2 * NT * p + tid, i1 = i0 + NT;
      float4 a = make_float4(0.f, 0.f, 0.f, 0.f), c = a;
      if (p < npairs) {
        if (i0 < n) a = ldg4(pts + i0);
        if (i1 < n) c = ldg4(pts + i1);
        if (i0 < n) s_dup[i0] = dup_point(a);
        if (i1 < n) s_dup[i1] = dup_point(c);
      }
      X[p] = pack2(a.x, c.x);
      Y[p] = pack2(a.y, c.y);
      Z[p] = pack2(a.z, c.z);
      T[p] = pack2(a.w, c.w);
      dist[2 * p] = i0 < n ? __int_as_float(0x7f800000) : kEmptySlot;
      dist[2 * p + 1] = i1 < n ? __int_as_float(0x7f800000) : kEmptySlot;
      lab[2 * p] = 0;
      lab[2 * p + 1] = 0;
      if (i0 >= n) taken |= 1u << (2 * p);
      if (i1 >= n) taken |= 1u << (2 * p + 1);
    }
    __syncthreads();

    int c = start_local ? start_local[b] : 0;
    for (int s = 0; s < K; ++s) {
      const DupPoint cp = s_dup[c];
      if (tid == 0) {
        centroid_idx[(int64_t)b * K + s] = (int32_t)(off + c);
        centroids[(int64_t)b * K + s] = dup_to_float4(cp);
      }
      if (c % NT == tid) taken |= 1u << (c / NT);
      const Cent2 C = cent2_dup(cp);
      float m0 = kEmptySlot, m1 = kEmptySlot;
#define C_UPD(p)                                                  \
  {                                                               \
    const uint64_t d = dist2(X[p], Y[p], Z[p], T[p], C);          \
    relax(lo2(d), dist[2 * (p)], lab[2 * (p)], s);                \
    relax(hi2(d), dist[2 * (p) + 1], lab[2 * (p) + 1], s);        \
    if ((p) & 1)                                                  \
      m1 = max3f(m1, dist[2 * (p)], dist[2 * (p) + 1]);           \
    else                                                          \
      m0 = max3f(m0, dist[2 * (p)], dist[2 * (p) + 1]);           \
  }
      FPS_FALL(npairs, C_UPD)
#undef C_UPD
      if (s == K - 1) break;
      const int key = fkey(fmaxf(m0, m1));
      const int wM = __reduce_max_sync(kFull, key);
      unsigned cand = 0xffffffffu;
      if (key == wM) {
#define C_SCAN(p)                                                                      \
  {                                                                                    \
    if (fkey(dist[2 * (p) + 1]) == wM) cand = (unsigned)((2 * (p) + 1) * NT + tid);    \
    if (fkey(dist[2 * (p)]) == wM) cand = (unsigned)((2 * (p)) * NT + tid);            \
  }
        FPS_FALL(npairs, C_SCAN)
#undef C_SCAN
      }
      const unsigned widx = __reduce_min_sync(kFull, cand);
      int M;
      unsigned idx;
      exchange(wM, widx, M, idx);
      if (M == 0) {  // only duplicates of chosen points remain
        const unsigned free_slots = ~taken & low_bits(2 * npairs);
        const unsigned mine = free_slots ? (unsigned)((__ffs(free_slots) - 1) * NT + tid) : 0xffffffffu;
        const unsigned wmin = __reduce_min_sync(kFull, mine);
        exchange(wmin != 0xffffffffu ? 1 : 0, wmin, M, idx);
      }
      c = (int)idx;
    }
    if (token_id) {
#pragma unroll
      for (int j = 0; j < 2 * PR; ++j) {
        const int i = j * NT + tid;
        if (i < n) token_id[off + i] = lab[j];
      }
    }
    __syncthreads();  // the next event overwrites the shared copy
  }
}

// ------------------------------------------------------------------ CTA / cluster, points in shared memory

template <int CL, int NT, int PS>
__global__ void __launch_bounds__(NT, 1) k_fps_block(const float4* __restrict__ coords,
                                                     const int64_t* __restrict__ offsets,
                                                     const int32_t* __restrict__ start_local,
                                                     const int* __restrict__ list, WsHeader* hdr,
                                                     int list_id, int K,
                                                     int32_t* __restrict__ centroid_idx,
                                                     int32_t* __restrict__ token_id,
                                                     float4* __restrict__ centroids) {
  constexpr int kMaxPairs = PS;
  static_assert(2 * PS <= 64, "selected-slot mask is 64 bits");
  constexpr int NW = NT / 32;
  constexpr int E = CL * NW;
  extern __shared__ __align__(16) unsigned char smem_raw[];
  ulonglong2* sXY = reinterpret_cast<ulonglong2*>(smem_raw);  // [PS][NT] packed (x, y)
  ulonglong2* sZT = sXY + PS * NT;                            // [PS][NT] packed (z, t)
  int2* xkey = reinterpret_cast<int2*>(sZT + PS * NT);        // [2][E] (key, index)
  float4* xpos = reinterpret_cast<float4*>(xkey + 2 * E);     // [2][E] candidate position

  const int tid = threadIdx.x;
  const int lane = tid & 31;
  const int warp = tid >> 5;
  int rank = 0;
  if constexpr (CL > 1) {
    rank = (int)cg::this_cluster().block_rank();
    cg::this_cluster().sync();  // every CTA of the cluster is running before DSMEM use
  }
  const int G = CL * NT;
  const int g = rank * NT + tid;
  const int nclusters = gridDim.x / CL;
  const int count = hdr->n_items[list_id];
  int round = 0;

  // Posts (key, idx, pos) of this warp into slot [round&1][rank*NW+warp] of every CTA.
  auto post = [&](int key, unsigned idx, float4 pos) {
    const int slot = (round & 1) * E + rank * NW + warp;
    if constexpr (CL > 1) {
      if (lane < CL) {
        cg::cluster_group cl = cg::this_cluster();
        int2* rk = cl.map_shared_rank(xkey, lane);
        float4* rp = cl.map_shared_rank(xpos, lane);
        rk[slot] = make_int2(key, (int)idx);
        rp[slot] = pos;
      }
    } else {
      if (lane == 0) {
        xkey[slot] = make_int2(key, (int)idx);
        xpos[slot] = pos;
      }
    }
  };
  auto barrier = [&]() {
    if constexpr (CL > 1) {
      cg::this_cluster().sync();
    } else {
      __syncthreads();
    }
  };
  // Reduces the posted entries of this round: largest key, then smallest index.
  auto gather = [&](int& M, unsigned& idx, float4& pos) {
    const int base = (round & 1) * E;
    int bk = -0x7fffffff - 1;
    unsigned bi = 0xffffffffu;
    int be = 0;
#pragma unroll
    for (int e = lane; e < E; e += 32) {
      const int2 v = xkey[base + e];
      if (v.x > bk || (v.x == bk && (unsigned)v.y < bi)) {
        bk = v.x;
        bi = (unsigned)v.y;
        be = e;
      }
    }
    warp_argmax(bk, bi, M, idx);
    const unsigned who = __ballot_sync(kFull, bk == M && bi == idx);
    const int e = __shfl_sync(kFull, be, __ffs(who) - 1);
    pos = xpos[base + e];
    ++round;
  };
  // Position of a point this CTA holds, from its shared-memory pair.
  auto local_pos = [&](unsigned idx) {
    const int gi = (int)(idx % (unsigned)G);
    const int j = (int)(idx / (unsigned)G);
    const int t = gi - rank * NT;
    const ulonglong2 xy = sXY[(j >> 1) * NT + t];
    const ulonglong2 zt = sZT[(j >> 1) * NT + t];
    return (j & 1) ? make_float4(hi2(xy.x), hi2(xy.y), hi2(zt.x), hi2(zt.y))
                   : make_float4(lo2(xy.x), lo2(xy.y), lo2(zt.x), lo2(zt.y));
  };

  for (int item = blockIdx.x / CL; item < count; item += nclusters) {
    const int b = list[item];
    const int64_t off = offsets[b];
    const int n = (int)(offsets[b + 1] - off);
    const int npairs = (n + 2 * G - 1) / (2 * G);
    const float4* pts = coords + off;

    float dist[2 * PS];
    int lab[2 * PS];
    unsigned long long taken = 0;
#pragma unroll
    for (int p = 0; p < PS; ++p) {
      const int i0 = g + G * (2 * p), i1 = i0 + G;
      if (p < npairs) {
        float4 a = make_float4(0.f, 0.f, 0.f, 0.f), c = a;
        if (i0 < n) a = ldg4(pts + i0);
        if (i1 < n) c = ldg4(pts + i1);
        sXY[p * NT + tid] = make_ulonglong2(pack2(a.x, c.x), pack2(a.y, c.y));
        sZT[p * NT + tid] = make_ulonglong2(pack2(a.z, c.z), pack2(a.w, c.w));
      }
      dist[2 * p] = i0 < n ? __int_as_float(0x7f800000) : kEmptySlot;
      dist[2 * p + 1] = i1 < n ? __int_as_float(0x7f800000) : kEmptySlot;
      lab[2 * p] = 0;
      lab[2 * p + 1] = 0;
      if (i0 >= n) taken |= 1ull << (2 * p);
      if (i1 >= n) taken |= 1ull << (2 * p + 1);
    }

    int c = start_local ? start_local[b] : 0;
    float4 cc = ldg4(pts + c);
    for (int s = 0; s < K; ++s) {
      if (rank == 0 && tid == 0) {
        centroid_idx[(int64_t)b * K + s] = (int32_t)(off + c);
        centroids[(int64_t)b * K + s] = cc;
      }
      if (c % G == g) taken |= 1ull << (c / G);
      const Cent2 C = cent2(cc);
      float m0 = kEmptySlot, m1 = kEmptySlot;
#define B_UPD(p)                                                   \
  {                                                                \
    const ulonglong2 xy = sXY[(p) * NT + tid];                     \
    const ulonglong2 zt = sZT[(p) * NT + tid];                     \
    const uint64_t d = dist2(xy.x, xy.y, zt.x, zt.y, C);           \
    relax(lo2(d), dist[2 * (p)], lab[2 * (p)], s);                 \
    relax(hi2(d), dist[2 * (p) + 1], lab[2 * (p) + 1], s);         \
    if ((p) & 1)                                                   \
      m1 = max3f(m1, dist[2 * (p)], dist[2 * (p) + 1]);            \
    else                                                           \
      m0 = max3f(m0, dist[2 * (p)], dist[2 * (p) + 1]);            \
  }
      FPS_FALL(npairs, B_UPD)
#undef B_UPD
      if (s == K - 1) break;

      const int key = fkey(fmaxf(m0, m1));
      const int wM = __reduce_max_sync(kFull, key);
      unsigned wcand = 0xffffffffu;
      if (key == wM) {
#define B_SCAN(p)                                                                     \
  {                                                                                   \
    if (fkey(dist[2 * (p) + 1]) == wM) wcand = (unsigned)(g + G * (2 * (p) + 1));     \
    if (fkey(dist[2 * (p)]) == wM) wcand = (unsigned)(g + G * (2 * (p)));             \
  }
        FPS_FALL(npairs, B_SCAN)
#undef B_SCAN
      }
      const unsigned widx = __reduce_min_sync(kFull, wcand);
      float4 wpos = make_float4(0.f, 0.f, 0.f, 0.f);
      if (wM >= 0) wpos = local_pos(widx);
      post(wM, widx, wpos);
      barrier();
      int M;
      unsigned idx;
      gather(M, idx, cc);
      if (M == 0) {  // only duplicates of chosen points remain
        const int nslots = 2 * npairs;
        const unsigned long long mask = nslots >= 64 ? ~0ull : ((1ull << nslots) - 1ull);
        const unsigned long long free_slots = ~taken & mask;
        unsigned cand = 0xffffffffu;
        if (free_slots) cand = (unsigned)(g + G * (__ffsll((long long)free_slots) - 1));
        const unsigned wmin = __reduce_min_sync(kFull, cand);
        float4 p = make_float4(0.f, 0.f, 0.f, 0.f);
        if (wmin != 0xffffffffu) p = local_pos(wmin);
        // keys: 1 for a real candidate, 0 for none; ties resolve to the lowest index
        post(wmin != 0xffffffffu ? 1 : 0, wmin, p);
        barrier();
        gather(M, idx, cc);
      }
      c = (int)idx;
    }
    if (token_id) {
#pragma unroll
      for (int j = 0; j < 2 * PS; ++j) {
        const int i = g + G * j;
        if (j < 2 * npairs && i < n) token_id[off + i] = lab[j];
      }
    }
  }
  if constexpr (CL > 1) cg::this_cluster().sync();  // no CTA leaves while peers may post into it
}

#undef FPS_FALL
#undef FPS_CASE

// ------------------------------------------------------------------ launch

constexpr int kWarpBlock = 128;
constexpr size_t kWarpSmem = (size_t)(kWarpBlock / 32) * 64 * kWarpPairs * sizeof(DupPoint);
constexpr size_t kCtaSmem = (size_t)2 * 128 * kCtaPairs * sizeof(DupPoint);

template <int CL>
constexpr size_t block_smem_bytes() {
  return (size_t)2 * kBlockPairs * kBlockThreads * sizeof(ulonglong2) +
         (size_t)2 * CL * (kBlockThreads / 32) * (sizeof(int2) + sizeof(float4));
}

template <int CL>
static cudaError_t prepare_block_kernel() {
  auto kern = k_fps_block<CL, kBlockThreads, kBlockPairs>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)block_smem_bytes<CL>());
  if (e != cudaSuccess) return e;
  if (CL > 8) {
    e = cudaFuncSetAttribute(kern, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
    if (e != cudaSuccess) return e;
  }
  return cudaSuccess;
}

template <int CL>
static cudaError_t launch_block(const Problem& pb, const Workspace& ws, int list_id, int n_groups,
                                cudaStream_t s) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(n_groups * CL);
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
  const int* list = list_id == kListCtaSmem ? ws.list_cta_smem : ws.list_cluster;
  count_launch();
  return cudaLaunchKernelEx(&cfg, k_fps_block<CL, kBlockThreads, kBlockPairs>, pb.coords,
                            pb.offsets, pb.start_local, list, ws.hdr, list_id, pb.K, pb.centroid_idx,
                            pb.token_id, pb.centroids);
}

// Per-device state: occupancy figures and the helper streams / events that
// let the four schedules run concurrently.
struct DeviceCtx {
  DeviceInfo info;
  cudaStream_t helper[3];
  cudaEvent_t fork, join[3];
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
  if ((e = prepare_block_kernel<1>()) != cudaSuccess) return e;
  if ((e = prepare_block_kernel<kMaxCluster>()) != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(kMaxCluster);
  cfg.blockDim = dim3(kBlockThreads);
  cfg.dynamicSmemBytes = block_smem_bytes<kMaxCluster>();
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = kMaxCluster;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  e = cudaOccupancyMaxActiveClusters(&info.cluster_max_active,
                                     k_fps_block<kMaxCluster, kBlockThreads, kBlockPairs>, &cfg);
  if (e != cudaSuccess) return e;
  if ((e = prepare_aux_kernels()) != cudaSuccess) return e;
  for (int i = 0; i < 3; ++i) {
    if ((e = cudaStreamCreateWithFlags(&ctx.helper[i], cudaStreamNonBlocking))) return e;
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

cudaError_t launch_fps(const Problem& pb, const Workspace& ws, cudaStream_t s, StageMark mark) {
  const int dev = current_device();
  if (dev < 0) return cudaErrorInvalidDevice;
  cudaError_t e = prepare(dev);
  if (e != cudaSuccess) return e;
  DeviceCtx& ctx = g_ctx[dev];
  const DeviceInfo& di = ctx.info;
  // Launch a schedule unless the size hint rules out every event it could get:
  // schedule q receives events above `lower[q]` (or above K when forced).
  const int hint = pb.max_event_hint;
  const int f = pb.force_schedule;
  const int lower[4] = {pb.K, kWarpCap, kCtaCap, kCtaSmemCap};
  bool run[4];
  for (int q = 0; q < 4; ++q) {
    const int lo = f >= q ? pb.K : lower[q];
    run[q] = (q == 3 || f <= q) && (hint == 0 || hint > lo);
  }

  std::lock_guard<std::mutex> lock(ctx.launch_mu);  // the fork/join events are shared per device
  const bool forked = run[1] || run[2] || run[3];
  if (forked && (e = cudaEventRecord(ctx.fork, s))) return e;
  for (int h = 0; h < 3; ++h) {
    if (!run[h + 1]) continue;
    cudaStream_t hs = ctx.helper[h];
    if ((e = cudaStreamWaitEvent(hs, ctx.fork, 0))) return e;
    mark(2 + h, 0, hs);
    if (h == 0) {
      count_launch();
      k_fps_cta<kCtaPairs><<<di.sm_count, 128, kCtaSmem, hs>>>(pb.coords, pb.offsets, pb.start_local, ws.list_cta,
                                                               ws.hdr, pb.K, pb.centroid_idx, pb.token_id,
                                                               pb.centroids);
      e = cudaGetLastError();
    } else if (h == 1) {
      e = launch_block<1>(pb, ws, kListCtaSmem, di.sm_count, hs);
    } else {
      const int groups = di.cluster_max_active > 0 ? di.cluster_max_active : 1;
      e = launch_block<kMaxCluster>(pb, ws, kListCluster, groups, hs);
    }
    if (e != cudaSuccess) return e;
    mark(2 + h, 1, hs);
    if ((e = cudaEventRecord(ctx.join[h], hs))) return e;
  }
  if (run[0]) {
    const int blocks = di.sm_count * (di.warp_blocks_per_sm > 0 ? di.warp_blocks_per_sm : 1);
    mark(1, 0, s);
    count_launch();
    k_fps_warp<kWarpPairs><<<blocks, kWarpBlock, kWarpSmem, s>>>(pb.coords, pb.offsets, pb.start_local,
                                                                 ws.list_warp, ws.hdr, pb.K, pb.centroid_idx,
                                                                 pb.token_id, pb.centroids);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    mark(1, 1, s);
  }
  for (int h = 0; h < 3; ++h)
    if (run[h + 1] && (e = cudaStreamWaitEvent(s, ctx.join[h], 0))) return e;
  return cudaSuccess;
}

}  // namespace fpstok
