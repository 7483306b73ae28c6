// Farthest point sampling fused with the Voronoi labels, three schedules.
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
// Schedules (chosen per event by the binning kernel):
//   warp    N <= 448     one warp per event, points held in registers
//                        (lane l owns points l + 32 j), shuffle-free
//                        arg-max with two redux.sync per step.
//   CTA     N <= 12288   one 512-thread CTA per event, points in shared
//                        memory as packed f32x2 pairs, distances and labels
//                        in registers, one barrier per step.
//   cluster N <= 196608  a 16-CTA thread-block cluster per event; every warp
//                        posts its candidate (key, index, position) into every
//                        CTA's shared memory over DSMEM, one barrier.cluster
//                        per step, then each warp reduces the posted entries.
#include <cooperative_groups.h>

#include "common.cuh"
#include "internal.h"

namespace cg = cooperative_groups;

namespace fpstok {

// ------------------------------------------------------------------ warp

template <int PPL>
__global__ void __launch_bounds__(128, 3) k_fps_warp(const float4* __restrict__ coords,
                                                  const int64_t* __restrict__ offsets,
                                                  const int32_t* __restrict__ start_local,
                                                  const int* __restrict__ list, WsHeader* hdr, int K,
                                                  int32_t* __restrict__ centroid_idx,
                                                  int32_t* __restrict__ token_id,
                                                  float4* __restrict__ centroids) {
  static_assert(PPL % 2 == 0 && PPL <= 32, "points per lane must be even and <= 32");
  constexpr int NP = PPL / 2;
  const int lane = threadIdx.x & 31;
  const int gw = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int nw = (gridDim.x * blockDim.x) >> 5;
  const int count = hdr->n_items[kListWarp];

  for (int w = gw; w < count; w += nw) {
    const int b = list[w];
    const int64_t off = offsets[b];
    const int n = (int)(offsets[b + 1] - off);
    const int npairs = (((n + 31) >> 5) + 1) >> 1;
    const float4* pts = coords + off;

    uint64_t X[NP], Y[NP], Z[NP], T[NP];
    float dist[PPL];
    int lab[PPL];
    unsigned taken = 0;  // bit j: slot j is selected or holds no point
#pragma unroll
    for (int p = 0; p < NP; ++p) {
      const int i0 = (2 * p) * 32 + lane, i1 = i0 + 32;
      float4 a = make_float4(0.f, 0.f, 0.f, 0.f), c = a;
      if (p < npairs) {
        if (i0 < n) a = ldg4(pts + i0);
        if (i1 < n) c = ldg4(pts + i1);
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

    int c = start_local ? start_local[b] : 0;
    float4 cc = ldg4(pts + c);
    for (int s = 0; s < K; ++s) {
      if (lane == 0) {
        centroid_idx[(int64_t)b * K + s] = (int32_t)(off + c);
        centroids[(int64_t)b * K + s] = cc;
      }
      if ((c & 31) == lane) taken |= 1u << (c >> 5);
      const Cent2 C = cent2(cc);
      float m = kEmptySlot;
#pragma unroll
      for (int p = 0; p < NP; ++p) {
        if (p < npairs) {
          const uint64_t d = dist2(X[p], Y[p], Z[p], T[p], C);
          relax(lo2(d), dist[2 * p], lab[2 * p], s);
          relax(hi2(d), dist[2 * p + 1], lab[2 * p + 1], s);
          m = fmaxf(m, fmaxf(dist[2 * p], dist[2 * p + 1]));
        }
      }
      if (s == K - 1) break;
      const int key = fkey(m);
      const int M = __reduce_max_sync(kFull, key);
      unsigned cand = 0xffffffffu;
      if (key == M) {
#pragma unroll
        for (int j = PPL - 1; j >= 0; --j)
          if (fkey(dist[j]) == M) cand = (unsigned)(j * 32 + lane);
      }
      unsigned idx = __reduce_min_sync(kFull, cand);
      if (M == 0) {  // only duplicates of chosen points remain
        const unsigned free_slots = ~taken & ((PPL == 32) ? 0xffffffffu : ((1u << PPL) - 1u));
        cand = free_slots ? (unsigned)((__ffs(free_slots) - 1) * 32 + lane) : 0xffffffffu;
        idx = __reduce_min_sync(kFull, cand);
      }
      c = (int)idx;
      cc = ldg4(pts + c);
    }
    if (token_id) {
#pragma unroll
      for (int j = 0; j < PPL; ++j) {
        const int i = j * 32 + lane;
        if (i < n) token_id[off + i] = lab[j];
      }
    }
  }
}

// ------------------------------------------------------------------ CTA / cluster

template <int CL, int NT, int PSP>
__global__ void __launch_bounds__(NT, 1) k_fps_block(const float4* __restrict__ coords,
                                                     const int64_t* __restrict__ offsets,
                                                     const int32_t* __restrict__ start_local,
                                                     const int* __restrict__ list, WsHeader* hdr,
                                                     int list_id, int K,
                                                     int32_t* __restrict__ centroid_idx,
                                                     int32_t* __restrict__ token_id,
                                                     float4* __restrict__ centroids) {
  static_assert(2 * PSP <= 32, "selected-slot mask is 32 bits");
  constexpr int NW = NT / 32;
  constexpr int E = CL * NW;
  extern __shared__ __align__(16) unsigned char smem_raw[];
  ulonglong2* sXY = reinterpret_cast<ulonglong2*>(smem_raw);  // [PSP][NT] packed (x, y)
  ulonglong2* sZT = sXY + PSP * NT;                           // [PSP][NT] packed (z, t)
  int2* xkey = reinterpret_cast<int2*>(sZT + PSP * NT);       // [2][E] (key, index)
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

    float dist[2 * PSP];
    int lab[2 * PSP];
    unsigned taken = 0;
#pragma unroll
    for (int p = 0; p < PSP; ++p) {
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
      if (i0 >= n) taken |= 1u << (2 * p);
      if (i1 >= n) taken |= 1u << (2 * p + 1);
    }

    int c = start_local ? start_local[b] : 0;
    float4 cc = ldg4(pts + c);
    for (int s = 0; s < K; ++s) {
      if (rank == 0 && tid == 0) {
        centroid_idx[(int64_t)b * K + s] = (int32_t)(off + c);
        centroids[(int64_t)b * K + s] = cc;
      }
      if (c % G == g) taken |= 1u << (c / G);
      const Cent2 C = cent2(cc);
      float m = kEmptySlot;
#pragma unroll
      for (int p = 0; p < PSP; ++p) {
        if (p < npairs) {
          const ulonglong2 xy = sXY[p * NT + tid];
          const ulonglong2 zt = sZT[p * NT + tid];
          const uint64_t d = dist2(xy.x, xy.y, zt.x, zt.y, C);
          relax(lo2(d), dist[2 * p], lab[2 * p], s);
          relax(hi2(d), dist[2 * p + 1], lab[2 * p + 1], s);
          m = fmaxf(m, fmaxf(dist[2 * p], dist[2 * p + 1]));
        }
      }
      if (s == K - 1) break;

      const int key = fkey(m);
      int wM;
      unsigned wcand = 0xffffffffu, widx;
      wM = __reduce_max_sync(kFull, key);
      if (key == wM) {
#pragma unroll
        for (int j = 2 * PSP - 1; j >= 0; --j)
          if (fkey(dist[j]) == wM) wcand = (unsigned)(g + G * j);
      }
      widx = __reduce_min_sync(kFull, wcand);
      float4 wpos = make_float4(0.f, 0.f, 0.f, 0.f);
      if (wM >= 0) wpos = local_pos(widx);
      post(wM, widx, wpos);
      barrier();
      int M;
      unsigned idx;
      gather(M, idx, cc);
      if (M == 0) {  // only duplicates of chosen points remain
        const unsigned free_slots = ~taken & ((2 * PSP == 32) ? 0xffffffffu : ((1u << (2 * PSP)) - 1u));
        unsigned cand = 0xffffffffu;
        if (free_slots) {
          const int j = __ffs(free_slots) - 1;
          if (j < 2 * npairs) cand = (unsigned)(g + G * j);
        }
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
      for (int j = 0; j < 2 * PSP; ++j) {
        const int i = g + G * j;
        if (j < 2 * npairs && i < n) token_id[off + i] = lab[j];
      }
    }
  }
  if constexpr (CL > 1) cg::this_cluster().sync();  // no CTA leaves while peers may post into it
}

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
  const int* list = list_id == kListCta ? ws.list_cta : ws.list_cluster;
  count_launch();
  return cudaLaunchKernelEx(&cfg, k_fps_block<CL, kBlockThreads, kBlockPairs>, pb.coords,
                            pb.offsets, pb.start_local, list, ws.hdr, list_id, pb.K, pb.centroid_idx,
                            pb.token_id, pb.centroids);
}

constexpr int kMaxDevices = 64;
static bool g_prepared[kMaxDevices];
static DeviceInfo g_info[kMaxDevices];

static int current_device() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return -1;
  return dev;
}

// One-time set-up per device: kernel attributes and occupancy figures.
static cudaError_t prepare(int dev) {
  if (g_prepared[dev]) return cudaSuccess;
  DeviceInfo info = {};
  cudaError_t e = cudaDeviceGetAttribute(&info.sm_count, cudaDevAttrMultiProcessorCount, dev);
  if (e != cudaSuccess) return e;
  e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&info.warp_blocks_per_sm, k_fps_warp<kWarpPPL>, 128, 0);
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
  info.ready = true;
  g_info[dev] = info;
  g_prepared[dev] = true;
  return cudaSuccess;
}

static const DeviceInfo g_none = {};

const DeviceInfo& device_info() {
  const int dev = current_device();
  if (dev < 0 || prepare(dev) != cudaSuccess) return g_none;
  return g_info[dev];
}

cudaError_t launch_fps(const Problem& pb, const Workspace& ws, cudaStream_t s, StageMark mark) {
  const DeviceInfo& di = device_info();
  if (!di.ready) return cudaErrorInitializationError;
  cudaError_t e;
  // Launch a schedule unless the size hint rules out every event it could get.
  const int hint = pb.max_event_hint;
  const int f = pb.force_schedule;
  const bool any_warp = f <= 0 && (hint == 0 || hint > pb.K);
  const bool any_cta = f <= 1 && (hint == 0 || hint > (f >= 1 ? pb.K : kWarpCap));
  const bool any_cluster = hint == 0 || hint > (f >= 2 ? pb.K : kCtaCap);
  if (any_warp) {
    const int blocks = di.sm_count * (di.warp_blocks_per_sm > 0 ? di.warp_blocks_per_sm : 1);
    mark(1, 0, s);
    count_launch();
    k_fps_warp<kWarpPPL><<<blocks, 128, 0, s>>>(pb.coords, pb.offsets, pb.start_local, ws.list_warp,
                                                ws.hdr, pb.K, pb.centroid_idx, pb.token_id,
                                                pb.centroids);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    mark(1, 1, s);
  }
  if (any_cta) {
    mark(2, 0, s);
    if ((e = launch_block<1>(pb, ws, kListCta, di.sm_count, s)) != cudaSuccess) return e;
    mark(2, 1, s);
  }
  if (any_cluster) {
    const int groups = di.cluster_max_active > 0 ? di.cluster_max_active : 1;
    mark(3, 0, s);
    if ((e = launch_block<kMaxCluster>(pb, ws, kListCluster, groups, s)) != cudaSuccess) return e;
    mark(3, 1, s);
  }
  return cudaSuccess;
}

}  // namespace fpstok
