// Charge-weighted token summaries (graphnet PR #923, review thread on the
// no-charge case: the tokenizer uses the charge for weighting and for token
// summaries, unit charge without a charge column).  Per Voronoi token j of
// event b, with q = feats[:, charge_col] (or 1):
//   wsum = sum q,  wcoords = sum q * coords / wsum,  wfeats = sum q * feats / wsum,
// float64 sums, means 0 for an empty cell or wsum <= 0, each output rounded
// once to float32.
//
// k_token_sums gives every CTA one contiguous range of points (the whole
// array split evenly over the grid), so that the inputs stream through once.
// The CTA walks the events that meet its range; for each it takes the
// event's points in tiles: rows staged in shared memory, a counting sort by
// token, then one thread per (token, group of values) adds its points' q and
// q-weighted values in float64 registers and once into the event's
// accumulators [K, 5 + F] in shared memory (no atomics).  It then writes the
// event's means directly when the event lies inside its range, or else its
// partial sums into its own slot of the workspace.  k_token_finalize then adds, per event cut by a
// range boundary, the partial sums of the CTAs it spans in CTA order.
#include "../../include/fpstok.h"
#include "common.cuh"
#include "internal.h"
#include "token_summary.h"

namespace fpstok {

namespace {

constexpr int kSumThreads = 256;
constexpr int kSumTile = 1024;                   // points staged and sorted at a time
constexpr int kSumGroup = 8;                     // features summed together by one thread
constexpr int kSumMinPoints = 1024;              // points per CTA at least
constexpr int kSumMaxCtas = 512;                 // CTAs (partial-sum slots) at most
constexpr int kSumCtasPerSm = 3;                 // resident CTAs per SM (shared memory at K = 128, F <= 8)
constexpr int64_t kSumPartialBudget = 32ll << 20;  // bytes of partial sums at most

// First event b >= lo whose span ends after point p (offsets[b + 1] > p),
// searching [lo, hi]; hi when none.
__device__ __forceinline__ int sum_first_event_after(const int64_t* __restrict__ offsets, int lo, int hi,
                                                     int64_t p) {
  while (lo < hi) {
    const int mid = (lo + hi) >> 1;
    if (__ldg(offsets + mid + 1) > p) hi = mid;
    else lo = mid + 1;
  }
  return lo;
}

__global__ void __launch_bounds__(kSumThreads) k_token_sums(const float4* __restrict__ coords,
                                                            const float* __restrict__ feats, int F, int charge_col,
                                                            const int64_t* __restrict__ offsets, int B, int64_t P,
                                                            int K, const int32_t* __restrict__ token_id,
                                                            int64_t chunk, float* __restrict__ wsum,
                                                            float* __restrict__ wcoords, float* __restrict__ wfeats,
                                                            double* __restrict__ partial, WsHeader* hdr) {
  // the boundary kernel may be launched now; it waits for this one's sums
  asm volatile("griddepcontrol.launch_dependents;");
  extern __shared__ __align__(16) unsigned char s_raw[];
  const int V = 5 + F;
  const int KV = K * V;
  const bool staged = F <= kSumGroup;
  float4* s_c = reinterpret_cast<float4*>(s_raw);                        // [tile] coordinates (16-byte copies)
  double* s_acc = reinterpret_cast<double*>(s_c + kSumTile);              // [K, V]
  float* s_q = reinterpret_cast<float*>(s_acc + KV);                      // [tile] charges
  int* s_lab = reinterpret_cast<int*>(s_q + kSumTile);                    // [tile] tokens (-1: none)
  int* s_perm = s_lab + kSumTile;                                         // [tile] points sorted by token
  int* s_cnt = s_perm + kSumTile;                                         // [256] counts, [256] starts,
  int* s_start = s_cnt + 256;                                             // [256] fill cursors
  int* s_cur = s_start + 256;
  float* s_f = reinterpret_cast<float*>(s_cur + 256);                     // [tile, F] when staged
  const int NG = 1 + (F + kSumGroup - 1) / kSumGroup;  // value groups: (q, q*coords), then features
  const int tid = threadIdx.x;
  const bool last_cta = blockIdx.x == gridDim.x - 1;
  const int64_t p0 = (int64_t)blockIdx.x * chunk;
  const int64_t p1 = last_cta ? P : min(P, p0 + chunk);
  if (blockIdx.x == 0 && tid == 0 && (offsets[0] != 0 || offsets[B] != P)) record_error(hdr, kDevBadOffsets);
  // the event holding point p0, preceded by the empty events that start at p0
  int b = sum_first_event_after(offsets, 0, B - 1, p0);
  while (b > 0 && offsets[b - 1] >= p0 && offsets[b] == p0) --b;
  for (; b < B; ++b) {
    const int64_t e0 = offsets[b], e1 = offsets[b + 1];
    if (e0 >= p1 && !(last_cta && e0 == P)) break;  // the next range's events
    if (e1 < e0 || e0 < 0 || e1 > P) {
      if (tid == 0) record_error(hdr, kDevBadOffsets);
      continue;
    }
    const int64_t s0 = max(e0, p0), s1 = min(e1, p1);
    for (int e = tid; e < KV; e += kSumThreads) s_acc[e] = 0.0;
    for (int64_t t0 = s0; t0 < s1; t0 += kSumTile) {
      const int n = (int)min((int64_t)kSumTile, s1 - t0);
      // the tile's rows into shared memory by asynchronous copies, in flight
      // while the tokens are loaded and counted
      for (int j = tid; j < K; j += kSumThreads) s_cnt[j] = 0;
      const uint32_t sc0 = (uint32_t)__cvta_generic_to_shared(s_c);
#pragma unroll 4
      for (int li = tid; li < n; li += kSumThreads)
        asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(sc0 + 16u * (uint32_t)li), "l"(coords + t0 + li)
                     : "memory");
      if (staged) {
        const float* fr = feats + t0 * F;
        const uint32_t sf0 = (uint32_t)__cvta_generic_to_shared(s_f);
#pragma unroll 8
        for (int e = tid; e < n * F; e += kSumThreads)
          asm volatile("cp.async.ca.shared.global [%0], [%1], 4;" ::"r"(sf0 + 4u * (uint32_t)e), "l"(fr + e)
                       : "memory");
      }
      asm volatile("cp.async.commit_group;" ::: "memory");
      __syncthreads();  // counts zeroed
#pragma unroll 4
      for (int li = tid; li < n; li += kSumThreads) {
        const int64_t i = t0 + li;
        int t = token_id[i];
        if (t < -1 || t >= K) {
          record_error(hdr, kDevBadToken);
          t = -1;
        }
        s_lab[li] = t;
        if (!staged) s_q[li] = charge_col >= 0 ? __ldg(feats + i * F + charge_col) : 1.f;
        if (t >= 0) atomicAdd(&s_cnt[t], 1);
      }
      asm volatile("cp.async.wait_group 0;" ::: "memory");
      __syncthreads();
      if (staged)
        for (int li = tid; li < n; li += kSumThreads) s_q[li] = charge_col >= 0 ? s_f[li * F + charge_col] : 1.f;
      if (tid < 32) count_scan(s_cnt, s_start, s_cur, K, tid);
      __syncthreads();
      for (int li = tid; li < n; li += kSumThreads) {
        const int t = s_lab[li];
        if (t >= 0) s_perm[atomicAdd(&s_cur[t], 1)] = li;
      }
      __syncthreads();
      // one thread per (token, value group): its points in sorted order,
      // float64 sums in registers, added once into the token's accumulators
      for (int it = tid; it < K * NG; it += kSumThreads) {
        const int j = it / NG, g = it - j * NG;
        const int c = s_cnt[j];
        if (c == 0) continue;
        const int* pj = s_perm + s_start[j];
        double a[kSumGroup];
#pragma unroll
        for (int v = 0; v < kSumGroup; ++v) a[v] = 0.0;
        double* dst = s_acc + j * V;
        if (g == 0) {
          for (int m = 0; m < c; ++m) {
            const int li = pj[m];
            const double q = (double)s_q[li];
            const float4 p = s_c[li];
            a[0] += q;
            a[1] += q * (double)p.x;
            a[2] += q * (double)p.y;
            a[3] += q * (double)p.z;
            a[4] += q * (double)p.w;
          }
#pragma unroll
          for (int v = 0; v < 5; ++v) dst[v] += a[v];
        } else {
          const int f0 = (g - 1) * kSumGroup;
          const int nf = min(kSumGroup, F - f0);
          for (int m = 0; m < c; ++m) {
            const int li = pj[m];
            const double q = (double)s_q[li];
            const float* row = staged ? s_f + li * F + f0 : feats + (t0 + li) * F + f0;
#pragma unroll
            for (int v = 0; v < kSumGroup; ++v)
              if (v < nf) a[v] += q * (double)row[v];
          }
#pragma unroll
          for (int v = 0; v < kSumGroup; ++v)
            if (v < nf) dst[5 + f0 + v] += a[v];
        }
      }
      __syncthreads();
    }
    if (s0 >= s1) __syncthreads();  // (no tile ran: the zeroing must still finish)
    if (e0 >= p0 && e1 <= p1) {  // the whole event lies in this range: its means
      for (int e = tid; e < KV; e += kSumThreads) {
        const int j = e / V, v = e - j * V;
        const double W = s_acc[j * V];
        const int64_t r = (int64_t)b * K + j;
        if (v == 0) wsum[r] = (float)W;
        else if (v < 5) wcoords[r * 4 + (v - 1)] = W > 0.0 ? (float)(s_acc[e] / W) : 0.f;
        else wfeats[r * F + (v - 5)] = W > 0.0 ? (float)(s_acc[e] / W) : 0.f;
      }
    } else {  // cut by a range boundary: slot 1 when it starts here, else slot 0
      double* dst = partial + ((int64_t)blockIdx.x * 2 + (e0 >= p0 ? 1 : 0)) * KV;
      for (int e = tid; e < KV; e += kSumThreads) dst[e] = s_acc[e];
    }
    __syncthreads();
  }
}

// One CTA per range boundary c * chunk (c = 1 .. G-1).  An event cut by
// nb boundaries gets nb CTAs, each taking a slice of its K (5 + F) values.
// Per block of up to 256 values the CTA's threads split the ranges the
// event spans into S consecutive groups, sum each group in range order, and
// one thread per value adds the group sums in group order: a fixed order,
// with the loads of all groups in flight together.
__global__ void __launch_bounds__(256) k_token_finalize(const int64_t* __restrict__ offsets, int B, int64_t P,
                                                        int K, int F, int64_t chunk, int G,
                                                        const double* __restrict__ partial,
                                                        float* __restrict__ wsum, float* __restrict__ wcoords,
                                                        float* __restrict__ wfeats) {
  __shared__ double s_w[256], s_x[256];
  const int c = blockIdx.x + 1;
  const int64_t p = (int64_t)c * chunk;
  if (p >= P) return;
  const int b = sum_first_event_after(offsets, 0, B - 1, p);
  const int64_t e0 = offsets[b], e1 = offsets[b + 1];
  if (!(e0 < p && p < e1) || e0 < 0 || e1 > P) return;  // no event is cut here (uniform)
  const int cf = (int)(e0 / chunk);
  const int cl = (int)min((int64_t)G - 1, (e1 - 1) / chunk);
  const int nb = cl - cf;        // boundaries inside the event: one CTA each
  const int slice = c - cf - 1;  // this CTA's share of the values
  const int V = 5 + F;
  const int KV = K * V;
  const int R = cl - cf + 1;     // ranges the event spans
  const int lo = (int)((int64_t)KV * slice / nb), hi = (int)((int64_t)KV * (slice + 1) / nb);
  // launched as the sums kernel's programmatic dependent: the search above
  // ran while it finished; its partial sums are read from here on
  asm volatile("griddepcontrol.wait;" ::: "memory");
  const int tid = threadIdx.x;
  for (int v0 = lo; v0 < hi; v0 += 256) {
    const int nv = min(256, hi - v0);
    const int S = min(R, 256 / nv);      // range groups
    const int per = (R + S - 1) / S;     // ranges per group
    if (tid < nv * S) {
      const int ev = tid % nv, grp = tid / nv;
      const int e = v0 + ev, j = e / V;
      const int r0 = cf + grp * per, r1 = min(cl + 1, r0 + per);
      double W = 0.0, x = 0.0;
#pragma unroll 4
      for (int r = r0; r < r1; ++r) {
        const double* src = partial + ((int64_t)r * 2 + (r == cf ? 1 : 0)) * KV;
        W += src[j * V];
        x += src[e];
      }
      s_w[tid] = W;
      s_x[tid] = x;
    }
    __syncthreads();
    if (tid < nv) {
      const int e = v0 + tid, j = e / V, v = e - j * V;
      double W = 0.0, x = 0.0;
      for (int g = 0; g < S; ++g) {
        W += s_w[g * nv + tid];
        x += s_x[g * nv + tid];
      }
      const int64_t row = (int64_t)b * K + j;
      if (v == 0) wsum[row] = (float)W;
      else if (v < 5) wcoords[row * 4 + (v - 1)] = W > 0.0 ? (float)(x / W) : 0.f;
      else wfeats[row * F + (v - 5)] = W > 0.0 ? (float)(x / W) : 0.f;
    }
    __syncthreads();
  }
}

// Shared memory of k_token_sums: the tile's coordinates, the accumulators,
// the tile's charges, tokens and counting sort, and its feature rows.
size_t token_sums_smem(int K, int F) {
  return (size_t)K * (5 + F) * sizeof(double) + (size_t)kSumTile * (sizeof(float4) + sizeof(float) + 2 * sizeof(int)) +
         3 * 256 * sizeof(int) + (F <= kSumGroup ? (size_t)kSumTile * F * sizeof(float) : 0);
}

}  // namespace

int token_summary_ctas(int K, int F) {
  const int64_t per = 2ll * K * (5 + F) * (int64_t)sizeof(double);
  int64_t g = per > 0 ? kSumPartialBudget / per : kSumMaxCtas;
  if (g > kSumMaxCtas) g = kSumMaxCtas;
  return g < 1 ? 1 : (int)g;
}

size_t token_summary_partial_bytes(int K, int F) {
  return (size_t)token_summary_ctas(K, F) * 2 * K * (5 + F) * sizeof(double);
}

cudaError_t launch_token_summaries(const float* coords, const float* feats, int F, int charge_col,
                                   const int64_t* offsets, int B, int64_t P, int K, const int32_t* token_id,
                                   double* partial, float* wsum, float* wcoords, float* wfeats, WsHeader* hdr,
                                   cudaStream_t s) {
  int64_t G = (P + kSumMinPoints - 1) / kSumMinPoints;
  if (G > token_summary_ctas(K, F)) G = token_summary_ctas(K, F);
  const int64_t resident = (int64_t)device_info().sm_count * kSumCtasPerSm;  // one wave
  if (G > resident) G = resident;
  if (G < 1) G = 1;
  const int64_t chunk = P > 0 ? (P + G - 1) / G : 1;
  const size_t smem = token_sums_smem(K, F);
  static bool attr_set[64] = {};
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev >= 0 && dev < 64 && !attr_set[dev]) {
    const int most = (int)token_sums_smem(FPS_MAX_K, FPS_MAX_F);
    if ((e = cudaFuncSetAttribute(k_token_sums, cudaFuncAttributeMaxDynamicSharedMemorySize, most))) return e;
    attr_set[dev] = true;
  }
  count_launch();
  k_token_sums<<<(unsigned)G, kSumThreads, smem, s>>>(reinterpret_cast<const float4*>(coords), feats, F, charge_col,
                                                      offsets, B, P, K, token_id, chunk, wsum, wcoords, wfeats,
                                                      partial, hdr);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  if (G > 1) {
    count_launch();
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)(G - 1));
    cfg.blockDim = dim3(256);
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    e = cudaLaunchKernelEx(&cfg, k_token_finalize, offsets, B, P, K, F, chunk, (int)G, (const double*)partial, wsum,
                           wcoords, wfeats);
  }
  return e;
}

}  // namespace fpstok
