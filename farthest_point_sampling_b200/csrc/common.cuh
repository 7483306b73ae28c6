// Device-side building blocks shared by the fpstok kernels (sm_100a only).
//
// The squared distance follows the tokenizer's fixed float32 contract:
// d(i, c) = ((dx*dx + dy*dy) + dz*dz) + dt*dt, every operation rounded to
// nearest-even and never fused (4D (x, y, z, t) points: graphnet PR #923 "Add
// Neptune point-transformer backbone", Summary; float32 only: same page,
// review thread on the FPS `precision` argument).  Two points are evaluated
// at once with the packed f32x2 instructions of sm_100a: each lane of a pair
// is an ordinary IEEE round-to-nearest float32 operation, so the result is
// bit-identical to the scalar formula while using half the issue slots.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#if defined(__CUDA_ARCH__) && (__CUDA_ARCH__ < 1000)
#error "fpstok kernels are written for sm_100a (B200) only"
#endif

namespace fpstok {

constexpr int kWarp = 32;
constexpr int FPS_MAX_K_DEV = 256;  // FPS_MAX_K of the C ABI
constexpr unsigned kFull = 0xffffffffu;
// Running-minimum value of a slot that holds no point: negative, so it never
// wins the arg-max (whose keys are the bit patterns of non-negative floats).
constexpr float kEmptySlot = -1.0f;

// Device status codes (match FPS_DEV_* in fpstok.h).
constexpr int kDevBadOffsets = 1;
constexpr int kDevBadStart = 2;
constexpr int kDevBadToken = 3;
constexpr int kDevTooLarge = 4;
constexpr int kDevExchangeTimeout = 5;

// Workspace header: status word, detail word, work-list sizes and the
// cursors the persistent kernels take items from (all reset by the binning
// kernel at the start of every call).
struct WsHeader {
  int status;
  int detail;
  int n_items[14];  // per work list
  int next_item[8];  // per schedule: next unclaimed item
};

__device__ __forceinline__ void record_error(WsHeader* h, int code) {
  atomicCAS(&h->status, 0, code);
}

// ---------------------------------------------------------------- packed f32x2

__device__ __forceinline__ uint64_t pack2(float lo, float hi) {
  return (uint64_t)__float_as_uint(lo) | ((uint64_t)__float_as_uint(hi) << 32);
}
__device__ __forceinline__ float lo2(uint64_t v) { return __uint_as_float((uint32_t)v); }
__device__ __forceinline__ float hi2(uint64_t v) { return __uint_as_float((uint32_t)(v >> 32)); }

__device__ __forceinline__ uint64_t sub2(uint64_t a, uint64_t b) {
  uint64_t d;
  asm("sub.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}
__device__ __forceinline__ uint64_t mul2(uint64_t a, uint64_t b) {
  uint64_t d;
  asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}
__device__ __forceinline__ uint64_t add2(uint64_t a, uint64_t b) {
  uint64_t d;
  asm("add.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}

// A centroid broadcast into both halves of four packed registers.
struct __align__(16) Cent2 {
  uint64_t x, y, z, t;
};
__device__ __forceinline__ Cent2 cent2(float4 c) {
  return Cent2{pack2(c.x, c.x), pack2(c.y, c.y), pack2(c.z, c.z), pack2(c.w, c.w)};
}

// A packed zero the compiler cannot prove to be zero: a volatile load of a
// device variable that is never written.  ptxas merges a packed multiply
// that feeds a packed add into one fused multiply-add even with contraction
// disabled (-fmad=false, .rn), which rounds d*d + s once instead of twice.
// The squares are therefore formed as fma(d, d, z) with this runtime zero:
// d*d + 0 rounds exactly like d*d, and an FMA whose addend is an unknown
// register is not merged with the add that follows.
static __device__ uint64_t g_opaque_zero2;
__device__ __forceinline__ uint64_t opaque_zero2() { return *reinterpret_cast<volatile uint64_t*>(&g_opaque_zero2); }

// d * d of both lanes, rounded once each (z: opaque_zero2()).
__device__ __forceinline__ uint64_t sq2(uint64_t d, uint64_t z) {
  uint64_t r;
  asm("fma.rn.f32x2 %0, %1, %1, %2;" : "=l"(r) : "l"(d), "l"(z));
  return r;
}

// Distances of two points (packed component-wise) to one centroid:
// ((dx*dx + dy*dy) + dz*dz) + dt*dt per lane, every operation rounded to
// nearest on its own (z: opaque_zero2()).
__device__ __forceinline__ uint64_t dist2(uint64_t X, uint64_t Y, uint64_t Z, uint64_t T,
                                          const Cent2& c, uint64_t z) {
  uint64_t dx = sub2(X, c.x);
  uint64_t dy = sub2(Y, c.y);
  uint64_t dz = sub2(Z, c.z);
  uint64_t dt = sub2(T, c.t);
  uint64_t s = add2(sq2(dx, z), sq2(dy, z));
  s = add2(s, sq2(dz, z));
  s = add2(s, sq2(dt, z));
  return s;
}

// Scalar form of the same distance.
__device__ __forceinline__ float dist1(float4 p, float4 c) {
  float dx = __fsub_rn(p.x, c.x);
  float dy = __fsub_rn(p.y, c.y);
  float dz = __fsub_rn(p.z, c.z);
  float dt = __fsub_rn(p.w, c.w);
  float s = __fadd_rn(__fmul_rn(dx, dx), __fmul_rn(dy, dy));
  s = __fadd_rn(s, __fmul_rn(dz, dz));
  s = __fadd_rn(s, __fmul_rn(dt, dt));
  return s;
}

// A point under the per-axis scale of the distance: each coordinate times
// its weight, rounded to nearest on its own (scalar multiplies, which ptxas
// never fuses into the subtract that follows).  w = (1, 1, 1, 1) returns the
// same bits.
__device__ __forceinline__ float4 scale4(float4 p, float4 w) {
  return make_float4(__fmul_rn(p.x, w.x), __fmul_rn(p.y, w.y), __fmul_rn(p.z, w.z), __fmul_rn(p.w, w.w));
}

// Running-min / label update of one slot: strict '<' so that, over slots
// visited in increasing order, the lowest slot wins ties.
__device__ __forceinline__ void relax(float d, float& dist, int& lab, int s) {
  lab = d < dist ? s : lab;
  dist = fminf(dist, d);
}

__device__ __forceinline__ int fkey(float v) { return __float_as_int(v); }

// Three-input float32 maximum (sm_100): one instruction for two new values.
__device__ __forceinline__ float max3f(float a, float b, float c) {
  float d;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
  return d;
}

// Three-input float32 minimum (sm_100).
__device__ __forceinline__ float min3f(float a, float b, float c) {
  float d;
  asm("min.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
  return d;
}

// Largest of the per-pair maxima pm[0 .. NP) of one lane (two interleaved
// three-input chains, so the depth is about NP / 4).
template <int NP>
__device__ __forceinline__ float lane_max(const float (&pm)[NP]) {
  float a = pm[0], b = NP > 1 ? pm[1] : kEmptySlot;
#pragma unroll
  for (int p = 2; p < NP; p += 4) {
    a = p + 1 < NP ? max3f(a, pm[p], pm[p + 1]) : fmaxf(a, pm[p]);
    if (p + 2 < NP) b = p + 3 < NP ? max3f(b, pm[p + 2], pm[p + 3]) : fmaxf(b, pm[p + 2]);
  }
  return fmaxf(a, b);
}

// The lane's lowest slot holding the arg-max key M: slots 2p and 2p+1 are
// the two halves of packed pair p (lower slot = lower point index), pm[p] the
// larger of their running minima.  One pass over the pairs from the top (so
// the lowest pair wins) selects the pair and the value of its low half with
// one compare; the low half wins when it holds M.  Returns the slot, or -1
// when no slot of this lane holds M.
template <int NP>
__device__ __forceinline__ int lane_first_slot(const float (&pm)[NP], const float (&dist)[2 * NP], int M) {
  int cp = -1;
  float lo = 0.f;
#pragma unroll
  for (int p = NP - 1; p >= 0; --p) {
    const bool h = fkey(pm[p]) == M;
    cp = h ? p : cp;
    lo = h ? dist[2 * p] : lo;
  }
  return cp < 0 ? -1 : 2 * cp + (fkey(lo) == M ? 0 : 1);
}

// Centroid position stored with every component duplicated, so that two
// 128-bit shared-memory loads give the four packed registers of Cent2.
struct DupPoint {
  uint4 xy;  // (x, x, y, y)
  uint4 zt;  // (z, z, t, t)
};
__device__ __forceinline__ DupPoint dup_point(float4 a) {
  return DupPoint{make_uint4(__float_as_uint(a.x), __float_as_uint(a.x), __float_as_uint(a.y), __float_as_uint(a.y)),
                  make_uint4(__float_as_uint(a.z), __float_as_uint(a.z), __float_as_uint(a.w), __float_as_uint(a.w))};
}
__device__ __forceinline__ Cent2 cent2_dup(const DupPoint& p) {
  return Cent2{(uint64_t)p.xy.x | ((uint64_t)p.xy.y << 32), (uint64_t)p.xy.z | ((uint64_t)p.xy.w << 32),
               (uint64_t)p.zt.x | ((uint64_t)p.zt.y << 32), (uint64_t)p.zt.z | ((uint64_t)p.zt.w << 32)};
}
__device__ __forceinline__ float4 dup_to_float4(const DupPoint& p) {
  return make_float4(__uint_as_float(p.xy.x), __uint_as_float(p.xy.z), __uint_as_float(p.zt.x),
                     __uint_as_float(p.zt.z));
}

// Warp arg-max of (key, idx): the largest key, then the smallest idx among
// the lanes holding it.  Both results are warp-uniform.
__device__ __forceinline__ void warp_argmax(int key, unsigned idx, int& mkey, unsigned& midx) {
  mkey = __reduce_max_sync(kFull, key);
  midx = __reduce_min_sync(kFull, key == mkey ? idx : 0xffffffffu);
}

__device__ __forceinline__ float4 ldg4(const float4* p) { return __ldg(p); }

// ---------------------------------------------------------------- per-token sums

// Exclusive prefix sum of cnt[0 .. K) into start[] and cur[] by one warp
// (lane = rank < 32), 8 entries per lane; K <= 256.
__device__ __forceinline__ void count_scan(const int* cnt, int* start, int* cur, int K, int lane) {
  int local[8];
  int sum = 0;
#pragma unroll
  for (int q = 0; q < 8; ++q) {
    const int j = lane * 8 + q;
    local[q] = j < K ? cnt[j] : 0;
    sum += local[q];
  }
  int x = sum;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(kFull, x, o);
    if (lane >= o) x += y;
  }
  int run = x - sum;
#pragma unroll
  for (int q = 0; q < 8; ++q) {
    const int j = lane * 8 + q;
    if (j < K) {
      start[j] = run;
      cur[j] = run;
    }
    run += local[q];
  }
}

// Counting sort of npts labelled points by a group of threads (a warp or a
// CTA; `rank` / `size` are this thread's index in it and its size, `sync` its
// barrier): cnt[j] = number of points labelled j, start[j] = exclusive prefix
// sum, perm[start[j] .. start[j] + cnt[j]) = the local indices of those
// points and slab[] the token of every sorted position.  Labels outside
// [0, K) are left out (the sorted range then ends before npts).  K <= 256.
// All arrays are in shared memory; cur[K] is scratch.
template <typename Sync>
__device__ __forceinline__ void label_sort(const int* lab, int npts, int K, int* cnt, int* start, int* cur,
                                           int* perm, int* slab, int rank, int size, Sync sync) {
  for (int j = rank; j < K; j += size) cnt[j] = 0;
  sync();
  for (int i = rank; i < npts; i += size) {
    const int l = lab[i];
    if ((unsigned)l < (unsigned)K) atomicAdd(&cnt[l], 1);
  }
  sync();
  if (rank < 32) count_scan(cnt, start, cur, K, rank);
  sync();
  for (int i = rank; i < npts; i += size) {
    const int l = lab[i];
    if ((unsigned)l < (unsigned)K) {
      const int pos = atomicAdd(&cur[l], 1);
      perm[pos] = i;
      slab[pos] = l;
    }
  }
  sync();
}

// Per-token float64 sums over the first nsorted positions of a counting
// sort, balanced over the group: every thread takes an equal run of sorted
// positions, adds val(i, v) for v < V along it and flushes its partial sums
// into acc[token * V + v] (shared memory, zeroed beforehand) whenever the
// token changes and at the end of its run.  V <= 8 per call.
template <typename Val>
__device__ __forceinline__ void segment_sums(const int* perm, const int* slab, int nsorted, int V, int v0,
                                             int ldacc, double* acc, int rank, int size, Val val) {
  const int per = (nsorted + size - 1) / size;
  const int p0 = rank * per, p1 = min(nsorted, p0 + per);
  if (p0 >= p1) return;
  double s[8];
#pragma unroll
  for (int v = 0; v < 8; ++v) s[v] = 0.0;
  int cur = slab[p0];
  for (int q = p0; q < p1; ++q) {
    const int i = perm[q];
    const int l = slab[q];
    if (l != cur) {
#pragma unroll
      for (int v = 0; v < 8; ++v)
        if (v < V) {
          atomicAdd(&acc[cur * ldacc + v0 + v], s[v]);
          s[v] = 0.0;
        }
      cur = l;
    }
#pragma unroll
    for (int v = 0; v < 8; ++v)
      if (v < V) s[v] += val(i, v0 + v);
  }
#pragma unroll
  for (int v = 0; v < 8; ++v)
    if (v < V) atomicAdd(&acc[cur * ldacc + v0 + v], s[v]);
}

// Per-token float64 sums, warp-tile form (for cheap val() reads such as
// staged shared memory): each warp of the group takes tiles of 32 consecutive sorted
// positions, forms a segmented inclusive scan of val(i, v) over the lanes of
// each token with shuffles, and the last lane of every token in the tile adds
// the tile's partial sum into acc[token * ldacc + v] (shared memory, zeroed
// beforehand).  A token therefore gets one atomic per tile it spans, not one
// per point.  The group size is a multiple of 32; v runs over [v0, v0 + V).
template <typename Val>
__device__ __forceinline__ void segment_sums_scan(const int* perm, const int* slab, int nsorted, int V, int v0,
                                             int ldacc, double* acc, int rank, int size, Val val) {
  const int lane = rank & 31, warp = rank >> 5, nwarps = size >> 5;
  for (int tile = warp * 32; tile < nsorted; tile += nwarps * 32) {
    const int q = tile + lane;
    const bool valid = q < nsorted;
    const int tok = valid ? slab[q] : -1 - lane;  // empty lanes form singleton segments
    const int i = valid ? perm[q] : 0;
    // every lane takes part in every shuffle: none sits behind a short-circuit
    const int next_tok = __shfl_down_sync(kFull, tok, 1);
    const bool last = valid && (lane == 31 || next_tok != tok);
    bool same[5];
#pragma unroll
    for (int k = 0; k < 5; ++k) {
      const int o = 1 << k;
      const int up_tok = __shfl_up_sync(kFull, tok, o);
      same[k] = lane >= o && up_tok == tok;
    }
    for (int v = 0; v < V; ++v) {
      double x = valid ? val(i, v0 + v) : 0.0;
#pragma unroll
      for (int k = 0; k < 5; ++k) {
        const double y = __shfl_up_sync(kFull, x, 1 << k);
        if (same[k]) x += y;
      }
      if (last) atomicAdd(&acc[tok * ldacc + v0 + v], x);
    }
  }
}

}  // namespace fpstok
