// In-run FP32 rate microbenchmark for the roofline of the FPS kernels.
//
// The FPS distance ((dx*dx + dy*dy) + dz*dz) + dt*dt is made of separately
// rounded float32 subtracts, multiplies and adds, so its ceiling is the rate
// of non-FMA FP32 operations.  Each mode runs independent dependency chains
// (8 per thread, so latency is hidden) on every SM:
//   0  scalar FMUL + FADD (round-to-nearest intrinsics, never fused)
//   1  packed f32x2 adds only
//   2  packed f32x2 multiplies only
//   3  packed f32x2 fused multiply-adds with a register addend (2 ops each)
//   4  the packed distance exactly as the FPS kernels compute it (squares as
//      FMAs with a runtime zero addend, see common.cuh), 11 ops per lane.
//      Every one of its four coordinate inputs is loop-carried: each chain
//      holds (X, Y, Z, T) and every distance overwrites one of them from all
//      four, so no subtract or square can be hoisted out of the loop and the
//      11 counted operations are the instructions issued.
// A packed multiply feeding a packed add is merged into one FMA by ptxas, so
// modes 1 and 2 keep the two operations in separate chains.  The result is
// stored only when an impossible value appears, which keeps the work alive.
// No mode can exceed the issue ceiling of one packed instruction per
// scheduler per clock (148 SMs x 4 x 64 lane-ops x clock); the non-FMA modes
// are bounded by half of it, one float32 operation per lane per clock.
#include <cuda_runtime.h>
#include <stdint.h>

namespace {

__device__ __forceinline__ uint64_t mul2(uint64_t a, uint64_t b) {
  uint64_t d;
  asm volatile("mul.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}
__device__ __forceinline__ uint64_t add2(uint64_t a, uint64_t b) {
  uint64_t d;
  asm volatile("add.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}
__device__ __forceinline__ uint64_t sub2(uint64_t a, uint64_t b) {
  uint64_t d;
  asm volatile("sub.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}
__device__ __forceinline__ uint64_t fma2(uint64_t a, uint64_t b, uint64_t c) {
  uint64_t d;
  asm volatile("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
  return d;
}

__device__ uint64_t g_zero2;  // never written: a zero the compiler cannot see

__device__ __forceinline__ uint64_t pk(float lo, float hi) {
  return (uint64_t)__float_as_uint(lo) | ((uint64_t)__float_as_uint(hi) << 32);
}
__device__ __forceinline__ uint64_t splat(float v) { return pk(v, v); }

__global__ void k_scalar(float* out, int iters, float seed) {
  float a[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) a[i] = seed + (float)(threadIdx.x + i);
  const float m = 0.999999f, c = 1e-7f;
  for (int it = 0; it < iters; ++it) {
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      a[i] = __fmul_rn(a[i], m);
      a[i] = __fadd_rn(a[i], c);
    }
  }
  float s = 0.f;
#pragma unroll
  for (int i = 0; i < 8; ++i) s += a[i];
  if (s == -1.2345f) out[blockIdx.x] = s;
}

template <int MODE>
__global__ void k_packed(float* out, int iters, float seed) {
  uint64_t a[8];
  const float base = seed + (float)threadIdx.x;
#pragma unroll
  for (int i = 0; i < 8; ++i) a[i] = pk(base + i, base - i);
  const uint64_t m = splat(0.999999f), c = splat(1e-7f);
  for (int it = 0; it < iters; ++it) {
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      if (MODE == 1) {
        a[i] = add2(a[i], c);
        a[i] = add2(a[i], m);
      } else if (MODE == 2) {
        a[i] = mul2(a[i], m);
        a[i] = mul2(a[i], m);
      } else {
        a[i] = fma2(a[i], m, c);
        a[i] = fma2(a[i], m, c);
      }
    }
  }
  float s = 0.f;
#pragma unroll
  for (int i = 0; i < 8; ++i) s += __uint_as_float((uint32_t)a[i]) + __uint_as_float((uint32_t)(a[i] >> 32));
  if (s == -1.2345f) out[blockIdx.x] = s;
}

// The exact packed distance of (X, Y, Z, T) to a fixed centroid, squares as
// FMAs with the runtime zero z (as in the FPS kernels).
__device__ __forceinline__ uint64_t dist_link(uint64_t X, uint64_t Y, uint64_t Z, uint64_t T, uint64_t z) {
  const uint64_t cx = 0x3f0000003f000000ull, cy = 0xbe800000be800000ull;  // (0.5, 0.5), (-0.25, -0.25)
  const uint64_t cz = 0x3e0000003e000000ull, ct = 0x4000000040000000ull;  // (0.125, 0.125), (2, 2)
  const uint64_t dx = sub2(X, cx), dy = sub2(Y, cy), dz = sub2(Z, cz), dt = sub2(T, ct);
  uint64_t s = add2(fma2(dx, dx, z), fma2(dy, dy, z));
  s = add2(s, fma2(dz, dz, z));
  return add2(s, fma2(dt, dt, z));
}

// Mode 4: four chains per thread, each a loop-carried (X, Y, Z, T); every
// link overwrites one coordinate with the distance of all four, in rotation,
// so all inputs of every subtract change from link to link.  Values grow to
// +inf within a few links; float32 arithmetic on infinities runs at full rate.
__global__ void k_distance(float* out, int iters, float seed) {
  uint64_t X[4], Y[4], Z[4], T[4];
  const float base = seed + (float)threadIdx.x;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    X[i] = pk(base + i, base - i);
    Y[i] = pk(base * 0.5f + i, base * 0.5f - i);
    Z[i] = pk(base * 0.25f + i, base * 0.25f - i);
    T[i] = pk(base * 0.125f + i, base * 0.125f - i);
  }
  const uint64_t z = *reinterpret_cast<volatile uint64_t*>(&g_zero2);
  for (int it = 0; it < iters; it += 2) {  // 8 links per chain per pass: 2 iterations' worth
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      X[i] = dist_link(X[i], Y[i], Z[i], T[i], z);
      Y[i] = dist_link(Y[i], Z[i], T[i], X[i], z);
      Z[i] = dist_link(Z[i], T[i], X[i], Y[i], z);
      T[i] = dist_link(T[i], X[i], Y[i], Z[i], z);
    }
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      X[i] = dist_link(X[i], Y[i], Z[i], T[i], z);
      Y[i] = dist_link(Y[i], Z[i], T[i], X[i], z);
      Z[i] = dist_link(Z[i], T[i], X[i], Y[i], z);
      T[i] = dist_link(T[i], X[i], Y[i], Z[i], z);
    }
  }
  float s = 0.f;
#pragma unroll
  for (int i = 0; i < 4; ++i)
    s += __uint_as_float((uint32_t)X[i]) + __uint_as_float((uint32_t)(Y[i] >> 32)) + __uint_as_float((uint32_t)Z[i]) +
         __uint_as_float((uint32_t)(T[i] >> 32));
  if (s == -1.2345f) out[blockIdx.x] = s;
}

}  // namespace

extern "C" {

// Runs mode `mode` (0..4, see above) over `blocks` x `threads` threads for
// `iters` iterations on `stream` between the caller's two events; returns
// the number of float32 operations it performs (an FMA counts as two), or
// -1 on a bad mode or a launch error.  `out`: at least `blocks` floats.
double fpstok_microbench_fp32(int mode, int blocks, int threads, int iters, float* out, void* start_event,
                              void* stop_event, void* stream) {
  if (mode < 0 || mode > 4) return -1.0;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  cudaEventRecord(reinterpret_cast<cudaEvent_t>(start_event), s);
  switch (mode) {
    case 0: k_scalar<<<blocks, threads, 0, s>>>(out, iters, 1.0f); break;
    case 1: k_packed<1><<<blocks, threads, 0, s>>>(out, iters, 1.0f); break;
    case 2: k_packed<2><<<blocks, threads, 0, s>>>(out, iters, 1.0f); break;
    case 3: k_packed<3><<<blocks, threads, 0, s>>>(out, iters, 1.0f); break;
    default: k_distance<<<blocks, threads, 0, s>>>(out, iters, 1.0f); break;
  }
  cudaEventRecord(reinterpret_cast<cudaEvent_t>(stop_event), s);
  if (cudaGetLastError() != cudaSuccess) return -1.0;
  const double links = (double)blocks * threads * (double)iters * 8.0;  // chain links per mode
  switch (mode) {
    case 0: return links * 2.0;        // one FMUL + one FADD
    case 1: case 2: return links * 4.0;  // two packed ops, two lanes each
    case 3: return links * 8.0;        // two packed FMAs, two lanes, two ops
    default: {                         // (iters rounded up to even) / 2 passes x 32 distances x 22 ops
      const double passes = (double)((iters + 1) / 2);
      return (double)blocks * threads * passes * 32.0 * 22.0;
    }
  }
}

}
