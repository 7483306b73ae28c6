// In-run FP32 issue-rate microbenchmark for the roofline of the FPS kernels.
//
// The FPS distance is made of separate (unfused) float32 adds and multiplies,
// so its ceiling is the rate of non-FMA FP32 operations.  Two kernels measure
// it on every SM: independent chains of scalar FADD/FMUL, and of the packed
// f32x2 forms (two float32 operations per instruction).  Each thread keeps 8
// independent chains so latency is hidden; the result is stored only when an
// impossible value appears, which keeps the compiler from removing the work.
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

__global__ void k_packed(float* out, int iters, float seed) {
  uint64_t a[8];
  const float base = seed + (float)threadIdx.x;
#pragma unroll
  for (int i = 0; i < 8; ++i)
    a[i] = (uint64_t)__float_as_uint(base + i) | ((uint64_t)__float_as_uint(base - i) << 32);
  const uint64_t m = (uint64_t)__float_as_uint(0.999999f) * 0x100000001ull;
  const uint64_t c = (uint64_t)__float_as_uint(1e-7f) * 0x100000001ull;
  for (int it = 0; it < iters; ++it) {
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      a[i] = mul2(a[i], m);
      a[i] = add2(a[i], c);
    }
  }
  float s = 0.f;
#pragma unroll
  for (int i = 0; i < 8; ++i) s += __uint_as_float((uint32_t)a[i]) + __uint_as_float((uint32_t)(a[i] >> 32));
  if (s == -1.2345f) out[blockIdx.x] = s;
}

}  // namespace

extern "C" {

// Runs one kernel (packed != 0: f32x2) over `blocks` x `threads` threads for
// `iters` iterations on `stream` between the caller's two events; returns
// the number of float32 operations it performs, or -1 on a launch error.
// `out` is a device buffer of at least `blocks` floats.
double fpstok_microbench_fp32(int packed, int blocks, int threads, int iters, float* out, void* start_event,
                              void* stop_event, void* stream) {
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  cudaEventRecord(reinterpret_cast<cudaEvent_t>(start_event), s);
  if (packed)
    k_packed<<<blocks, threads, 0, s>>>(out, iters, 1.0f);
  else
    k_scalar<<<blocks, threads, 0, s>>>(out, iters, 1.0f);
  cudaEventRecord(reinterpret_cast<cudaEvent_t>(stop_event), s);
  if (cudaGetLastError() != cudaSuccess) return -1.0;
  // 8 chains x (1 mul + 1 add) per iteration; f32x2 does two lanes each
  return (double)blocks * threads * (double)iters * 16.0 * (packed ? 2.0 : 1.0);
}

}
