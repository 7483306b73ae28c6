// Device side of the host-buffer entry point's chunk pipeline (fps_tokenize_host):
// the tokenizer runs on a slice of the batch's events at a time, so each
// slice's offsets are moved to start at 0 before the call, and its global
// point indices (centroid_idx, knn_idx) are moved back to the batch's
// numbering after it.
#include "common.cuh"
#include "internal.h"

namespace fpstok {

__global__ void __launch_bounds__(256) k_rebase_offsets(int64_t* __restrict__ off, int n, int64_t base) {
  for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < n; i += gridDim.x * blockDim.x) off[i] -= base;
}

__global__ void __launch_bounds__(256) k_shift_indices(int32_t* __restrict__ idx, int64_t n, int32_t shift) {
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += (int64_t)gridDim.x * blockDim.x) {
    const int32_t v = idx[i];
    if (v >= 0) idx[i] = v + shift;
  }
}

cudaError_t launch_rebase_offsets(int64_t* off, int n, int64_t base, cudaStream_t s) {
  if (n <= 0 || base == 0) return cudaSuccess;
  int blocks = (n + 255) / 256;
  if (blocks > 1024) blocks = 1024;
  count_launch();
  k_rebase_offsets<<<blocks, 256, 0, s>>>(off, n, base);
  return cudaGetLastError();
}

cudaError_t launch_shift_indices(int32_t* idx, int64_t n, int32_t shift, cudaStream_t s) {
  if (n <= 0 || shift == 0) return cudaSuccess;
  int64_t blocks = (n + 255) / 256;
  if (blocks > 1024) blocks = 1024;
  count_launch();
  k_shift_indices<<<(int)blocks, 256, 0, s>>>(idx, n, shift);
  return cudaGetLastError();
}

}  // namespace fpstok
