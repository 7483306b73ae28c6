// Random FPS start points (graphnet PR #923, review thread on the FPS
// arguments: start_idx, random_start and a generator).  Event b starts at
// floor(u * N_b / 2^32), u the first word of Philox4x32-10 (Salmon, Moraes,
// Dror and Shaw, "Parallel random numbers: as easy as 1, 2, 3", SC 2011) at
// counter (b, stream, 0, 0) under the key (seed low word, seed high word);
// empty events start at 0.  The generator is written here from its
// definition: ten rounds of two 32 x 32 -> 64-bit products (multipliers
// 0xD2511F53 and 0xCD9E8D57) and a word shuffle, the key raised by the Weyl
// constants 0x9E3779B9 and 0xBB67AE85 between rounds.
#include "../../include/fpstok.h"
#include "common.cuh"
#include "internal.h"
#include "random_start.h"

namespace fpstok {

namespace {

__device__ __forceinline__ uint4 philox4x32_10(uint4 c, uint32_t k0, uint32_t k1) {
#pragma unroll
  for (int round = 0; round < 10; ++round) {
    if (round > 0) {
      k0 += 0x9E3779B9u;
      k1 += 0xBB67AE85u;
    }
    const uint32_t lo0 = 0xD2511F53u * c.x, hi0 = __umulhi(0xD2511F53u, c.x);
    const uint32_t lo1 = 0xCD9E8D57u * c.z, hi1 = __umulhi(0xCD9E8D57u, c.z);
    c = make_uint4(hi1 ^ c.y ^ k0, lo1, hi0 ^ c.w ^ k1, lo0);
  }
  return c;
}

__global__ void __launch_bounds__(256) k_random_starts(const int64_t* __restrict__ offsets, int B, uint32_t k0,
                                                       uint32_t k1, uint32_t stream_id,
                                                       int32_t* __restrict__ start_local, WsHeader* hdr) {
  const int b = blockIdx.x * blockDim.x + threadIdx.x;
  if (b >= B) return;
  const int64_t n = offsets[b + 1] - offsets[b];
  if (n < 0 || n >= ((int64_t)1 << 31)) {
    if (hdr) record_error(hdr, kDevBadOffsets);
    start_local[b] = 0;
    return;
  }
  const uint4 x = philox4x32_10(make_uint4((uint32_t)b, stream_id, 0u, 0u), k0, k1);
  start_local[b] = (int32_t)(((uint64_t)x.x * (uint64_t)n) >> 32);
}

}  // namespace

cudaError_t launch_random_starts(const int64_t* offsets, int B, uint64_t seed, uint32_t stream_id,
                                 int32_t* start_local, WsHeader* hdr, cudaStream_t s) {
  if (B == 0) return cudaSuccess;
  count_launch();
  k_random_starts<<<(B + 255) / 256, 256, 0, s>>>(offsets, B, (uint32_t)seed, (uint32_t)(seed >> 32), stream_id,
                                                  start_local, hdr);
  return cudaGetLastError();
}

}  // namespace fpstok
