// Launcher of the random FPS start points (random_start.cu).
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

namespace fpstok {

struct WsHeader;

// start_local[b] = floor(u_b * N_b / 2^32), u_b the first word of
// Philox4x32-10 at counter (b, stream_id, 0, 0), key (seed low, seed high).
// hdr may be null (no device status recorded).
cudaError_t launch_random_starts(const int64_t* offsets, int B, uint64_t seed, uint32_t stream_id,
                                 int32_t* start_local, WsHeader* hdr, cudaStream_t s);

}  // namespace fpstok
