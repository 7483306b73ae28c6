// fps_tokenize_static: the whole tokenizer without a caller-provided workspace.
//
// Who needs it: some callers cannot obtain device scratch memory at all.  A
// plugin living inside a host program that owns the GPU's memory (for example
// an online event filter that reserves all device memory at start-up and only
// hands its plugins the input and output buffers) may not call cudaMalloc or
// any allocating library routine (torch's caching allocator included); and a
// caller on a latency-critical path may not accept the device-wide
// synchronisation that cudaMalloc/cudaFree can cause.  fps_tokenize needs a
// workspace such callers cannot provide, so this entry point takes the same
// inputs and outputs but keeps its scratch in the file-scope device array
// below (FPS_STATIC_SCRATCH_BYTES = 8 MiB), which every GPU that loads the
// library holds until the process exits.  It calls no cudaMalloc, cudaFree or
// allocating library routine.
//
// Host code must not hand `g_static_scratch` itself to a kernel: in host code
// that name is only a host-side stand-in, not a device address.  The device
// address is looked up once per device with cudaGetSymbolAddress, on the
// first call made while that device is current; make that first call before
// any stream capture.  The looked-up address is kept for the life of the
// process: after cudaDeviceReset (or anything else that destroys the primary
// context and unloads the module) it is stale, and calls to this entry point
// on that device are not supported.  All calls share the one array and it
// keeps the last call's contents; the tokenizer's kernels clear every scratch
// word that must start at zero.  Calls whose work overlaps on the GPU (for
// example on two streams) race on the array.
//
// fps_static_device_status reads back the device-side status word of the
// last call on the current device (bad offsets, a start index outside its
// event, an exchange that ran out of time), which fps_tokenize keeps at the
// start of its workspace -- here, of the static array.
#include <mutex>

#include "../../include/fpstok.h"
#include "internal.h"

static __device__ __align__(256) unsigned char g_static_scratch[FPS_STATIC_SCRATCH_BYTES];

namespace {

constexpr int kMaxDevices = 64;
void* g_scratch_addr[kMaxDevices];
std::mutex g_scratch_mu;

// Device address of g_static_scratch on the current device (looked up once).
int static_scratch_address(void** out) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return FPS_ERR_CUDA;
  std::lock_guard<std::mutex> lock(g_scratch_mu);
  if (g_scratch_addr[dev] == nullptr) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_static_scratch) != cudaSuccess || p == nullptr) return FPS_ERR_CUDA;
    g_scratch_addr[dev] = p;
  }
  *out = g_scratch_addr[dev];
  return FPS_OK;
}

}  // namespace

extern "C" int fps_tokenize_static(const float* coords, const float* feats, int F, const int64_t* offsets,
                                   int B, int64_t P, const int32_t* start_local, const fps_opts* opts,
                                   int32_t* centroid_idx, int32_t* token_id, int32_t* knn_idx,
                                   float* centroids, float* pooled, int32_t* counts, fps_stream_t stream) {
  if (opts != nullptr && P >= 0 && B >= 0 &&
      fpstok::tokenize_workspace_need(P, B, F, opts, token_id) > (size_t)FPS_STATIC_SCRATCH_BYTES)
    return FPS_ERR_TOO_LARGE;  // the batch needs more scratch than the static array holds
  void* scratch = nullptr;
  if (B > 0) {
    const int rc = static_scratch_address(&scratch);
    if (rc != FPS_OK) return rc;
  }
  return fps_tokenize(coords, feats, F, offsets, B, P, start_local, opts, centroid_idx, token_id, knn_idx,
                      centroids, pooled, counts, scratch, scratch ? (size_t)FPS_STATIC_SCRATCH_BYTES : 0, stream);
}

extern "C" int fps_static_device_status(fps_stream_t stream, int* detail) {
  void* scratch = nullptr;
  const int rc = static_scratch_address(&scratch);
  if (rc != FPS_OK) return rc;
  return fps_device_status(scratch, stream, detail);
}
