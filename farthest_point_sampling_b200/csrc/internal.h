// Internal host-side interfaces between the C ABI and the kernel files.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

struct fps_opts;  // include/fpstok.h

namespace fpstok {

// Event classes written by the binning kernel.
enum EventClass : int { kClsSkip = 0, kClsEmpty = 1, kClsPass = 2, kClsFps = 3 };

// Work lists (indices into WsHeader::n_items).
enum ListId : int {
  kListWarp = 0,
  kListCta = 1,
  kListCtaSmem = 2,
  kListCluster8 = 3,
  kListCluster16 = 4,
  kListChunks = 5,      // nearest-centroid passes over FPS events (Lloyd, assignment)
  kListPoolSlots = 6,   // global pooling accumulator slots in use
  kListFps = 7,         // number of FPS events (Lloyd slots)
  kListPoolChunks = 8,  // (event, chunk) items of the events k_pool_voronoi pools
  kListPoolEvents = 9,  // events pooled in several chunks (k_pool_finalize)
  kNumLists = 10,
};
constexpr int kNumSchedules = 5;  // warp, CTA, CTA-smem, 8-CTA cluster, 16-CTA cluster
constexpr int kStagePassthrough = 9;  // stage id of the passthrough kernel (helper stream)

// Schedule capacities (points per event).
constexpr int kWarpPairs = 7;                          // point pairs per lane, warp schedule
constexpr int kWarpCap = 64 * kWarpPairs;              // 448
constexpr int kCtaThreads = 256;                       // register-resident CTA schedule
constexpr int kCtaPairs = 5;                           // pairs per thread
constexpr int kCtaCap = 2 * kCtaThreads * kCtaPairs;   // 2560
constexpr size_t kCtaSmemBytes = 104 * 1024;           // register-CTA shared memory (event copy / pooling)
constexpr int kBlockThreads = 256;                     // shared-memory CTA / cluster schedules
constexpr int kBlockPairs = 24;                        // pairs per thread (all in shared memory, the first
                                                       // ones also cached in registers)
constexpr int kCtaSmemCap = kBlockThreads * 2 * kBlockPairs;  // 12288
constexpr int kCluster8Cap = 8 * kCtaSmemCap;                 // 98304
constexpr int kMaxCluster = 16;
constexpr int kClusterCap = kMaxCluster * kCtaSmemCap;        // 196608
constexpr int kPass = 1024;                            // points per Lloyd / assignment pass (256 threads x 4)
#ifndef FPS_PASS_CTAS_PER_SM
#define FPS_PASS_CTAS_PER_SM 3
#endif
constexpr int kPassCtasPerSm = FPS_PASS_CTAS_PER_SM;   // resident CTAs per SM of the pass kernels
constexpr int kPoolChunk = 512;                        // points per pooling work item
constexpr int kPoolReplicas = 16;                      // accumulator copies per event pooled in several chunks
// With at most this many FPS events per SM, events of the warp class run on
// the CTA schedule instead (lower latency per step when the GPU is not full).
constexpr int kLatencyEventsPerSm = 1;

struct Workspace {
  struct WsHeader* hdr;
  int* list_warp;
  int* list_cta;
  int* list_cta_smem;
  int* list_cluster8;
  int* list_cluster16;
  int2* passes;     // (event, first point) of every nearest-centroid pass, in batch order
  int2* pool_chunks; // (event, chunk) items of events pooled by the pool kernel
  int* cls;         // EventClass per event
  int* fps_slot;    // compact index of FPS events, -1 otherwise
  int* pool_slot;   // first accumulator slot of events pooled in several chunks, -1 otherwise
  int* pool_event;  // [events] the events pooled in several chunks
  double* pool_acc; // [pool slots][K][F]
  int* pool_cnt;    // [pool slots][K]
  double* lloyd[3]; // 3 x [fps slots][K][5] cell sums (W, S_x, S_y, S_z, S_t)
  int* labels;      // [P] internal Voronoi labels (kNN mode with Lloyd)
  int fps_slots;    // capacity of the Lloyd slot range
  int pool_slots;   // capacity of the pooling slot range
  size_t bytes;
};

struct Problem {
  const float4* coords;
  const float* feats;
  int F;
  const int64_t* offsets;
  int B;
  int64_t P;
  const int32_t* start_local;
  int K, assign_mode, k, lloyd_iters, charge_col, force_schedule, max_event_hint;
  int32_t* centroid_idx;
  int32_t* token_id;
  int32_t* knn_idx;
  float4* centroids;
  float* pooled;
  int32_t* counts;
  int fused_pool;  // bit 0 / bit 1: the warp / register-CTA FPS kernels pool their own events
  float4 w;        // per-axis scale of the distance ((1, 1, 1, 1) when unscaled)
  int scaled;      // w differs from (1, 1, 1, 1)
};

// The per-axis scale of a call: (1, 1, 1, 1) for NULL or all-zero weights.
// Returns false when a weight is not finite.
bool axis_scale_of(const float* w, float4* out, int* scaled);

// Kernel launchers (return the cudaError_t of the launch).
cudaError_t launch_bin(const Problem& pb, const Workspace& ws, int chunk_all, cudaStream_t s);
cudaError_t launch_pool_clear(const Problem& pb, const Workspace& ws, cudaStream_t s);
cudaError_t launch_passthrough(const Problem& pb, const Workspace& ws, cudaStream_t s);
typedef void (*StageMark)(int stage, int end, cudaStream_t s);
void stage_mark(int stage, int end, cudaStream_t s);
// FPS schedules plus the passthrough kernel (`pt`), all concurrent after the
// binning kernel; returns once the work is enqueued and joined into `s`.
cudaError_t launch_fps(const Problem& pb, const Problem& pt, const Workspace& ws, cudaStream_t s, StageMark mark);
// kNN mode without Lloyd: launch_fps runs each schedule's kNN rows on that
// schedule's stream right after its FPS kernel.
inline bool knn_with_fps(const Problem& pb) { return pb.assign_mode == 1 && pb.lloyd_iters == 0; }
// Bytes of shared memory of one warp of the warp schedule and of
// the register-CTA schedule (per CTA): fused pooling must fit into them.
size_t warp_region_bytes();
size_t cta_region_bytes();
// Lloyd refinement; in the tokenizer's Voronoi mode (lloyd_pools) the last
// iteration also pools the token means (k_pool_finalize still follows for
// the events pooled over several pieces).
inline bool lloyd_pools(const Problem& pb) { return pb.assign_mode == 0 && pb.pooled && pb.feats; }
// Voronoi mode without Lloyd: with a size hint that keeps every FPS event on
// the warp and register-CTA schedules, which pool in place, no pool kernel
// runs after the FPS kernels, and the pooling accumulators go unused.
inline bool pool_kernel_needed(const Problem& pb) {
  return !(pb.max_event_hint > 0 && pb.max_event_hint <= kCtaCap && pb.force_schedule <= 1 &&
           (pb.fused_pool & 3) == 3);
}
cudaError_t launch_lloyd(const Problem& pb, const Workspace& ws, int32_t* labels, cudaStream_t s);
cudaError_t launch_pool_finalize(const int64_t* offsets, int K, int F, float* pooled, int32_t* counts,
                                 const Workspace& ws, cudaStream_t s);
cudaError_t launch_pool_voronoi(const float* feats, int F, const int64_t* offsets, int B, int K,
                                const int32_t* labels, float* pooled, int32_t* counts,
                                const Workspace& ws, cudaStream_t s);
cudaError_t launch_knn(const float4* coords, const int64_t* offsets, int B, const float4* centroids,
                       const int32_t* valid_tokens, int K, int k, int32_t* knn_idx,
                       const float* feats, int F, float* pooled, int32_t* counts, const Workspace* ws,
                       struct WsHeader* hdr, cudaStream_t s, float4 w, int scaled, int only_schedule = -1);
cudaError_t launch_assign(const float4* coords, const int64_t* offsets, const float4* centroids,
                          const int32_t* valid_tokens, int K, int32_t* token_id, const Workspace& ws,
                          cudaStream_t s, float4 w);
cudaError_t launch_pool_knn(const float* feats, int F, int B, int K, int k, const int32_t* knn_idx,
                            int64_t P, float* pooled, int32_t* counts, struct WsHeader* hdr,
                            cudaStream_t s);

// Device properties cached per device.
struct DeviceInfo {
  int sm_count;
  int warp_blocks_per_sm;
  int cluster8_max_active;   // co-resident 8-CTA clusters of the shared-memory kernel
  int cluster16_max_active;  // co-resident 16-CTA clusters
  bool ready;
};
const DeviceInfo& device_info();  // prepares the current device on first use
cudaError_t prepare_aux_kernels();   // shared-memory attributes of the auxiliary kernels

void count_launch(int n = 1);

// Chunk pipeline of the host-buffer entry point: offsets[i] -= base, and
// non-negative indices += shift.
cudaError_t launch_rebase_offsets(int64_t* off, int n, int64_t base, cudaStream_t s);
cudaError_t launch_shift_indices(int32_t* idx, int64_t n, int32_t shift, cudaStream_t s);

// Test setting of the cluster exchange of the next launches: the poll limit
// of each wait (<= 0: the default) and a CTA rank that skips its post in the
// first exchange of every event (-1: none).
void set_exchange_test(int spin_limit, int skip_rank);

// Workspace bytes fps_tokenize needs for this exact call (the labels area is
// reserved only when kNN mode runs Lloyd without a caller token_id buffer).
size_t tokenize_workspace_need(int64_t P, int B, int F, const ::fps_opts* o, const int32_t* token_id);

}  // namespace fpstok
