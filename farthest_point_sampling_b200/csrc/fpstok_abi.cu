// C ABI of the fpstok tokenizer (declared in include/fpstok.h): argument
// checks, workspace carving and the launch sequence.  No allocation, no
// synchronisation (except fps_device_status, which exists to read back).
#include <algorithm>
#include <atomic>
#include <mutex>
#include <cmath>
#include <cstring>

#include "../../include/fpstok.h"
#include "common.cuh"
#include "internal.h"
#include "pool_backward.h"
#include "token_pack.h"
#include "token_summary.h"
#include "random_start.h"

namespace fpstok {

static std::atomic<uint64_t> g_launches{0};
void count_launch(int n) { g_launches.fetch_add((uint64_t)n, std::memory_order_relaxed); }

static void* g_stage_events[32];
static int g_n_stage_events = 0;

static unsigned g_stage_mask;  // stages marked since the last fps_set_stage_events

void stage_mark(int stage, int end, cudaStream_t s) {
  const int e = 2 * stage + end;
  if (!end) g_stage_mask |= 1u << stage;
  if (e < g_n_stage_events && g_stage_events[e])
    cudaEventRecord(reinterpret_cast<cudaEvent_t>(g_stage_events[e]), s);
}

static size_t align256(size_t x) { return (x + 255) & ~(size_t)255; }

struct Carver {
  char* base;
  size_t off = 0;
  template <typename T>
  T* take(size_t n) {
    T* p = base ? reinterpret_cast<T*>(base + off) : nullptr;
    off = align256(off + n * sizeof(T));
    return p;
  }
};

// Lays out the workspace; with base == nullptr only computes the size.
static Workspace carve(void* base, int64_t P, int B, int K, int F, bool lloyd, bool labels) {
  Carver c{static_cast<char*>(base)};
  Workspace w = {};
  const int64_t nb = B > 0 ? B : 1;
  const int64_t passes = nb + P / kPass + 1;
  const int64_t pool_chunks = nb + P / kPoolChunk + 1;
  // an event pooled in c > 1 chunks takes min(kPoolReplicas, c) slots: at most
  // ceil(n / kPoolChunk) <= n / kPoolChunk + 1 with n > kPoolChunk
  const int64_t pool_slots = 2 * (P / kPoolChunk) + 1;
  int64_t fps_slots = P / (K + 1) + 1;
  if (fps_slots > nb) fps_slots = nb;
  w.hdr = c.take<WsHeader>(1);
  w.list_warp = c.take<int>(nb);
  w.list_cta = c.take<int>(nb);
  w.list_cta_smem = c.take<int>(nb);
  w.list_cluster8 = c.take<int>(nb);
  w.list_cluster16 = c.take<int>(nb);
  w.passes = c.take<int2>(passes);
  w.pool_chunks = c.take<int2>(pool_chunks);
  w.cls = c.take<int>(nb);
  w.fps_slot = c.take<int>(nb);
  w.pool_slot = c.take<int>(nb);
  w.pool_event = c.take<int>(nb);
  w.pool_acc = c.take<double>(pool_slots * K * (F > 0 ? F : 1));
  w.pool_cnt = c.take<int>(pool_slots * K);
  for (int i = 0; i < 3; ++i) w.lloyd[i] = lloyd ? c.take<double>(fps_slots * K * 5) : nullptr;
  w.labels = labels ? c.take<int>(P > 0 ? P : 1) : nullptr;
  w.fps_slots = (int)fps_slots;
  w.pool_slots = (int)pool_slots;
  w.bytes = c.off;
  return w;
}

static int from_cuda(cudaError_t e) { return e == cudaSuccess ? FPS_OK : FPS_ERR_CUDA; }

bool axis_scale_of(const float* w, float4* out, int* scaled) {
  *out = make_float4(1.f, 1.f, 1.f, 1.f);
  *scaled = 0;
  if (!w) return true;
  bool zero = true;
  for (int a = 0; a < 4; ++a) {
    if (!std::isfinite(w[a])) return false;
    if (w[a] != 0.f) zero = false;
  }
  if (zero) return true;  // the zero-initialised default: unscaled
  *out = make_float4(w[0], w[1], w[2], w[3]);
  *scaled = (w[0] != 1.f || w[1] != 1.f || w[2] != 1.f || w[3] != 1.f) ? 1 : 0;
  return true;
}

static bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

static int check_common(int64_t P, int B, const int64_t* offsets) {
  if (B < 0 || P < 0) return FPS_ERR_ARG;
  if (P >= ((int64_t)1 << 31)) return FPS_ERR_TOO_LARGE;
  if (B > 0 && offsets == nullptr) return FPS_ERR_ARG;
  return FPS_OK;
}

static int check_opts(const fps_opts* o, int F) {
  if (!o) return FPS_ERR_ARG;
  if (o->K < 1) return FPS_ERR_ARG;
  if (o->K > FPS_MAX_K) return FPS_ERR_TOO_LARGE;
  if (o->assign_mode != FPS_ASSIGN_VORONOI && o->assign_mode != FPS_ASSIGN_KNN) return FPS_ERR_ARG;
  if (o->assign_mode == FPS_ASSIGN_KNN) {
    if (o->k < 1) return FPS_ERR_ARG;
    if (o->k > o->K || o->k > FPS_MAX_KNN) return FPS_ERR_TOO_LARGE;
  }
  if (o->lloyd_iters < 0) return FPS_ERR_ARG;
  if (F < 1) return FPS_ERR_ARG;
  if (F > FPS_MAX_F) return FPS_ERR_TOO_LARGE;
  if (o->charge_col < -1 || o->charge_col >= F) return FPS_ERR_ARG;
  if (o->force_schedule < -1 || o->force_schedule > 4) return FPS_ERR_ARG;
  if (o->max_event_hint < 0) return FPS_ERR_ARG;
  if (o->max_event_hint > kClusterCap) return FPS_ERR_TOO_LARGE;
  float4 w;
  int scaled;
  if (!axis_scale_of(o->axis_scale, &w, &scaled)) return FPS_ERR_ARG;
  return FPS_OK;
}

static bool needs_labels(const fps_opts* o, const int32_t* token_id) {
  return o->assign_mode == FPS_ASSIGN_KNN && o->lloyd_iters > 0 && token_id == nullptr;
}

size_t tokenize_workspace_need(int64_t P, int B, int F, const fps_opts* o, const int32_t* token_id) {
  if (!o || P < 0 || B < 0 || o->K < 1) return 0;
  return carve(nullptr, P, B, o->K, F, o->lloyd_iters > 0, needs_labels(o, token_id)).bytes;
}

static int run_tokenize(const Problem& pb0, const Workspace& ws, cudaStream_t s) {
  Problem pb = pb0;
  int32_t* labels = pb.token_id ? pb.token_id : ws.labels;
  pb.token_id = labels;  // FPS writes the Voronoi labels here (may be null in plain kNN mode)
  cudaError_t e;
  stage_mark(0, 0, s);
  if ((e = launch_bin(pb, ws, 0, s))) return from_cuda(e);
  stage_mark(0, 1, s);
  Problem pt = pb;
  pt.token_id = pb0.token_id;
  pt.knn_idx = pb.assign_mode == FPS_ASSIGN_KNN ? pb.knn_idx : nullptr;
  if ((e = launch_fps(pb, pt, ws, s, stage_mark))) return from_cuda(e);
  if (pb.lloyd_iters > 0) {
    stage_mark(6, 0, s);
    if ((e = launch_lloyd(pb, ws, labels, s))) return from_cuda(e);
    stage_mark(6, 1, s);
  }
  if (pb.assign_mode == FPS_ASSIGN_KNN && knn_with_fps(pb)) {
    // done by launch_fps, schedule by schedule
  } else if (pb.assign_mode == FPS_ASSIGN_KNN) {
    stage_mark(7, 0, s);
    if ((e = launch_knn(pb.coords, pb.offsets, pb.B, pb.centroids, nullptr, pb.K, pb.k, pb.knn_idx,
                        pb.feats, pb.F, pb.pooled, pb.counts, &ws, ws.hdr, s, pb.w, pb.scaled)))
      return from_cuda(e);
    stage_mark(7, 1, s);
  } else {
    // with a size hint, a batch whose events all fit the schedules that pool
    // in place needs no pool kernel
    const bool none_left = !pool_kernel_needed(pb);
    if (pb.lloyd_iters > 0 && lloyd_pools(pb)) {  // the last Lloyd iteration pooled; the replicas' means
      stage_mark(8, 0, s);
      if ((e = launch_pool_finalize(pb.offsets, pb.K, pb.F, pb.pooled, pb.counts, ws, s))) return from_cuda(e);
      stage_mark(8, 1, s);
    } else if (!none_left) {
      stage_mark(8, 0, s);
      if ((e = launch_pool_voronoi(pb.feats, pb.F, pb.offsets, pb.B, pb.K, labels, pb.pooled, pb.counts, ws, s)))
        return from_cuda(e);
      stage_mark(8, 1, s);
    }
  }
  return FPS_OK;
}

}  // namespace fpstok

using namespace fpstok;

extern "C" {

int64_t fps_max_event_points(void) { return kClusterCap; }

int fps_schedule_for(int64_t n, int K, int force_schedule) {
  if (n > kClusterCap) return -2;
  if (n <= 0 || n <= K) return -1;
  int q = n <= kWarpCap ? 0 : (n <= kCtaCap ? 1 : (n <= kCtaSmemCap ? 2 : (n <= kCluster8Cap ? 3 : 4)));
  if (force_schedule > q) q = force_schedule > 4 ? 4 : force_schedule;
  return q;
}

size_t fps_workspace_bytes(int64_t P, int B, int F, const fps_opts* opts) {
  if (!opts || P < 0 || B < 0 || opts->K < 1) return 0;
  const bool lab = opts->assign_mode == FPS_ASSIGN_KNN && opts->lloyd_iters > 0;
  return carve(nullptr, P, B, opts->K, F, opts->lloyd_iters > 0, lab).bytes;
}

int fps_tokenize(const float* coords, const float* feats, int F, const int64_t* offsets, int B, int64_t P,
                 const int32_t* start_local, const fps_opts* opts, int32_t* centroid_idx, int32_t* token_id,
                 int32_t* knn_idx, float* centroids, float* pooled, int32_t* counts, void* workspace,
                 size_t workspace_bytes, fps_stream_t stream) {
  int rc = check_common(P, B, offsets);
  if (rc) return rc;
  if ((rc = check_opts(opts, F))) return rc;
  if (B == 0) return FPS_OK;
  if (!centroid_idx || !centroids || !pooled || !counts) return FPS_ERR_ARG;
  if (opts->assign_mode == FPS_ASSIGN_VORONOI && !token_id && P > 0) return FPS_ERR_ARG;
  if (opts->assign_mode == FPS_ASSIGN_KNN && !knn_idx) return FPS_ERR_ARG;
  if (P > 0 && (!coords || !feats)) return FPS_ERR_ARG;
  if (!aligned(coords, 16) || !aligned(centroids, 16)) return FPS_ERR_ARG;
  const bool lab = needs_labels(opts, token_id);
  const Workspace need = carve(nullptr, P, B, opts->K, F, opts->lloyd_iters > 0, lab);
  if (!workspace || workspace_bytes < need.bytes || !aligned(workspace, 256)) return FPS_ERR_WORKSPACE;
  const Workspace ws = carve(workspace, P, B, opts->K, F, opts->lloyd_iters > 0, lab);
  Problem pb = {reinterpret_cast<const float4*>(coords), feats, F, offsets, B, P, start_local,
                opts->K, opts->assign_mode, opts->k, opts->lloyd_iters, opts->charge_col,
                opts->force_schedule, opts->max_event_hint, centroid_idx, token_id,
                opts->assign_mode == FPS_ASSIGN_KNN ? knn_idx : nullptr,
                reinterpret_cast<float4*>(centroids), pooled, counts, 0};
  axis_scale_of(opts->axis_scale, &pb.w, &pb.scaled);
  if (opts->assign_mode == FPS_ASSIGN_VORONOI && opts->lloyd_iters == 0) {
    const size_t K = (size_t)opts->K, Fz = (size_t)F;
    if ((size_t)kWarpCap * sizeof(float) + 2 * K * sizeof(int) <= warp_region_bytes()) pb.fused_pool |= 1;
    if ((size_t)(3 * kCtaCap + 768) * sizeof(int) + (size_t)kCtaCap * Fz * sizeof(float) <= cta_region_bytes())
      pb.fused_pool |= 2;
  }
  return run_tokenize(pb, ws, reinterpret_cast<cudaStream_t>(stream));
}

// Host-pointer variant: staging layout after the regular workspace.  The
// batch goes through in up to kHostChunks slices of consecutive events, each
// slice's offsets in its own staging rows (slice c: rows b0 + c .. b1 + c).
constexpr int kHostChunks = 6;
constexpr int64_t kHostChunkMinPoints = 65536;  // smaller batches go in one piece
constexpr int kHostChunkMinEvents = 256;        // and so do batches of few (large) events: a slice of them
                                                // would leave the GPU mostly idle

struct HostStage {
  size_t coords, feats, offsets, start, cidx, tok, knn, cents, pooled, counts, total;
};

static HostStage host_stage(size_t base, int64_t P, int B, int F, const fps_opts* o, bool has_start) {
  HostStage h;
  size_t off = align256(base);
  auto take = [&](size_t n) {
    const size_t at = off;
    off = align256(off + n);
    return at;
  };
  const int K = o->K;
  const int k = o->assign_mode == FPS_ASSIGN_KNN ? o->k : 0;
  h.coords = take((size_t)P * 16);
  h.feats = take((size_t)P * F * 4);
  h.offsets = take((size_t)(B + 1 + kHostChunks) * 8);
  h.start = take(has_start ? (size_t)B * 4 : 0);
  h.cidx = take((size_t)B * K * 4);
  h.tok = take((size_t)P * 4);
  h.knn = take((size_t)B * K * k * 4);
  h.cents = take((size_t)B * K * 16);
  h.pooled = take((size_t)B * K * F * 4);
  h.counts = take((size_t)B * K * 4);
  h.total = off;
  return h;
}

// Streams and events of the host-buffer pipeline, per device: copies in and
// out run on their own streams beside the caller's (compute) stream.
struct HostPipe {
  cudaStream_t in, out;
  cudaEvent_t fork, in_done[kHostChunks], comp_done[kHostChunks], out_done;
  bool ready;
};
constexpr int kMaxHostDevices = 64;
static HostPipe g_pipe[kMaxHostDevices];
static std::mutex g_pipe_mu;

static cudaError_t host_pipe(HostPipe** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxHostDevices) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lock(g_pipe_mu);
  HostPipe& hp = g_pipe[dev];
  if (!hp.ready) {
    if ((e = cudaStreamCreateWithFlags(&hp.in, cudaStreamNonBlocking))) return e;
    if ((e = cudaStreamCreateWithFlags(&hp.out, cudaStreamNonBlocking))) return e;
    if ((e = cudaEventCreateWithFlags(&hp.fork, cudaEventDisableTiming))) return e;
    if ((e = cudaEventCreateWithFlags(&hp.out_done, cudaEventDisableTiming))) return e;
    for (int c = 0; c < kHostChunks; ++c) {
      if ((e = cudaEventCreateWithFlags(&hp.in_done[c], cudaEventDisableTiming))) return e;
      if ((e = cudaEventCreateWithFlags(&hp.comp_done[c], cudaEventDisableTiming))) return e;
    }
    hp.ready = true;
  }
  *out = &hp;
  return cudaSuccess;
}

size_t fps_host_workspace_bytes(int64_t P, int B, int F, const fps_opts* opts) {
  const size_t base = fps_workspace_bytes(P, B, F, opts);
  if (!base) return 0;
  return host_stage(base, P, B, F, opts, true).total;
}

int fps_tokenize_host(const float* coords, const float* feats, int F, const int64_t* offsets, int B,
                      int64_t P, const int32_t* start_local, const fps_opts* opts, int32_t* centroid_idx,
                      int32_t* token_id, int32_t* knn_idx, float* centroids, float* pooled, int32_t* counts,
                      void* workspace, size_t workspace_bytes, fps_stream_t stream) {
  int rc = check_common(P, B, offsets);
  if (rc) return rc;
  if ((rc = check_opts(opts, F))) return rc;
  if (B == 0) return FPS_OK;
  if (!centroid_idx || !centroids || !pooled || !counts) return FPS_ERR_ARG;
  if (opts->assign_mode == FPS_ASSIGN_VORONOI && !token_id && P > 0) return FPS_ERR_ARG;
  if (opts->assign_mode == FPS_ASSIGN_KNN && !knn_idx) return FPS_ERR_ARG;
  if (P > 0 && (!coords || !feats)) return FPS_ERR_ARG;
  if (offsets[0] != 0 || offsets[B] != P) return FPS_ERR_ARG;  // host offsets: checked here
  for (int b = 0; b < B; ++b) {
    const int64_t n = offsets[b + 1] - offsets[b];
    if (n < 0) return FPS_ERR_ARG;
    if (n > kClusterCap) return FPS_ERR_TOO_LARGE;
    if (start_local && n > opts->K && (start_local[b] < 0 || start_local[b] >= n)) return FPS_ERR_ARG;
  }
  const size_t base = fps_workspace_bytes(P, B, F, opts);
  const HostStage h = host_stage(base, P, B, F, opts, start_local != nullptr);
  if (!workspace || workspace_bytes < h.total || !aligned(workspace, 256)) return FPS_ERR_WORKSPACE;
  char* w = static_cast<char*>(workspace);
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  const int K = opts->K;
  const int k = opts->assign_mode == FPS_ASSIGN_KNN ? opts->k : 0;
  HostPipe* hp = nullptr;
  cudaError_t e;
  if ((e = host_pipe(&hp))) return from_cuda(e);

  // slices of consecutive events by points: the first and the last half as
  // large as the others, so that compute starts early and the tail (last
  // compute and copy out) is short
  const int nc = (P >= kHostChunkMinPoints && B >= kHostChunkMinEvents) ? kHostChunks : 1;
  int bnd[kHostChunks + 1];
  bnd[0] = 0;
  for (int c = 1; c < nc; ++c) {
    const int64_t target = P * (2 * c - 1) / (2 * (nc - 1));  // 1/(2(nc-1)) first, 1/(nc-1) each middle one
    int lo = bnd[c - 1] + 1, hi = B - (nc - c);  // at least one event per slice
    while (lo < hi) {  // first b with offsets[b] >= target
      const int mid = lo + (hi - lo) / 2;
      if (offsets[mid] < target) lo = mid + 1;
      else hi = mid;
    }
    bnd[c] = lo;
  }
  bnd[nc] = B;

  auto h2d = [&](size_t at, const void* src, size_t n) {
    return n ? cudaMemcpyAsync(w + at, src, n, cudaMemcpyHostToDevice, hp->in) : cudaSuccess;
  };
  auto d2h = [&](void* dst, size_t at, size_t n) {
    return (n && dst) ? cudaMemcpyAsync(dst, w + at, n, cudaMemcpyDeviceToHost, hp->out) : cudaSuccess;
  };
  // copies in wait for the caller's earlier work (staging rows are reused across calls)
  if ((e = cudaEventRecord(hp->fork, s)) || (e = cudaStreamWaitEvent(hp->in, hp->fork, 0)) ||
      (e = cudaStreamWaitEvent(hp->out, hp->fork, 0)))
    return from_cuda(e);
  for (int c = 0; c < nc; ++c) {  // every slice's inputs, back to back
    const int b0 = bnd[c], b1 = bnd[c + 1];
    const int64_t p0 = offsets[b0], p1 = offsets[b1];
    if ((e = h2d(h.coords + (size_t)p0 * 16, coords + p0 * 4, (size_t)(p1 - p0) * 16)) ||
        (e = h2d(h.feats + (size_t)p0 * F * 4, feats + p0 * F, (size_t)(p1 - p0) * F * 4)) ||
        (e = h2d(h.offsets + (size_t)(b0 + c) * 8, offsets + b0, (size_t)(b1 - b0 + 1) * 8)) ||
        (e = h2d(h.start + (size_t)b0 * 4, start_local ? start_local + b0 : nullptr,
                 start_local ? (size_t)(b1 - b0) * 4 : 0)) ||
        (e = cudaEventRecord(hp->in_done[c], hp->in)))
      return from_cuda(e);
  }
  for (int c = 0; c < nc; ++c) {  // each slice: rebase, tokenize, renumber on the caller's stream; copy out
    const int b0 = bnd[c], b1 = bnd[c + 1], bc = b1 - b0;
    const int64_t p0 = offsets[b0], pc = offsets[b1] - p0;
    // the sizes are on the host: the slice's largest event is an exact size
    // hint, so schedules and the pool kernel with nothing to do are not launched
    fps_opts oc = *opts;
    int64_t nmax = 0;
    for (int b = b0; b < b1; ++b) nmax = std::max(nmax, offsets[b + 1] - offsets[b]);
    if (nmax > 0 && (oc.max_event_hint <= 0 || nmax < oc.max_event_hint)) oc.max_event_hint = (int)nmax;
    if ((e = cudaStreamWaitEvent(s, hp->in_done[c], 0))) return from_cuda(e);
    int64_t* off_c = reinterpret_cast<int64_t*>(w + h.offsets) + b0 + c;
    if ((e = launch_rebase_offsets(off_c, bc + 1, p0, s))) return from_cuda(e);
    int32_t* cidx_c = reinterpret_cast<int32_t*>(w + h.cidx) + (int64_t)b0 * K;
    int32_t* knn_c = k ? reinterpret_cast<int32_t*>(w + h.knn) + (int64_t)b0 * K * k : nullptr;
    rc = fps_tokenize(reinterpret_cast<const float*>(w + h.coords) + p0 * 4,
                      reinterpret_cast<const float*>(w + h.feats) + p0 * F, F, off_c, bc, pc,
                      start_local ? reinterpret_cast<const int32_t*>(w + h.start) + b0 : nullptr, &oc, cidx_c,
                      token_id ? reinterpret_cast<int32_t*>(w + h.tok) + p0 : nullptr, knn_c,
                      reinterpret_cast<float*>(w + h.cents) + (int64_t)b0 * K * 4,
                      reinterpret_cast<float*>(w + h.pooled) + (int64_t)b0 * K * F,
                      reinterpret_cast<int32_t*>(w + h.counts) + (int64_t)b0 * K, workspace, base, stream);
    if (rc) return rc;
    if ((e = launch_shift_indices(cidx_c, (int64_t)bc * K, (int32_t)p0, s))) return from_cuda(e);
    if (knn_c && (e = launch_shift_indices(knn_c, (int64_t)bc * K * k, (int32_t)p0, s))) return from_cuda(e);
    if ((e = cudaEventRecord(hp->comp_done[c], s)) || (e = cudaStreamWaitEvent(hp->out, hp->comp_done[c], 0)))
      return from_cuda(e);
    if ((e = d2h(centroid_idx + (int64_t)b0 * K, h.cidx + (size_t)b0 * K * 4, (size_t)bc * K * 4)) ||
        (e = d2h(token_id ? token_id + p0 : nullptr, h.tok + (size_t)p0 * 4, (size_t)pc * 4)) ||
        (e = d2h(k ? knn_idx + (int64_t)b0 * K * k : nullptr, h.knn + (size_t)b0 * K * k * 4,
                 (size_t)bc * K * k * 4)) ||
        (e = d2h(centroids + (int64_t)b0 * K * 4, h.cents + (size_t)b0 * K * 16, (size_t)bc * K * 16)) ||
        (e = d2h(pooled + (int64_t)b0 * K * F, h.pooled + (size_t)b0 * K * F * 4, (size_t)bc * K * F * 4)) ||
        (e = d2h(counts + (int64_t)b0 * K, h.counts + (size_t)b0 * K * 4, (size_t)bc * K * 4)))
      return from_cuda(e);
  }
  if ((e = cudaEventRecord(hp->out_done, hp->out)) || (e = cudaStreamWaitEvent(s, hp->out_done, 0)))
    return from_cuda(e);
  return FPS_OK;
}

size_t fps_assign_workspace_bytes(int64_t P, int B) { return carve(nullptr, P, B, 1, 1, false, false).bytes; }

int fps_assign(const float* coords, const int64_t* offsets, int B, int64_t P, const float* centroids,
               const int32_t* valid_tokens, int K, int32_t* token_id, const float* axis_scale, void* workspace,
               size_t workspace_bytes, fps_stream_t stream) {
  int rc = check_common(P, B, offsets);
  if (rc) return rc;
  float4 w;
  int scaled;
  if (!axis_scale_of(axis_scale, &w, &scaled)) return FPS_ERR_ARG;
  if (K < 1) return FPS_ERR_ARG;
  if (K > FPS_MAX_K) return FPS_ERR_TOO_LARGE;
  if (B == 0 || P == 0) return FPS_OK;
  if (!coords || !centroids || !token_id) return FPS_ERR_ARG;
  if (!aligned(coords, 16) || !aligned(centroids, 16)) return FPS_ERR_ARG;
  const size_t need = fps_assign_workspace_bytes(P, B);
  if (!workspace || workspace_bytes < need || !aligned(workspace, 256)) return FPS_ERR_WORKSPACE;
  const Workspace ws = carve(workspace, P, B, 1, 1, false, false);
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  // every non-empty event becomes (event, chunk) items: K here only splits classes
  Problem pb = {};
  pb.offsets = offsets;
  pb.B = B;
  pb.P = P;
  pb.K = K;
  pb.force_schedule = -1;
  cudaError_t e;
  if ((e = launch_bin(pb, ws, 1, s))) return from_cuda(e);
  return from_cuda(launch_assign(reinterpret_cast<const float4*>(coords), offsets,
                                 reinterpret_cast<const float4*>(centroids), valid_tokens, K, token_id, ws, s, w));
}

size_t fps_knn_workspace_bytes(int64_t P, int B) {
  (void)P;
  (void)B;
  return align256(sizeof(WsHeader));
}

int fps_knn(const float* coords, const int64_t* offsets, int B, int64_t P, const float* centroids,
            const int32_t* valid_tokens, int K, int k, int32_t* knn_idx, const float* axis_scale, void* workspace,
            size_t workspace_bytes, fps_stream_t stream) {
  int rc = check_common(P, B, offsets);
  if (rc) return rc;
  float4 w;
  int scaled;
  if (!axis_scale_of(axis_scale, &w, &scaled)) return FPS_ERR_ARG;
  if (K < 1 || k < 1) return FPS_ERR_ARG;
  if (K > FPS_MAX_K || k > FPS_MAX_KNN) return FPS_ERR_TOO_LARGE;
  if (B == 0) return FPS_OK;
  if (!centroids || !knn_idx || (P > 0 && !coords)) return FPS_ERR_ARG;
  if (!aligned(coords, 16) || !aligned(centroids, 16)) return FPS_ERR_ARG;
  if (!workspace || workspace_bytes < fps_knn_workspace_bytes(P, B) || !aligned(workspace, 256))
    return FPS_ERR_WORKSPACE;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  WsHeader* hdr = static_cast<WsHeader*>(workspace);
  cudaError_t e;
  if ((e = cudaMemsetAsync(hdr, 0, sizeof(WsHeader), s))) return from_cuda(e);
  return from_cuda(launch_knn(reinterpret_cast<const float4*>(coords), offsets, B,
                              reinterpret_cast<const float4*>(centroids), valid_tokens, K, k, knn_idx, nullptr,
                              0, nullptr, nullptr, nullptr, hdr, s, w, scaled));
}

size_t lloyd_workspace_bytes(int64_t P, int B, int K) {
  if (K < 1) return 0;
  return carve(nullptr, P, B, K, 1, true, false).bytes;
}

int lloyd_refine(const float* coords, const float* feats, int F, int charge_col, const int64_t* offsets, int B,
                 int64_t P, int K, int iters, float* centroids, int32_t* token_id, const float* axis_scale,
                 void* workspace, size_t workspace_bytes, fps_stream_t stream) {
  int rc = check_common(P, B, offsets);
  if (rc) return rc;
  float4 w;
  int scaled;
  if (!axis_scale_of(axis_scale, &w, &scaled)) return FPS_ERR_ARG;
  if (K < 1 || iters < 0 || charge_col < -1) return FPS_ERR_ARG;
  if (K > FPS_MAX_K) return FPS_ERR_TOO_LARGE;
  if (charge_col >= 0 && (F < 1 || charge_col >= F || !feats)) return FPS_ERR_ARG;
  if (B == 0 || P == 0 || iters == 0) return FPS_OK;
  if (!coords || !centroids || !token_id) return FPS_ERR_ARG;
  if (!aligned(coords, 16) || !aligned(centroids, 16)) return FPS_ERR_ARG;
  const size_t need = lloyd_workspace_bytes(P, B, K);
  if (!workspace || workspace_bytes < need || !aligned(workspace, 256)) return FPS_ERR_WORKSPACE;
  const Workspace ws = carve(workspace, P, B, K, 1, true, false);
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  Problem pb = {};
  pb.coords = reinterpret_cast<const float4*>(coords);
  pb.feats = feats;
  pb.F = F;
  pb.offsets = offsets;
  pb.B = B;
  pb.P = P;
  pb.K = K;
  pb.lloyd_iters = iters;
  pb.charge_col = charge_col;
  pb.force_schedule = -1;
  pb.centroids = reinterpret_cast<float4*>(centroids);
  pb.w = w;
  pb.scaled = scaled;
  cudaError_t e;
  stage_mark(6, 0, s);
  if ((e = launch_bin(pb, ws, 0, s))) return from_cuda(e);
  const size_t zbytes = (size_t)ws.fps_slots * K * 5 * sizeof(double);
  if ((e = cudaMemsetAsync(ws.lloyd[0], 0, zbytes, s)) || (e = cudaMemsetAsync(ws.lloyd[1], 0, zbytes, s)))
    return from_cuda(e);
  if ((e = launch_lloyd(pb, ws, token_id, s))) return from_cuda(e);
  stage_mark(6, 1, s);
  return FPS_OK;
}

size_t segment_pool_workspace_bytes(int64_t P, int B, int K, int F) {
  if (K < 1 || F < 1) return 0;
  return carve(nullptr, P, B, K, F, false, false).bytes;
}

int segment_pool(const float* feats, int F, const int64_t* offsets, int B, int64_t P, int K, int mode,
                 const int32_t* token_id, const int32_t* knn_idx, int k, float* pooled, int32_t* counts,
                 void* workspace, size_t workspace_bytes, fps_stream_t stream) {
  if (B < 0 || P < 0) return FPS_ERR_ARG;
  if (P >= ((int64_t)1 << 31)) return FPS_ERR_TOO_LARGE;
  if (K < 1 || F < 1) return FPS_ERR_ARG;
  if (K > FPS_MAX_K || F > FPS_MAX_F) return FPS_ERR_TOO_LARGE;
  if (mode != FPS_ASSIGN_VORONOI && mode != FPS_ASSIGN_KNN) return FPS_ERR_ARG;
  if (B == 0) return FPS_OK;
  if (!pooled || !counts || (P > 0 && !feats)) return FPS_ERR_ARG;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  cudaError_t e;
  if (mode == FPS_ASSIGN_KNN) {
    if (k < 1) return FPS_ERR_ARG;
    if (k > FPS_MAX_KNN) return FPS_ERR_TOO_LARGE;
    if (!knn_idx) return FPS_ERR_ARG;
    if (!workspace || workspace_bytes < align256(sizeof(WsHeader)) || !aligned(workspace, 256))
      return FPS_ERR_WORKSPACE;
    WsHeader* hdr = static_cast<WsHeader*>(workspace);
    if ((e = cudaMemsetAsync(hdr, 0, sizeof(WsHeader), s))) return from_cuda(e);
    return from_cuda(launch_pool_knn(feats, F, B, K, k, knn_idx, P, pooled, counts, hdr, s));
  }
  if (!offsets || (P > 0 && !token_id)) return FPS_ERR_ARG;
  const size_t need = segment_pool_workspace_bytes(P, B, K, F);
  if (!workspace || workspace_bytes < need || !aligned(workspace, 256)) return FPS_ERR_WORKSPACE;
  const Workspace ws = carve(workspace, P, B, K, F, false, false);
  Problem pb = {};
  pb.offsets = offsets;
  pb.B = B;
  pb.P = P;
  pb.K = K;
  pb.F = F;
  pb.force_schedule = -1;
  // empty rows first (events without points), then pooled rows of every event
  if ((e = cudaMemsetAsync(pooled, 0, (size_t)B * K * F * sizeof(float), s)) ||
      (e = cudaMemsetAsync(counts, 0, (size_t)B * K * sizeof(int32_t), s)))
    return from_cuda(e);
  if ((e = launch_bin(pb, ws, 1, s))) return from_cuda(e);
  if ((e = cudaMemsetAsync(ws.pool_acc, 0, (size_t)ws.pool_slots * K * F * sizeof(double), s)) ||
      (e = cudaMemsetAsync(ws.pool_cnt, 0, (size_t)ws.pool_slots * K * sizeof(int), s)))
    return from_cuda(e);
  return from_cuda(launch_pool_voronoi(feats, F, offsets, B, K, token_id, pooled, counts, ws, s));
}

size_t segment_pool_backward_workspace_bytes(int64_t P, int B, int K, int F, int mode) {
  if (P < 0 || B < 0 || K < 1 || F < 1) return 0;
  size_t n = align256(sizeof(WsHeader));
  if (mode == FPS_ASSIGN_KNN) n += align256((size_t)P * F * sizeof(double) * 2);
  else n += align256((size_t)B * K * F * sizeof(float));
  return n;
}

int segment_pool_backward(const float* grad_pooled, int F, const int64_t* offsets, int B, int64_t P, int K,
                          int mode, const int32_t* token_id, const int32_t* knn_idx, int k, const int32_t* counts,
                          float* grad_feats, void* workspace, size_t workspace_bytes, fps_stream_t stream) {
  if (B < 0 || P < 0) return FPS_ERR_ARG;
  if (P >= ((int64_t)1 << 31)) return FPS_ERR_TOO_LARGE;
  if (K < 1 || F < 1) return FPS_ERR_ARG;
  if (K > FPS_MAX_K || F > FPS_MAX_F || (int64_t)B * K >= ((int64_t)1 << 31)) return FPS_ERR_TOO_LARGE;
  if (mode != FPS_ASSIGN_VORONOI && mode != FPS_ASSIGN_KNN) return FPS_ERR_ARG;
  if (P == 0) return FPS_OK;
  if (!grad_feats || (B > 0 && (!grad_pooled || !counts))) return FPS_ERR_ARG;
  if (mode == FPS_ASSIGN_KNN) {
    if (k < 1) return FPS_ERR_ARG;
    if (k > FPS_MAX_KNN) return FPS_ERR_TOO_LARGE;
    if (B > 0 && !knn_idx) return FPS_ERR_ARG;
  } else if (B == 0 || !offsets || !token_id) {
    return FPS_ERR_ARG;  // every point belongs to an event
  }
  const size_t need = segment_pool_backward_workspace_bytes(P, B, K, F, mode);
  if (!workspace || workspace_bytes < need || !aligned(workspace, 256)) return FPS_ERR_WORKSPACE;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  WsHeader* hdr = static_cast<WsHeader*>(workspace);
  char* scratch = static_cast<char*>(workspace) + align256(sizeof(WsHeader));
  if (mode == FPS_ASSIGN_KNN) {
    cudaError_t e;
    if ((e = cudaMemsetAsync(hdr, 0, sizeof(WsHeader), s))) return from_cuda(e);
    double* acc = reinterpret_cast<double*>(scratch);
    return from_cuda(
        launch_pool_bwd_knn(grad_pooled, F, offsets, B, K, k, knn_idx, counts, P, acc, grad_feats, hdr, s));
  }
  // the quotient kernel resets the status word (Voronoi: B > 0, so it runs)
  return from_cuda(launch_pool_bwd_voronoi(grad_pooled, F, offsets, B, P, K, token_id, counts,
                                           reinterpret_cast<float*>(scratch), grad_feats, hdr, s));
}

int fps_random_starts(const int64_t* offsets, int B, uint64_t seed, uint32_t stream_id, int32_t* start_local,
                      fps_stream_t stream) {
  if (B < 0) return FPS_ERR_ARG;
  if (B == 0) return FPS_OK;
  if (!offsets || !start_local) return FPS_ERR_ARG;
  return from_cuda(launch_random_starts(offsets, B, seed, stream_id, start_local, nullptr,
                                        reinterpret_cast<cudaStream_t>(stream)));
}

size_t fps_token_summaries_workspace_bytes(int B, int K, int F) {
  if (B < 0 || K < 1 || F < 1) return 0;
  return align256(sizeof(WsHeader)) + align256(token_summary_partial_bytes(K, F));
}

int fps_token_summaries(const float* coords, const float* feats, int F, int charge_col, const int64_t* offsets,
                        int B, int64_t P, int K, const int32_t* token_id, float* wsum, float* wcoords,
                        float* wfeats, void* workspace, size_t workspace_bytes, fps_stream_t stream) {
  int rc = check_common(P, B, offsets);
  if (rc) return rc;
  if (K < 1 || F < 1 || charge_col < -1 || charge_col >= F) return FPS_ERR_ARG;
  if (K > FPS_MAX_K || F > FPS_MAX_F) return FPS_ERR_TOO_LARGE;
  if (B == 0) return FPS_OK;
  if (!wsum || !wcoords || !wfeats || (P > 0 && (!coords || !feats || !token_id))) return FPS_ERR_ARG;
  if (P > 0 && !aligned(coords, 16)) return FPS_ERR_ARG;
  const size_t need = fps_token_summaries_workspace_bytes(B, K, F);
  if (!workspace || workspace_bytes < need || !aligned(workspace, 256)) return FPS_ERR_WORKSPACE;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  WsHeader* hdr = static_cast<WsHeader*>(workspace);
  double* partial = reinterpret_cast<double*>(static_cast<char*>(workspace) + align256(sizeof(WsHeader)));
  cudaError_t e;
  if ((e = cudaMemsetAsync(hdr, 0, sizeof(WsHeader), s))) return from_cuda(e);
  return from_cuda(launch_token_summaries(coords, feats, F, charge_col, offsets, B, P, K, token_id, partial, wsum,
                                          wcoords, wfeats, hdr, s));
}

size_t fps_pack_workspace_bytes(void) { return align256(sizeof(WsHeader)); }

int fps_pack_tokens(const float* src, int D, const int64_t* offsets, const int32_t* valid_tokens, int B, int K,
                    float* dst, int32_t* doc_id, int64_t* tok_offsets, void* workspace, size_t workspace_bytes,
                    fps_stream_t stream) {
  if (B < 0 || K < 1 || D < 1) return FPS_ERR_ARG;
  if ((int64_t)K * D >= ((int64_t)1 << 31)) return FPS_ERR_TOO_LARGE;
  if (!tok_offsets || (B > 0 && (!src || !dst || !doc_id || (!offsets && !valid_tokens)))) return FPS_ERR_ARG;
  if (!workspace || workspace_bytes < fps_pack_workspace_bytes() || !aligned(workspace, 256))
    return FPS_ERR_WORKSPACE;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  WsHeader* hdr = static_cast<WsHeader*>(workspace);  // its status word is reset by the scan kernel
  return from_cuda(launch_pack_tokens(src, D, offsets, valid_tokens, B, K, dst, doc_id, tok_offsets, hdr, s));
}

int fps_unpack_tokens(const float* src, int D, int64_t n_tok, const int64_t* tok_offsets, int B, int K, float* dst,
                      void* workspace, size_t workspace_bytes, fps_stream_t stream) {
  if (B < 0 || K < 1 || D < 1 || n_tok < 0) return FPS_ERR_ARG;
  if ((int64_t)K * D >= ((int64_t)1 << 31)) return FPS_ERR_TOO_LARGE;
  if (B == 0) return FPS_OK;
  if (!tok_offsets || !dst || (n_tok > 0 && !src)) return FPS_ERR_ARG;
  if (!workspace || workspace_bytes < fps_pack_workspace_bytes() || !aligned(workspace, 256))
    return FPS_ERR_WORKSPACE;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  WsHeader* hdr = static_cast<WsHeader*>(workspace);
  cudaError_t e;
  if ((e = cudaMemsetAsync(hdr, 0, sizeof(WsHeader), s))) return from_cuda(e);
  return from_cuda(launch_unpack_tokens(src, D, n_tok, tok_offsets, B, K, dst, hdr, s));
}

int fps_device_status(void* workspace, fps_stream_t stream, int* detail) {
  if (!workspace) return FPS_ERR_ARG;
  WsHeader h;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  cudaError_t e = cudaMemcpyAsync(&h, workspace, sizeof(WsHeader), cudaMemcpyDeviceToHost, s);
  if (e == cudaSuccess) e = cudaStreamSynchronize(s);
  if (e != cudaSuccess) return FPS_ERR_CUDA;
  if (detail) *detail = h.status;
  if (h.status == 0) return FPS_OK;
  const int zero[2] = {0, 0};
  cudaMemcpyAsync(workspace, zero, sizeof(zero), cudaMemcpyHostToDevice, s);
  cudaStreamSynchronize(s);
  return FPS_ERR_DEVICE;
}

const char* fps_status_string(int status) {
  switch (status) {
    case FPS_OK: return "ok";
    case FPS_ERR_ARG: return "invalid argument";
    case FPS_ERR_TOO_LARGE: return "size above a library limit";
    case FPS_ERR_WORKSPACE: return "workspace missing, too small or misaligned";
    case FPS_ERR_CUDA: return "CUDA launch or copy failed";
    case FPS_ERR_DEVICE: return "device-side check failed";
    default: return "unknown status";
  }
}

uint64_t fps_launch_count(void) { return g_launches.load(std::memory_order_relaxed); }

void fps_set_exchange_test(int spin_limit, int skip_rank) { set_exchange_test(spin_limit, skip_rank); }

void fps_set_stage_events(void* const* events, int n_events) {
  g_stage_mask = 0;
  if (!events || n_events <= 0) {
    g_n_stage_events = 0;
    return;
  }
  if (n_events > 32) n_events = 32;
  for (int i = 0; i < n_events; ++i) g_stage_events[i] = events[i];
  g_n_stage_events = n_events;
}

unsigned fps_stage_mask(void) { return g_stage_mask; }

}  // extern "C"
