/*
 * fpstok: batched 4D farthest-point-sampling tokenizer on B200 (sm_100a).
 *
 * What the library computes follows the Neptune tokenizer as the pages state it:
 *   - Neptune README, "How it works", step 1 (Tokenization): farthest-point
 *     sampling down to num_patches (K) centroids, then per-token pooling by
 *     nearest-centroid (Voronoi) assignment or a k-NN gather
 *     (assign_mode="knn", k_neighbors), with optional charge-weighted Lloyd
 *     refinement of the centroids (lloyd_iters).
 *   - graphnet PR #923 "Add Neptune point-transformer backbone", "What is
 *     added": FPSTokenizer keeps one token per pulse for small events;
 *     components/fps.py provides farthest_point_sampling, the _with_assign and
 *     _with_knn variants, and nearest_assign.  Review thread on the FPS
 *     `precision` argument: computation is float32 only.  Review thread on
 *     the no-charge case: unit charge when no charge column is given.
 *   - Neptune README, "Usage": coords [N, 4] = (x, y, z, t) with time in the
 *     fourth column, features [N, F], per-point event ids.
 *
 * Exact semantics (readings where the pages are silent):
 *   d(i, c) = ((dx*dx + dy*dy) + dz*dz) + dt*dt in float32, each operation
 *   rounded to nearest-even, never fused; with an optional per-axis scale w
 *   (the time scale of graphnet PR #923's review thread on the FPS
 *   arguments), both points' coordinates are first multiplied by w in float32
 *   (only the metric changes: centroid positions, Lloyd means and pooled
 *   values stay in the caller's units); first centroid = start_local[b]
 *   (default 0); each next centroid = the unselected point with the largest
 *   running minimum distance, lowest index on ties (when every unselected
 *   point is at distance 0, the lowest-index unselected point); Voronoi label
 *   = nearest centroid, lowest slot on ties; kNN row = the k points with the
 *   smallest (d, index), ascending, -1 padded; pooling = arithmetic mean of
 *   every feature column plus a count; Lloyd: c_j = sum(q p) / sum(q) over
 *   the cell (q = features[:, charge_col] or 1), c_j kept when the cell is
 *   empty or its weight <= 0, then re-assign; sums accumulate in float64 and
 *   round once to float32.  Indices, labels and kNN ids are exact; pooled
 *   values and Lloyd centroids agree with a sequential float64 sum to well
 *   within 1e-5 relative (1e-6 absolute floor).
 *
 * Layout (all row-major, packed by event):
 *   coords   float32 [P, 4], 16-byte aligned; event b is rows
 *            offsets[b] .. offsets[b+1]-1.
 *   feats    float32 [P, F], F >= 1.
 *   offsets  int64 [B + 1], offsets[0] = 0, non-decreasing, offsets[B] = P.
 *
 * Outputs per event b with N = offsets[b+1] - offsets[b] points:
 *   N == 0      : no tokens; rows are -1 (indices) or 0 (floats, counts).
 *   N <= K      : passthrough, token j is point j (j < N): centroid_idx =
 *                 offsets[b] + j, token_id = local index, kNN row =
 *                 [point, -1, ...], pooled = that point's features, count 1.
 *   N  > K      : K tokens from FPS; Lloyd applies only to these events.
 *   centroid_idx int32 [B, K]  global packed indices of the FPS points, -1 pad.
 *   token_id     int32 [P]     local token slot 0..K-1 of every point.
 *   knn_idx      int32 [B,K,k] global packed indices, -1 pad.
 *   centroids    float32 [B,K,4] centroid positions (Lloyd-refined if any).
 *   pooled       float32 [B,K,F], counts int32 [B, K].
 *
 * Ownership and execution: every pointer is a caller-owned buffer; the
 * library never allocates, frees or synchronises.  Unless stated otherwise
 * pointers are DEVICE pointers and all work is enqueued on `stream`.  Scratch
 * space is the caller's `workspace` (device, 256-byte aligned) of at least the
 * size the matching *_workspace_bytes() call returns.
 *
 * Errors: every call returns FPS_OK or an FPS_ERR_* code.  Argument errors
 * are found on the host before anything is launched.  Problems only visible
 * on the device (inconsistent offsets, a start index outside its event, a
 * token id outside 0..K-1) make the kernels skip the offending event and
 * record a code in the workspace; fps_device_status() reads it back (this
 * one call synchronises the stream).
 */
#ifndef FPSTOK_H
#define FPSTOK_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct CUstream_st *fps_stream_t; /* same type as cudaStream_t */

enum {
    FPS_OK = 0,
    FPS_ERR_ARG = 1,        /* null pointer, bad size, bad mode, misaligned */
    FPS_ERR_TOO_LARGE = 2,  /* K > FPS_MAX_K, k > K or > FPS_MAX_KNN, P >= 2^31,
                               an event above FPS_MAX_EVENT points, F > FPS_MAX_F */
    FPS_ERR_WORKSPACE = 3,  /* workspace missing, too small or misaligned */
    FPS_ERR_CUDA = 4,       /* a CUDA launch or copy failed */
    FPS_ERR_DEVICE = 5      /* a device-side check failed (fps_device_status) */
};

#define FPS_MAX_K 256
#define FPS_MAX_KNN 128
#define FPS_MAX_F 64

/* assign_mode */
#define FPS_ASSIGN_VORONOI 0
#define FPS_ASSIGN_KNN 1

/* force_schedule: -1 picks by event size; 0 warp (N <= 448), 1 CTA with points
 * in registers (N <= 2560), 2 CTA with points in shared memory (N <= 12288),
 * 3 8-CTA cluster (N <= 98304), 4 16-CTA cluster (N <= 196608) means "use at
 * least this schedule" (events too large for it move up). */
typedef struct fps_opts {
    int K;             /* maximum tokens per event, 1..FPS_MAX_K */
    int assign_mode;   /* FPS_ASSIGN_VORONOI or FPS_ASSIGN_KNN */
    int k;             /* kNN size, 1..min(K, FPS_MAX_KNN); ignored for Voronoi */
    int lloyd_iters;   /* >= 0 */
    int charge_col;    /* feature column used as Lloyd weight; -1 = unit weight */
    int force_schedule;
    int max_event_hint;/* upper bound on the largest event's N, 0 = unknown */
    float axis_scale[4];/* per-axis weights (wx, wy, wz, wt) of the distance: both points'
                           coordinates are multiplied by them (float32, rounded) before the
                           distance; all zero (a zero-initialised struct) = unscaled.  Finite. */
} fps_opts;

/* Largest event (points) the FPS schedules accept. */
int64_t fps_max_event_points(void);

/* Workspace bytes fps_tokenize needs for P points, B events and these options. */
size_t fps_workspace_bytes(int64_t P, int B, int F, const fps_opts *opts);

/*
 * The whole tokenizer: FPS (fused with the Voronoi labels) -> optional Lloyd
 * -> Voronoi mean-pool, or kNN gather around the final centroids and kNN
 * mean-pool.  start_local: int32 [B] local start index per event, or NULL for
 * 0.  token_id is required for Voronoi and optional (NULL) for kNN, where it
 * receives the Voronoi labels when given.  knn_idx is required for kNN and
 * ignored for Voronoi.  feats is required (F >= 1).
 */
int fps_tokenize(const float *coords, const float *feats, int F, const int64_t *offsets, int B,
                 int64_t P, const int32_t *start_local, const fps_opts *opts,
                 int32_t *centroid_idx, int32_t *token_id, int32_t *knn_idx, float *centroids,
                 float *pooled, int32_t *counts, void *workspace, size_t workspace_bytes,
                 fps_stream_t stream);

/*
 * Same as fps_tokenize but every input and output pointer is a HOST pointer
 * (page-locked memory gives asynchronous copies).  The inputs are staged into
 * the device workspace, the tokenizer runs there and the outputs are copied
 * back; the results are valid once `stream` is synchronised.  Batches of at
 * least 65,536 points and 256 events go through in 6 slices of consecutive
 * events (by points; the first and the last half as large as the others):
 * a slice's inputs are copied in on one internal
 * stream, it is tokenized on `stream`, and its outputs are copied out on
 * another internal stream, so that copies in, compute and copies out of
 * different slices overlap; `stream` waits for everything before it is
 * synchronised.  Because offsets and start_local are host data, they are
 * checked here (non-decreasing, offsets[0] = 0, offsets[B] = P, each start
 * inside its event) and a violation returns FPS_ERR_ARG before anything is
 * copied.  Workspace size: fps_host_workspace_bytes().
 */
size_t fps_host_workspace_bytes(int64_t P, int B, int F, const fps_opts *opts);
int fps_tokenize_host(const float *coords, const float *feats, int F, const int64_t *offsets,
                      int B, int64_t P, const int32_t *start_local, const fps_opts *opts,
                      int32_t *centroid_idx, int32_t *token_id, int32_t *knn_idx,
                      float *centroids, float *pooled, int32_t *counts, void *workspace,
                      size_t workspace_bytes, fps_stream_t stream);

/*
 * fps_tokenize for callers that cannot allocate device memory.  The pages
 * have no counterpart: this exists for callers embedded in a host program
 * that owns all device memory and may not call cudaMalloc or an allocating
 * library routine, or that cannot accept the synchronisation cudaMalloc can
 * cause.  Same arguments and results as fps_tokenize, without the workspace:
 * the scratch is a file-scope device array of FPS_STATIC_SCRATCH_BYTES
 * (8 MiB) that every GPU loading the library holds until the process exits.
 * Returns FPS_ERR_TOO_LARGE when the batch needs more scratch than that:
 * as much as fps_tokenize would take for the same arguments, which is
 * fps_workspace_bytes() except that kNN mode with Lloyd and a non-NULL
 * token_id needs no internal labels area.  The first call on each device
 * looks up the array's device address (cudaGetSymbolAddress); make it before
 * any stream capture.  That address is kept for the life of the process:
 * after cudaDeviceReset on a device, calling this entry point there is not
 * supported.  All calls share the array: calls whose work overlaps on the
 * GPU race.  It allocates and frees nothing.
 */
#define FPS_STATIC_SCRATCH_BYTES (8u << 20)
int fps_tokenize_static(const float *coords, const float *feats, int F, const int64_t *offsets,
                        int B, int64_t P, const int32_t *start_local, const fps_opts *opts,
                        int32_t *centroid_idx, int32_t *token_id, int32_t *knn_idx,
                        float *centroids, float *pooled, int32_t *counts, fps_stream_t stream);

/* fps_device_status for fps_tokenize_static: reads (and clears) the status
 * word that the last fps_tokenize_static call on the current device left in
 * the static array; synchronises `stream`.  Same results as
 * fps_device_status. */
int fps_static_device_status(fps_stream_t stream, int *detail);

/*
 * Nearest-centroid assignment (components/fps.py nearest_assign):
 * token_id[i] = argmin over the event's first valid_tokens[b] centroid rows of
 * d(p_i, c_j), lowest slot on ties; -1 when the event has no valid row.
 * centroids float32 [B, K, 4]; valid_tokens int32 [B] or NULL for min(N, K);
 * axis_scale: HOST pointer to the 4 per-axis weights of the distance (see
 * fps_opts), or NULL for unscaled.
 */
size_t fps_assign_workspace_bytes(int64_t P, int B);
int fps_assign(const float *coords, const int64_t *offsets, int B, int64_t P,
               const float *centroids, const int32_t *valid_tokens, int K, int32_t *token_id,
               const float *axis_scale, void *workspace, size_t workspace_bytes, fps_stream_t stream);

/*
 * kNN gather (graphnet PR #923, "What is added": farthest_point_sampling_with_knn
 * in components/fps.py; Neptune README, "How it works", step 1 and
 * "Parameters": assign_mode="knn" with k_neighbors): for every valid centroid
 * row j of event b, the k points of the event with the smallest
 * (d(p_i, c_j), i), ascending, as global indices, -1 padded when the event has
 * fewer than k points; invalid rows are all -1.  centroids float32 [B, K, 4];
 * valid_tokens int32 [B] or NULL for min(N, K); knn_idx int32 [B, K, k];
 * axis_scale: HOST pointer to the 4 per-axis weights (see fps_opts) or NULL.
 * Workspace: fps_knn_workspace_bytes() (a status word), 256-byte aligned.
 */
size_t fps_knn_workspace_bytes(int64_t P, int B);
int fps_knn(const float *coords, const int64_t *offsets, int B, int64_t P,
            const float *centroids, const int32_t *valid_tokens, int K, int k,
            int32_t *knn_idx, const float *axis_scale, void *workspace, size_t workspace_bytes,
            fps_stream_t stream);

/*
 * Charge-weighted Lloyd refinement (README "How it works", step 1) of the
 * events with N > K: `iters` times, every centroid moves to the weighted mean
 * of its cell (q = feats[:, charge_col], or 1 when charge_col = -1; kept when
 * the cell is empty or its weight <= 0) and every point is re-assigned.
 * centroids [B,K,4] and token_id [P] are read and updated in place; events
 * with N <= K are left untouched.  feats may be NULL when charge_col = -1.
 * axis_scale: HOST pointer to the 4 per-axis weights of the re-assignment's
 * distance (see fps_opts) or NULL; the means stay in the caller's units.
 */
size_t lloyd_workspace_bytes(int64_t P, int B, int K);
int lloyd_refine(const float *coords, const float *feats, int F, int charge_col,
                 const int64_t *offsets, int B, int64_t P, int K, int iters, float *centroids,
                 int32_t *token_id, const float *axis_scale, void *workspace, size_t workspace_bytes,
                 fps_stream_t stream);

/*
 * Per-token mean-pool ("pools the pulses of each token", graphnet PR #923,
 * Summary).  mode FPS_ASSIGN_VORONOI: pooled[b,j,:] = mean of feats over the
 * points of event b with token_id == j (token_id -1 = unassigned, skipped).
 * mode FPS_ASSIGN_KNN: pooled[b,j,:] = mean of feats over the non-negative
 * entries of knn_idx[b,j,:] (k entries per row; `offsets` may be NULL).
 * Empty tokens give 0 and count 0.
 */
size_t segment_pool_workspace_bytes(int64_t P, int B, int K, int F);
int segment_pool(const float *feats, int F, const int64_t *offsets, int B, int64_t P, int K,
                 int mode, const int32_t *token_id, const int32_t *knn_idx, int k,
                 float *pooled, int32_t *counts, void *workspace, size_t workspace_bytes,
                 fps_stream_t stream);

/*
 * Backward of segment_pool: the gradient of the pooled rows with respect to
 * the features (graphnet PR #923, "What is added": the tokenizer sits inside
 * the training step, and the tests check gradients).  The pool is linear, so
 * with the forward's counts [B, K]:
 *   mode FPS_ASSIGN_VORONOI: grad_feats[i,:] = grad_pooled[b, t, :] / counts[b, t]
 *     for t = token_id[i] of point i of event b; 0 when t = -1 or the count
 *     is 0.  offsets and token_id are required.  The result is exact: the
 *     float32 division correctly rounded.
 *   mode FPS_ASSIGN_KNN: grad_feats[i,:] = sum over the rows (b, j) whose
 *     knn_idx entries hold i of grad_pooled[b, j, :] / counts[b, j]; 0 for a
 *     point no row gathered.  The shares are float64 and the sum rounds once
 *     to float32.  With offsets (else NULL), an event whose rows name only
 *     its own points and that fits the kernel's shared buffer (about 10^4
 *     points at K = 128, k = 32, F = 6) is summed in row order, exactly as a
 *     sequential loop over the rows would; other entries (they may name any
 *     point in 0..P-1) meet in float64 in no fixed order.
 * grad_pooled float32 [B, K, F]; grad_feats float32 [P, F] (every row is
 * written).  Device-side problems (a token outside -1..K-1, a kNN index >= P,
 * offsets that do not cover the points) leave that point's gradient 0 and
 * are reported by fps_device_status().  Workspace: the size below (device,
 * 256-byte aligned): about B * K * F * 4 bytes in Voronoi mode, P * F * 16
 * in kNN mode.
 */
size_t segment_pool_backward_workspace_bytes(int64_t P, int B, int K, int F, int mode);
int segment_pool_backward(const float *grad_pooled, int F, const int64_t *offsets, int B, int64_t P,
                          int K, int mode, const int32_t *token_id, const int32_t *knn_idx, int k,
                          const int32_t *counts, float *grad_feats, void *workspace,
                          size_t workspace_bytes, fps_stream_t stream);

/*
 * Random FPS start points (graphnet PR #923, review thread on the FPS
 * arguments: start_idx, random_start and a generator), for fps_tokenize's
 * start_local.  start_local[b] = floor(u * N_b / 2^32) with u the first word
 * of Philox4x32-10 (Salmon et al., SC 2011) at counter (b, stream_id, 0, 0)
 * under the key (seed & 0xffffffff, seed >> 32); 0 for an empty event (or
 * for an event whose offsets are inconsistent).  Deterministic for a given
 * seed and stream_id; change stream_id to draw new starts from the same
 * seed.  No workspace.
 */
int fps_random_starts(const int64_t *offsets, int B, uint64_t seed, uint32_t stream_id,
                      int32_t *start_local, fps_stream_t stream);

/*
 * Charge-weighted token summaries (graphnet PR #923, review thread on the
 * no-charge case: the tokenizer uses the charge for weighting and for token
 * summaries, unit charge when there is no charge column; review thread on
 * time encoding: the charge-weighted mean time).  The pages do not list the
 * summaries; this library's reading, per Voronoi token j of event b over the
 * points with token_id == j and q = feats[:, charge_col] (1 when
 * charge_col = -1):
 *   wsum    float32 [B, K]    = sum q
 *   wcoords float32 [B, K, 4] = sum q * coords / wsum   (x, y, z, t)
 *   wfeats  float32 [B, K, F] = sum q * feats / wsum
 * Sums in float64 (in no fixed order), each output rounded once to float32;
 * the means are 0 for an empty cell or wsum <= 0.  Token ids outside -1..K-1
 * and offsets that do not cover the points are skipped and reported by
 * fps_device_status().  Workspace: the size below (it does not depend on B),
 * 256-byte aligned: a status word and the float64 partial sums of the events
 * cut by the boundaries of the per-CTA point ranges, 2 * K * (5 + F) values
 * for each of up to 512 ranges (as many as fit in 32 MiB, at least one).
 */
size_t fps_token_summaries_workspace_bytes(int B, int K, int F);
int fps_token_summaries(const float *coords, const float *feats, int F, int charge_col,
                        const int64_t *offsets, int B, int64_t P, int K, const int32_t *token_id,
                        float *wsum, float *wcoords, float *wfeats, void *workspace,
                        size_t workspace_bytes, fps_stream_t stream);

/*
 * Packed token layout for block-diagonal attention (graphnet PR #923, "What
 * is added": models/utils.py pack / unpack / build_block_mask; review thread
 * on the block mask: doc_id is the event index of every packed token, and
 * tokens attend to each other when their doc_ids match).  Event b has v_b
 * tokens: valid_tokens[b] when given (0..K), else min(N_b, K) from the point
 * offsets (the slots the tokenizer fills).
 *   fps_pack_tokens: tok_offsets [B+1] = 0, v_0, v_0 + v_1, ... (int64);
 *     dst [tok_offsets[B], D] row tok_offsets[b] + j = src [B, K, D] row
 *     (b, j) for j < v_b; doc_id [tok_offsets[B]] int32 = b on those rows.
 *     dst and doc_id must hold B * K rows (the packed length is only known on
 *     the device: read tok_offsets[B]).  offsets may be NULL when
 *     valid_tokens is given.
 *   fps_unpack_tokens: dst [B, K, D] row (b, j) = src row tok_offsets[b] + j
 *     for j < v_b = tok_offsets[b+1] - tok_offsets[b], 0 for j >= v_b; src
 *     holds n_tok rows.  An event whose span is not inside 0..n_tok or whose
 *     v_b is outside 0..K is written as padding and reported by
 *     fps_device_status().
 * Workspace: fps_pack_workspace_bytes() (a status word), 256-byte aligned.
 */
size_t fps_pack_workspace_bytes(void);
int fps_pack_tokens(const float *src, int D, const int64_t *offsets, const int32_t *valid_tokens, int B,
                    int K, float *dst, int32_t *doc_id, int64_t *tok_offsets, void *workspace,
                    size_t workspace_bytes, fps_stream_t stream);
int fps_unpack_tokens(const float *src, int D, int64_t n_tok, const int64_t *tok_offsets, int B, int K,
                      float *dst, void *workspace, size_t workspace_bytes, fps_stream_t stream);

/* Reads (and clears) the device-side status word in `workspace`; synchronises
 * `stream`.  Returns FPS_OK or FPS_ERR_DEVICE; *detail (optional) receives the
 * recorded reason (see FPS_DEV_* below). */
int fps_device_status(void *workspace, fps_stream_t stream, int *detail);

#define FPS_DEV_BAD_OFFSETS 1
#define FPS_DEV_BAD_START 2
#define FPS_DEV_BAD_TOKEN 3
#define FPS_DEV_TOO_LARGE 4
/* A cluster FPS kernel gave up waiting for its peers' candidates (a bounded
 * wait ran out); that launch's results are not valid. */
#define FPS_DEV_EXCHANGE_TIMEOUT 5

/*
 * Test hook of the cluster schedules' bounded exchange wait (host side only;
 * it faults nothing).  Each exchange round of an 8- or 16-CTA cluster waits
 * at most spin_limit polls of its mbarrier (spin_limit <= 0: the default,
 * 2^20 polls); with skip_rank >= 0, CTA skip_rank of every cluster skips its
 * post in the first exchange of each event, so every wait of that round runs
 * out.  A wait that runs out records FPS_DEV_EXCHANGE_TIMEOUT; that CTA leaves
 * the event at once, its peers leave within one more round, and the whole
 * cluster then stops taking events: the launch's results are not valid, the
 * CUDA context stays usable.  Applies to the launches made after the call;
 * fps_set_exchange_test(0, -1) restores the defaults.
 */
void fps_set_exchange_test(int spin_limit, int skip_rank);

/* Human-readable name of a status code. */
const char *fps_status_string(int status);

/* Number of kernels this library has launched in this process (a counter
 * for measurement; it is not reset). */
uint64_t fps_launch_count(void);

/*
 * Measurement hook: when `events` is non-NULL the next calls record
 * events[2*s] before and events[2*s+1] after internal stage s on the
 * launching stream (the block schedules run on internal helper streams forked
 * from it; their events are recorded there).  Stages: 0 binning, 1 FPS warp
 * schedule, 2 FPS CTA schedule, 3 FPS CTA shared-memory schedule, 4 FPS 8-CTA
 * cluster, 5 FPS 16-CTA cluster, 6 Lloyd, 7 kNN gather + pool, 8 Voronoi pool
 * (events not pooled by their FPS kernel), 9 passthrough.  In kNN mode
 * without Lloyd each FPS stage also covers the kNN rows of its events (they
 * run on that schedule's stream) and stage 7 is not used.  A stage that does
 * not run records nothing.  The events are cudaEvent_t handles the caller created; at most 32
 * are used.  Pass NULL to turn it off.  Not thread-safe: meant for benchmarks.
 */
void fps_set_stage_events(void *const *events, int n_events);

/* Bit s set: stage s was started (its first event recorded) by a call since
 * the last fps_set_stage_events.  Host-side bookkeeping for benchmarks. */
unsigned fps_stage_mask(void);

/* Schedule fps_tokenize gives an event of n points: -1 none (n <= K, or n = 0),
 * 0 warp, 1 CTA, 2 CTA shared-memory, 3 8-CTA cluster, 4 16-CTA cluster; -2
 * if n exceeds fps_max_event_points().  Two batch-level rules apply on top
 * (automatic scheduling only): when a batch has at most one FPS event per SM,
 * events of class 0 run on schedule 1; when it has at most one class-2 event
 * per 8 SMs, those run on schedule 3. */
int fps_schedule_for(int64_t n, int K, int force_schedule);

#ifdef __cplusplus
}
#endif

#endif /* FPSTOK_H */
