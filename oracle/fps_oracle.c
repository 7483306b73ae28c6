/*
 * CPU oracle for the batched 4D farthest-point-sampling tokenizer.
 *
 * TEST INFRASTRUCTURE ONLY.  Only tests/, __graft_entry__.smoke() and the
 * CPU-baseline / reference legs of bench.py may load or run this file.  It
 * shares no code, header or constant with the CUDA library and never calls it.
 *
 * What it computes (plain loops, one event after another, no blocking):
 *
 *   Neptune README, "How it works", step 1 (Tokenization): farthest-point
 *   sampling of each event down to at most num_patches (K) centroids, then
 *   per-token pooling by nearest-centroid (Voronoi) assignment or by a kNN
 *   gather, with optional charge-weighted Lloyd refinement of the centroids.
 *
 *   graphnet PR #923 "Add Neptune point-transformer backbone", "What is
 *   added": FPSTokenizer keeps one token per pulse for small events;
 *   components/fps.py names farthest_point_sampling(_with_assign/_with_knn)
 *   and nearest_assign.  Review thread on the FPS `precision` argument: both
 *   backends always compute in float32.  Review thread on the no-charge case:
 *   unit charge when there is no charge column.
 *
 * Readings where the pages are silent:
 *   - distance d(i,c) = ((dx*dx + dy*dy) + dz*dz) + dt*dt in float32, each
 *     operation rounded to nearest, no fused multiply-add (build with
 *     -ffp-contract=off), raw (x,y,z,t), t unscaled by default;
 *   - optional per-axis scale w = (wx, wy, wz, wt) (the time scale of the
 *     review thread on the FPS arguments): both points' coordinates are
 *     first multiplied by their axis weight in float32, then the distance
 *     above is taken; w = NULL means no scaling, and w = (1,1,1,1) gives the
 *     same bits.  Only the metric changes: centroid positions, Lloyd means
 *     and pooled values stay in the caller's units;
 *   - first centroid = start_local[b] (default 0, the event's first point);
 *   - next centroid = the unselected point with the largest running minimum
 *     distance, lowest index on ties (so with only duplicates left it is the
 *     lowest-index unselected point and indices stay distinct);
 *   - events with N <= K pass through: token j is point j;
 *   - Voronoi label = nearest centroid, lowest slot on ties;
 *   - kNN row = the k points with smallest (d, index), ascending, -1 padded;
 *     a passthrough token's row is [its own point, -1, ...];
 *   - pooling = plain mean of all F feature columns plus a count;
 *   - Lloyd: c_j = sum(q_i p_i) / sum(q_i) over the cell of j (q = charge
 *     column, or 1), the old c_j kept when the cell is empty or the weight is
 *     <= 0; every iteration re-assigns; no Lloyd on passthrough events;
 *   - sums (pool, Lloyd) accumulate in float64 and round once to float32.
 *
 * Return values: 0 on success, -1 on an argument error.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

/* Squared 4D distance with the fixed operation order (see header comment). */
float fpso_dist(const float *p, const float *c)
{
    float dx = p[0] - c[0];
    float dy = p[1] - c[1];
    float dz = p[2] - c[2];
    float dt = p[3] - c[3];
    float s = dx * dx + dy * dy;
    s = s + dz * dz;
    s = s + dt * dt;
    return s;
}

/*
 * The same distance with a per-axis scale: p and c are scaled coordinate by
 * coordinate, each product rounded to float32, before the distance above.
 */
float fpso_dist_w(const float *p, const float *c, const float *w)
{
    if (w == NULL) return fpso_dist(p, c);
    float ps[4], cs[4];
    for (int a = 0; a < 4; ++a) {
        ps[a] = w[a] * p[a];
        cs[a] = w[a] * c[a];
    }
    return fpso_dist(ps, cs);
}

static int bad_offsets(const int64_t *offsets, int B)
{
    if (B < 0 || offsets == NULL) return 1;
    if (B > 0 && offsets[0] != 0) return 1;
    for (int b = 0; b < B; ++b)
        if (offsets[b + 1] < offsets[b]) return 1;
    return 0;
}

/*
 * Farthest point sampling (the greedy farthest-point recurrence).
 * centroid_idx [B,K]: global packed indices, -1 padded.
 * sel_dist [B,K] (optional): for slot s >= 1 the running minimum distance the
 * s-th centroid had when it was chosen; slot 0 and passthrough slots get -1.
 */
int fpso_fps(const float *coords, const int64_t *offsets, int B, int K,
             const int32_t *start_local, const float *w, int32_t *centroid_idx, float *sel_dist)
{
    if (K < 1 || bad_offsets(offsets, B)) return -1;
    for (int64_t e = 0; e < (int64_t)B * K; ++e) {
        centroid_idx[e] = -1;
        if (sel_dist) sel_dist[e] = -1.0f;
    }
    for (int b = 0; b < B; ++b) {
        int64_t off = offsets[b];
        int64_t n = offsets[b + 1] - off;
        int32_t *out = centroid_idx + (int64_t)b * K;
        if (n == 0) continue;
        if (n <= K) {
            for (int64_t j = 0; j < n; ++j) out[j] = (int32_t)(off + j);
            continue;
        }
        int64_t c = start_local ? start_local[b] : 0;
        if (c < 0 || c >= n) return -1;
        float *dist = (float *)malloc(sizeof(float) * n);
        unsigned char *chosen = (unsigned char *)calloc(n, 1);
        for (int64_t i = 0; i < n; ++i) dist[i] = INFINITY;
        for (int s = 0; s < K; ++s) {
            out[s] = (int32_t)(off + c);
            chosen[c] = 1;
            if (s == K - 1) break;
            const float *pc = coords + 4 * (off + c);
            for (int64_t i = 0; i < n; ++i) {
                float d = fpso_dist_w(coords + 4 * (off + i), pc, w);
                if (d < dist[i]) dist[i] = d;
            }
            int64_t best = -1;
            for (int64_t i = 0; i < n; ++i) {
                if (chosen[i]) continue;
                if (best < 0 || dist[i] > dist[best]) best = i;
            }
            if (sel_dist) sel_dist[(int64_t)b * K + s + 1] = dist[best];
            c = best;
        }
        free(dist);
        free(chosen);
    }
    return 0;
}

/* valid tokens of event b: valid[b] if given, else min(N, K). */
static int64_t n_valid(const int32_t *valid, int b, int64_t n, int K)
{
    if (valid) return valid[b];
    return n < K ? n : K;
}

/*
 * Nearest-centroid (Voronoi) assignment: token_id[i] = argmin_j d(p_i, c_j)
 * over the event's valid centroid rows, lowest slot on ties; -1 when the
 * event has no valid centroid.
 */
int fpso_assign(const float *coords, const int64_t *offsets, int B,
                const float *centroids, const int32_t *valid, int K, const float *w, int32_t *token_id)
{
    if (K < 1 || bad_offsets(offsets, B)) return -1;
    for (int b = 0; b < B; ++b) {
        int64_t off = offsets[b], n = offsets[b + 1] - off;
        int64_t nv = n_valid(valid, b, n, K);
        if (nv < 0 || nv > K) return -1;
        const float *cb = centroids + (int64_t)b * K * 4;
        for (int64_t i = 0; i < n; ++i) {
            const float *p = coords + 4 * (off + i);
            int32_t lab = -1;
            float best = 0.0f;
            for (int64_t j = 0; j < nv; ++j) {
                float d = fpso_dist_w(p, cb + 4 * j, w);
                if (lab < 0 || d < best) {
                    best = d;
                    lab = (int32_t)j;
                }
            }
            token_id[off + i] = lab;
        }
    }
    return 0;
}

typedef struct {
    float d;
    int64_t i;
} dkey;

static int dkey_cmp(const void *a, const void *b)
{
    const dkey *x = (const dkey *)a, *y = (const dkey *)b;
    if (x->d < y->d) return -1;
    if (x->d > y->d) return 1;
    return (x->i > y->i) - (x->i < y->i);
}

/*
 * kNN gather: for each valid centroid row j of event b, the k points of the
 * event with the smallest (d(p_i, c_j), i), ascending, as global indices;
 * -1 padded when the event has fewer than k points; invalid rows all -1.
 */
int fpso_knn(const float *coords, const int64_t *offsets, int B, const float *centroids,
             const int32_t *valid, int K, int k, const float *w, int32_t *knn_idx)
{
    if (K < 1 || k < 1 || bad_offsets(offsets, B)) return -1;
    for (int64_t e = 0; e < (int64_t)B * K * k; ++e) knn_idx[e] = -1;
    for (int b = 0; b < B; ++b) {
        int64_t off = offsets[b], n = offsets[b + 1] - off;
        int64_t nv = n_valid(valid, b, n, K);
        if (nv < 0 || nv > K) return -1;
        if (n == 0) continue;
        dkey *keys = (dkey *)malloc(sizeof(dkey) * n);
        for (int64_t j = 0; j < nv; ++j) {
            const float *c = centroids + ((int64_t)b * K + j) * 4;
            for (int64_t i = 0; i < n; ++i) {
                keys[i].d = fpso_dist_w(coords + 4 * (off + i), c, w);
                keys[i].i = i;
            }
            qsort(keys, (size_t)n, sizeof(dkey), dkey_cmp);
            int32_t *row = knn_idx + ((int64_t)b * K + j) * k;
            for (int64_t r = 0; r < k && r < n; ++r) row[r] = (int32_t)(off + keys[r].i);
        }
        free(keys);
    }
    return 0;
}

/*
 * Charge-weighted Lloyd refinement of events with N > K (all K rows valid).
 * Each iteration: W_j = sum q_i, S_j = sum q_i p_i over the points labelled j
 * (float64, point order), c_j = float(S_j / W_j) when W_j > 0, else c_j kept;
 * then every point is re-assigned to its nearest centroid.
 */
int fpso_lloyd(const float *coords, const float *feats, int F, int charge_col,
               const int64_t *offsets, int B, int K, int iters, const float *w,
               float *centroids, int32_t *token_id)
{
    if (K < 1 || iters < 0 || charge_col >= F || bad_offsets(offsets, B)) return -1;
    double *W = (double *)malloc(sizeof(double) * K);
    double *S = (double *)malloc(sizeof(double) * K * 4);
    for (int b = 0; b < B; ++b) {
        int64_t off = offsets[b], n = offsets[b + 1] - off;
        if (n <= K) continue;
        float *cb = centroids + (int64_t)b * K * 4;
        for (int it = 0; it < iters; ++it) {
            for (int j = 0; j < K; ++j) {
                W[j] = 0.0;
                for (int a = 0; a < 4; ++a) S[4 * j + a] = 0.0;
            }
            for (int64_t i = 0; i < n; ++i) {
                int32_t j = token_id[off + i];
                if (j < 0 || j >= K) {
                    free(W);
                    free(S);
                    return -1;
                }
                double q = charge_col < 0 ? 1.0 : (double)feats[(off + i) * F + charge_col];
                W[j] += q;
                for (int a = 0; a < 4; ++a) S[4 * j + a] += q * (double)coords[4 * (off + i) + a];
            }
            for (int j = 0; j < K; ++j)
                if (W[j] > 0.0)
                    for (int a = 0; a < 4; ++a) cb[4 * j + a] = (float)(S[4 * j + a] / W[j]);
            for (int64_t i = 0; i < n; ++i) {
                const float *p = coords + 4 * (off + i);
                int32_t lab = 0;
                float best = fpso_dist_w(p, cb, w);
                for (int j = 1; j < K; ++j) {
                    float d = fpso_dist_w(p, cb + 4 * j, w);
                    if (d < best) {
                        best = d;
                        lab = j;
                    }
                }
                token_id[off + i] = lab;
            }
        }
    }
    free(W);
    free(S);
    return 0;
}

/* Voronoi mean-pool: pooled[b,j,:] = mean of features over points labelled j. */
int fpso_pool_voronoi(const float *feats, int F, const int64_t *offsets, int B, int K,
                      const int32_t *token_id, float *pooled, int32_t *counts)
{
    if (K < 1 || F < 1 || bad_offsets(offsets, B)) return -1;
    double *sum = (double *)malloc(sizeof(double) * (size_t)K * F);
    int64_t *cnt = (int64_t *)malloc(sizeof(int64_t) * K);
    for (int b = 0; b < B; ++b) {
        int64_t off = offsets[b], n = offsets[b + 1] - off;
        for (int64_t e = 0; e < (int64_t)K * F; ++e) sum[e] = 0.0;
        for (int j = 0; j < K; ++j) cnt[j] = 0;
        for (int64_t i = 0; i < n; ++i) {
            int32_t j = token_id[off + i];
            if (j < 0) continue;
            if (j >= K) {
                free(sum);
                free(cnt);
                return -1;
            }
            cnt[j] += 1;
            for (int f = 0; f < F; ++f) sum[(int64_t)j * F + f] += (double)feats[(off + i) * F + f];
        }
        for (int j = 0; j < K; ++j) {
            counts[(int64_t)b * K + j] = (int32_t)cnt[j];
            for (int f = 0; f < F; ++f)
                pooled[((int64_t)b * K + j) * F + f] =
                    cnt[j] ? (float)(sum[(int64_t)j * F + f] / (double)cnt[j]) : 0.0f;
        }
    }
    free(sum);
    free(cnt);
    return 0;
}

/* kNN mean-pool: pooled[b,j,:] = mean of features over the valid row entries. */
int fpso_pool_knn(const float *feats, int F, int B, int K, int k, const int32_t *knn_idx,
                  float *pooled, int32_t *counts)
{
    if (K < 1 || F < 1 || k < 1 || B < 0) return -1;
    double *sum = (double *)malloc(sizeof(double) * F);
    for (int64_t r = 0; r < (int64_t)B * K; ++r) {
        const int32_t *row = knn_idx + r * k;
        int64_t cnt = 0;
        for (int f = 0; f < F; ++f) sum[f] = 0.0;
        for (int e = 0; e < k; ++e) {
            if (row[e] < 0) continue;
            cnt += 1;
            for (int f = 0; f < F; ++f) sum[f] += (double)feats[(int64_t)row[e] * F + f];
        }
        counts[r] = (int32_t)cnt;
        for (int f = 0; f < F; ++f) pooled[r * F + f] = cnt ? (float)(sum[f] / (double)cnt) : 0.0f;
    }
    free(sum);
    return 0;
}

/*
 * Backward of the Voronoi mean-pool: the vector-Jacobian product of
 * fpso_pool_voronoi with respect to the features (graphnet PR #923, "What is
 * added": the tests check gradients through the model, and the tokenizer sits
 * inside the training step).  The pool is linear: point i of cell j enters
 * pooled[b,j,:] with weight 1/counts[b,j], so
 *   grad_feats[i,f] = grad_pooled[b, token_id[i], f] / counts[b, token_id[i]],
 * the quotient taken in float64 and rounded once, and 0 for an unassigned
 * point (token_id -1) or a cell whose count is 0.  counts are the forward's.
 */
int fpso_pool_voronoi_backward(const float *grad_pooled, int F, const int64_t *offsets, int B, int K,
                               const int32_t *token_id, const int32_t *counts, float *grad_feats)
{
    if (K < 1 || F < 1 || bad_offsets(offsets, B)) return -1;
    for (int b = 0; b < B; ++b) {
        for (int64_t i = offsets[b]; i < offsets[b + 1]; ++i) {
            int32_t j = token_id[i];
            if (j >= K) return -1;
            int32_t c = j >= 0 ? counts[(int64_t)b * K + j] : 0;
            for (int f = 0; f < F; ++f) {
                float g = 0.0f;
                if (c > 0) g = (float)((double)grad_pooled[((int64_t)b * K + j) * F + f] / (double)c);
                grad_feats[i * F + f] = g;
            }
        }
    }
    return 0;
}

/*
 * Backward of the kNN mean-pool: every valid entry i of row r = (b, j) took
 * feats[i,:] with weight 1/counts[r], so grad_feats[i,:] is the sum over all
 * rows that gathered i of grad_pooled[r,:] / counts[r].  The quotients and the
 * sum are float64 (rows in order), rounded once to float32; points no row
 * gathered get 0.  P is the number of feature rows.
 */
int fpso_pool_knn_backward(const float *grad_pooled, int F, int B, int K, int k, const int32_t *knn_idx,
                           const int32_t *counts, int64_t P, float *grad_feats)
{
    if (K < 1 || F < 1 || k < 1 || B < 0 || P < 0) return -1;
    double *acc = (double *)calloc((size_t)(P > 0 ? P : 1) * F, sizeof(double));
    for (int64_t r = 0; r < (int64_t)B * K; ++r) {
        if (counts[r] <= 0) continue;
        for (int e = 0; e < k; ++e) {
            int32_t i = knn_idx[r * k + e];
            if (i < 0) continue;
            if (i >= P) {
                free(acc);
                return -1;
            }
            for (int f = 0; f < F; ++f)
                acc[(int64_t)i * F + f] += (double)grad_pooled[r * F + f] / (double)counts[r];
        }
    }
    for (int64_t e = 0; e < P * F; ++e) grad_feats[e] = (float)acc[e];
    free(acc);
    return 0;
}

/*
 * Philox4x32-10 (Salmon, Moraes, Dror and Shaw, "Parallel random numbers: as
 * easy as 1, 2, 3", SC 2011), written from its definition: ten rounds of
 *   (hi0, lo0) = M0 * c0,  (hi1, lo1) = M1 * c2   (32 x 32 -> 64-bit products)
 *   c <- (hi1 ^ c1 ^ k0, lo1, hi0 ^ c3 ^ k1, lo0)
 * with M0 = 0xD2511F53, M1 = 0xCD9E8D57, and the key raised by the Weyl
 * constants (0x9E3779B9, 0xBB67AE85) between rounds.
 */
void fpso_philox4x32_10(const uint32_t ctr_in[4], const uint32_t key_in[2], uint32_t out[4])
{
    uint32_t c0 = ctr_in[0], c1 = ctr_in[1], c2 = ctr_in[2], c3 = ctr_in[3];
    uint32_t k0 = key_in[0], k1 = key_in[1];
    for (int round = 0; round < 10; ++round) {
        if (round > 0) {
            k0 += 0x9E3779B9u;
            k1 += 0xBB67AE85u;
        }
        uint64_t p0 = (uint64_t)0xD2511F53u * c0;
        uint64_t p1 = (uint64_t)0xCD9E8D57u * c2;
        uint32_t hi0 = (uint32_t)(p0 >> 32), lo0 = (uint32_t)p0;
        uint32_t hi1 = (uint32_t)(p1 >> 32), lo1 = (uint32_t)p1;
        uint32_t n0 = hi1 ^ c1 ^ k0, n1 = lo1, n2 = hi0 ^ c3 ^ k1, n3 = lo0;
        c0 = n0;
        c1 = n1;
        c2 = n2;
        c3 = n3;
    }
    out[0] = c0;
    out[1] = c1;
    out[2] = c2;
    out[3] = c3;
}

/*
 * Random FPS start points (graphnet PR #923, review thread on the FPS
 * arguments: start_idx, random_start and a generator).  Reading: event b
 * starts at start_local[b] = floor(u * N_b / 2^32), u the first word of
 * Philox4x32-10 at counter (b, stream, 0, 0) under key (seed low word, seed
 * high word); 0 for an empty event.
 */
int fpso_random_starts(const int64_t *offsets, int B, uint64_t seed, uint32_t stream, int32_t *start_local)
{
    if (B < 0 || bad_offsets(offsets, B)) return -1;
    const uint32_t key[2] = {(uint32_t)seed, (uint32_t)(seed >> 32)};
    for (int b = 0; b < B; ++b) {
        const uint32_t ctr[4] = {(uint32_t)b, stream, 0u, 0u};
        uint32_t x[4];
        fpso_philox4x32_10(ctr, key, x);
        uint64_t n = (uint64_t)(offsets[b + 1] - offsets[b]);
        start_local[b] = (int32_t)(((uint64_t)x[0] * n) >> 32);
    }
    return 0;
}

/*
 * Charge-weighted token summaries (graphnet PR #923, review thread on the
 * no-charge case: the tokenizer uses the charge for weighting and for token
 * summaries, with unit charge when there is no charge column; review thread
 * on time encoding: a charge-weighted mean time).  The pages do not list the
 * summaries; the reading taken here, per Voronoi token j of event b with
 * cell C = {i in b : token_id[i] = j} and q_i = feats[i, charge_col] (1 when
 * charge_col = -1):
 *   wsum[b,j]      = sum_{i in C} q_i
 *   wcoords[b,j,:] = sum q_i * coords[i,:] / wsum   (position and time)
 *   wfeats[b,j,:]  = sum q_i * feats[i,:] / wsum
 * sums in float64 in point order, each output rounded once to float32; the
 * means are 0 when the cell is empty or wsum <= 0.
 */
int fpso_token_summaries(const float *coords, const float *feats, int F, int charge_col, const int64_t *offsets,
                         int B, int K, const int32_t *token_id, float *wsum, float *wcoords, float *wfeats)
{
    if (K < 1 || F < 1 || charge_col < -1 || charge_col >= F || bad_offsets(offsets, B)) return -1;
    const int V = 1 + 4 + F;
    double *acc = (double *)malloc(sizeof(double) * (size_t)K * V);
    for (int b = 0; b < B; ++b) {
        for (int64_t e = 0; e < (int64_t)K * V; ++e) acc[e] = 0.0;
        for (int64_t i = offsets[b]; i < offsets[b + 1]; ++i) {
            int32_t j = token_id[i];
            if (j < 0) continue;
            if (j >= K) {
                free(acc);
                return -1;
            }
            double q = charge_col >= 0 ? (double)feats[i * F + charge_col] : 1.0;
            double *a = acc + (int64_t)j * V;
            a[0] += q;
            for (int c = 0; c < 4; ++c) a[1 + c] += q * (double)coords[4 * i + c];
            for (int f = 0; f < F; ++f) a[5 + f] += q * (double)feats[i * F + f];
        }
        for (int j = 0; j < K; ++j) {
            const double *a = acc + (int64_t)j * V;
            int64_t r = (int64_t)b * K + j;
            wsum[r] = (float)a[0];
            for (int c = 0; c < 4; ++c) wcoords[r * 4 + c] = a[0] > 0.0 ? (float)(a[1 + c] / a[0]) : 0.0f;
            for (int f = 0; f < F; ++f) wfeats[r * F + f] = a[0] > 0.0 ? (float)(a[5 + f] / a[0]) : 0.0f;
        }
    }
    free(acc);
    return 0;
}

/*
 * Packed token layout for block-diagonal attention (graphnet PR #923, "What
 * is added": models/utils.py pack / unpack / build_block_mask; the review
 * thread on the block mask: doc_id holds the event index of every packed
 * token and two tokens attend to each other when their doc_ids match).
 * Event b has v_b tokens: valid[b] when given, else min(N_b, K) from the
 * point offsets (the tokens the tokenizer fills).  pack lists the first v_b
 * rows of src [B, K, D] of every event in event order:
 *   tok_offsets[0] = 0, tok_offsets[b+1] = tok_offsets[b] + v_b,
 *   dst[tok_offsets[b] + j, :] = src[b, j, :], doc_id[tok_offsets[b] + j] = b.
 */
int fpso_pack_tokens(const float *src, int D, const int64_t *offsets, const int32_t *valid, int B, int K,
                     float *dst, int32_t *doc_id, int64_t *tok_offsets)
{
    if (D < 1 || K < 1 || B < 0 || (!valid && bad_offsets(offsets, B))) return -1;
    tok_offsets[0] = 0;
    for (int b = 0; b < B; ++b) {
        int64_t v;
        if (valid) {
            v = valid[b];
            if (v < 0 || v > K) return -1;
        } else {
            int64_t n = offsets[b + 1] - offsets[b];
            v = n < K ? n : K;
        }
        for (int64_t j = 0; j < v; ++j) {
            int64_t t = tok_offsets[b] + j;
            doc_id[t] = b;
            for (int d = 0; d < D; ++d) dst[t * D + d] = src[((int64_t)b * K + j) * D + d];
        }
        tok_offsets[b + 1] = tok_offsets[b] + v;
    }
    return 0;
}

/* The inverse: dst[b, j, :] = src[tok_offsets[b] + j, :] for j < v_b, 0 after. */
int fpso_unpack_tokens(const float *src, int D, const int64_t *tok_offsets, int B, int K, float *dst)
{
    if (D < 1 || K < 1 || B < 0 || tok_offsets[0] != 0) return -1;
    for (int b = 0; b < B; ++b) {
        int64_t v = tok_offsets[b + 1] - tok_offsets[b];
        if (v < 0 || v > K) return -1;
        for (int64_t j = 0; j < K; ++j)
            for (int d = 0; d < D; ++d)
                dst[((int64_t)b * K + j) * D + d] = j < v ? src[(tok_offsets[b] + j) * D + d] : 0.0f;
    }
    return 0;
}

/*
 * The whole tokenizer: FPS (or passthrough) -> centroids -> Voronoi labels ->
 * Lloyd (events with N > K) -> Voronoi mean-pool, or kNN gather around the
 * final centroids and kNN mean-pool.  token_id may be NULL in kNN mode;
 * knn_idx is ignored in Voronoi mode; w (per-axis scale) may be NULL.
 */
int fpso_tokenize(const float *coords, const float *feats, int F, const int64_t *offsets, int B,
                  const int32_t *start_local, int K, int assign_mode, int k, int lloyd_iters,
                  int charge_col, const float *w, int32_t *centroid_idx, int32_t *token_id,
                  int32_t *knn_idx, float *centroids, float *pooled, int32_t *counts)
{
    if (K < 1 || F < 1 || (assign_mode != 0 && assign_mode != 1) || lloyd_iters < 0 ||
        charge_col >= F || bad_offsets(offsets, B))
        return -1;
    if (assign_mode == 1 && (k < 1 || knn_idx == NULL)) return -1;
    if (assign_mode == 0 && token_id == NULL) return -1;
    int64_t P = B > 0 ? offsets[B] : 0;
    int rc = fpso_fps(coords, offsets, B, K, start_local, w, centroid_idx, NULL);
    if (rc) return rc;
    for (int64_t r = 0; r < (int64_t)B * K; ++r)
        for (int a = 0; a < 4; ++a)
            centroids[4 * r + a] = centroid_idx[r] >= 0 ? coords[4 * (int64_t)centroid_idx[r] + a] : 0.0f;
    int32_t *lab = (int32_t *)malloc(sizeof(int32_t) * (P > 0 ? P : 1));
    rc = fpso_assign(coords, offsets, B, centroids, NULL, K, w, lab);
    /* passthrough events: token j is point j */
    for (int b = 0; b < B && rc == 0; ++b) {
        int64_t off = offsets[b], n = offsets[b + 1] - off;
        if (n <= K)
            for (int64_t i = 0; i < n; ++i) lab[off + i] = (int32_t)i;
    }
    if (rc == 0 && lloyd_iters > 0)
        rc = fpso_lloyd(coords, feats, F, charge_col, offsets, B, K, lloyd_iters, w, centroids, lab);
    if (rc == 0 && token_id)
        memcpy(token_id, lab, sizeof(int32_t) * (size_t)P);
    if (rc == 0 && assign_mode == 0) {
        rc = fpso_pool_voronoi(feats, F, offsets, B, K, lab, pooled, counts);
    } else if (rc == 0) {
        rc = fpso_knn(coords, offsets, B, centroids, NULL, K, k, w, knn_idx);
        for (int b = 0; b < B && rc == 0; ++b) {
            int64_t off = offsets[b], n = offsets[b + 1] - off;
            if (n > K) continue;
            for (int64_t j = 0; j < n; ++j) {
                int32_t *row = knn_idx + ((int64_t)b * K + j) * k;
                row[0] = (int32_t)(off + j);
                for (int e = 1; e < k; ++e) row[e] = -1;
            }
        }
        if (rc == 0) rc = fpso_pool_knn(feats, F, B, K, k, knn_idx, pooled, counts);
    }
    free(lab);
    return rc;
}
