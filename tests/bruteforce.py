"""Brute-force numpy restatements used to pin the oracle on tiny inputs.

Each routine takes a different route to the same definition than the oracle
does (recomputing from scratch, all-pairs tables, full sorts), so that a slip
in the oracle's loops shows up as a mismatch.  Only tests import this module.
"""
from __future__ import annotations

import numpy as np


def pair_dist(P, C):
    """f32 [n, m] table of squared 4D distances, same operation order, no FMA."""
    P = np.asarray(P, np.float32)
    C = np.asarray(C, np.float32)
    d = [P[:, None, a] - C[None, :, a] for a in range(4)]
    s = d[0] * d[0] + d[1] * d[1]
    s = s + d[2] * d[2]
    s = s + d[3] * d[3]
    return s.astype(np.float32)


def fps_event(pts, K, start=0):
    """Greedy farthest-point recurrence, recomputing each min over the chosen set."""
    n = pts.shape[0]
    if n == 0:
        return np.full(K, -1, np.int64), np.full(K, -1.0, np.float32)
    if n <= K:
        idx = np.full(K, -1, np.int64)
        idx[:n] = np.arange(n)
        return idx, np.full(K, -1.0, np.float32)
    chosen = [start]
    seld = [-1.0]
    D = pair_dist(pts, pts)
    for _ in range(K - 1):
        mind = D[:, chosen].min(axis=1)
        cand = np.ones(n, bool)
        cand[chosen] = False
        vals = np.where(cand, mind, -np.inf)
        best = int(np.argmax(vals))  # first maximum = lowest index
        chosen.append(best)
        seld.append(float(mind[best]))
    return np.array(chosen, np.int64), np.array(seld, np.float32)


def fps(coords, offsets, K, start_local=None):
    B = len(offsets) - 1
    out = np.full((B, K), -1, np.int64)
    for b in range(B):
        o0, o1 = int(offsets[b]), int(offsets[b + 1])
        s = 0 if start_local is None else int(start_local[b])
        idx, _ = fps_event(coords[o0:o1], K, s)
        out[b] = np.where(idx >= 0, idx + o0, -1)
    return out.astype(np.int32)


def assign(coords, offsets, centroids, valid):
    P = coords.shape[0]
    out = np.full(P, -1, np.int32)
    for b in range(len(offsets) - 1):
        o0, o1 = int(offsets[b]), int(offsets[b + 1])
        nv = int(valid[b])
        if o1 == o0 or nv == 0:
            continue
        D = pair_dist(coords[o0:o1], centroids[b, :nv])
        out[o0:o1] = np.argmin(D, axis=1)  # first minimum = lowest slot
    return out


def knn(coords, offsets, centroids, valid, k):
    B, K = centroids.shape[:2]
    out = np.full((B, K, k), -1, np.int32)
    for b in range(B):
        o0, o1 = int(offsets[b]), int(offsets[b + 1])
        n = o1 - o0
        for j in range(int(valid[b])):
            d = pair_dist(coords[o0:o1], centroids[b, j:j + 1])[:, 0]
            order = np.lexsort((np.arange(n), d))  # by d, then index
            m = min(k, n)
            out[b, j, :m] = order[:m] + o0
    return out


def pool_voronoi(feats, offsets, K, token_id):
    B = len(offsets) - 1
    F = feats.shape[1]
    pooled = np.zeros((B, K, F), np.float32)
    counts = np.zeros((B, K), np.int32)
    for b in range(B):
        o0, o1 = int(offsets[b]), int(offsets[b + 1])
        lab = token_id[o0:o1]
        for j in range(K):
            m = lab == j
            counts[b, j] = m.sum()
            if m.any():
                pooled[b, j] = np.mean(feats[o0:o1][m].astype(np.float64), axis=0)
    return pooled, counts


def lloyd_update(pts, q, labels, cents):
    """One centroid update: weighted mean per cell in f64 (numpy's own sums)."""
    new = cents.copy()
    for j in range(cents.shape[0]):
        m = labels == j
        if not m.any():
            continue
        w = q[m].astype(np.float64)
        W = w.sum()
        if W <= 0:
            continue
        new[j] = (np.sum(pts[m].astype(np.float64) * w[:, None], axis=0) / W).astype(np.float32)
    return new
