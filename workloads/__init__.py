"""Seeded synthetic events shaped like the neutrino workloads of the Neptune pages.

This module only draws random inputs; it holds none of the tokenizer's
arithmetic, so both the CPU oracle (``oracle/``) and the CUDA path
(``farthest_point_sampling_b200``) can be fed from it without sharing code.

The pages ("Add Neptune point-transformer backbone", graphnet PR #923, Summary;
Neptune README, Usage) describe an event as a variable-length 4D point cloud
``coords[N, 4] = (x, y, z, t)`` plus ``features[N, F]`` with F = 6 and a
per-point event id.  Here every batch is packed: events are contiguous and
``offsets[b]..offsets[b+1]`` spans event b.

The detector is a synthetic stand-in (not a real geometry file): 86 strings on
a triangular lattice with 125 m spacing (the 86 lattice sites nearest the
origin), 60 DOMs per string at a 17 m pitch, z in [-501.5, +501.5] m.
Times are in ns, unscaled; light travels at 0.3 m/ns.

Workloads (all seeded with ``numpy.random.default_rng(seed)``):

* ``c0`` tiny correctness batch: B=4, N={37,200,512,1000}, x,y,z ~ N(0,100 m),
  t ~ U(0,5000 ns); features N(0,1) with column 0 ~ lognormal(0,1); K=16.
* ``c1`` 64 track-like events: N ~ round(lognormal(ln 300, 1)) clipped to
  [8, 20000]; pulses on DOMs near a straight track; K=128, Voronoi.
* ``c2`` the ``c1`` generator at B=256, kNN with k=32, K=128.
* ``c3`` 8 bright showers: N ~ U(50000, 200000) pulses on the DOMs within 300 m
  of a vertex; K=128, Voronoi, 3 charge-weighted Lloyd iterations.
* ``c4`` 4096 small events: N ~ U{5..400}, pulses on DOMs drawn uniformly from
  the whole array; K=128 (also swept at 32/64/256).
"""
from __future__ import annotations

import dataclasses
from typing import Dict, Optional

import numpy as np

__all__ = [
    "Batch",
    "detector_doms",
    "make_workload",
    "random_batch",
    "WORKLOADS",
]

N_FEATURES = 6
C_LIGHT_M_PER_NS = 0.3
STRING_SPACING_M = 125.0
N_STRINGS = 86
DOMS_PER_STRING = 60
DOM_PITCH_M = 17.0


@dataclasses.dataclass
class Batch:
    """A packed batch of events plus the tokenizer settings it is run with."""

    coords: np.ndarray  # f32 [P, 4] (x, y, z, t)
    feats: np.ndarray  # f32 [P, F]
    offsets: np.ndarray  # i64 [B + 1]
    K: int
    assign_mode: int = 0  # 0 = Voronoi, 1 = kNN
    k: int = 0
    lloyd_iters: int = 0
    charge_col: int = -1
    start_local: Optional[np.ndarray] = None  # i32 [B] or None (= 0)
    name: str = ""
    axis_scale: Optional[tuple] = None  # (wx, wy, wz, wt) of the distance, or None (unscaled)

    @property
    def B(self) -> int:
        return int(self.offsets.shape[0] - 1)

    @property
    def P(self) -> int:
        return int(self.coords.shape[0])

    @property
    def F(self) -> int:
        return int(self.feats.shape[1])

    def sizes(self) -> np.ndarray:
        return np.diff(self.offsets)


def detector_doms() -> np.ndarray:
    """DOM positions f64 [86*60, 3] of the synthetic string array."""
    # Triangular lattice: a*(1,0) + b*(1/2, sqrt(3)/2), spacing 125 m.
    r = 12
    sites = []
    for a in range(-r, r + 1):
        for b in range(-r, r + 1):
            x = STRING_SPACING_M * (a + 0.5 * b)
            y = STRING_SPACING_M * (np.sqrt(3.0) / 2.0) * b
            sites.append((x * x + y * y, a, b, x, y))
    sites.sort()
    xy = np.array([[s[3], s[4]] for s in sites[:N_STRINGS]], dtype=np.float64)
    z = -501.5 + DOM_PITCH_M * np.arange(DOMS_PER_STRING, dtype=np.float64)
    doms = np.empty((N_STRINGS * DOMS_PER_STRING, 3), dtype=np.float64)
    doms[:, 0] = np.repeat(xy[:, 0], DOMS_PER_STRING)
    doms[:, 1] = np.repeat(xy[:, 1], DOMS_PER_STRING)
    doms[:, 2] = np.tile(z, N_STRINGS)
    return doms


def _features(rng: np.random.Generator, n: int) -> np.ndarray:
    f = rng.standard_normal((n, N_FEATURES))
    f[:, 0] = rng.lognormal(0.0, 1.0, n)  # charge
    return f.astype(np.float32)


def _pack(chunks_c, chunks_f, K, name, **kw) -> Batch:
    sizes = np.array([c.shape[0] for c in chunks_c], dtype=np.int64)
    offsets = np.zeros(len(sizes) + 1, dtype=np.int64)
    np.cumsum(sizes, out=offsets[1:])
    if len(chunks_c):
        coords = np.ascontiguousarray(np.concatenate(chunks_c).astype(np.float32))
        feats = np.ascontiguousarray(np.concatenate(chunks_f).astype(np.float32))
    else:
        coords = np.zeros((0, 4), np.float32)
        feats = np.zeros((0, N_FEATURES), np.float32)
    return Batch(coords, feats, offsets, K, name=name, **kw)


def _detector_bounds(doms):
    rmax = np.sqrt((doms[:, :2] ** 2).sum(1)).max()
    return rmax, doms[:, 2].min(), doms[:, 2].max()


def _random_vertex(rng, doms):
    rmax, zmin, zmax = _detector_bounds(doms)
    while True:
        x, y = rng.uniform(-rmax, rmax, 2)
        if x * x + y * y <= rmax * rmax:
            return np.array([x, y, rng.uniform(zmin, zmax)])


def _track_event(rng, doms, n):
    """Pulses on DOMs near a straight track through a random vertex."""
    while True:
        v = _random_vertex(rng, doms)
        u = rng.standard_normal(3)
        u /= np.linalg.norm(u)
        rel = doms - v
        along = rel @ u
        perp = np.sqrt(np.maximum((rel * rel).sum(1) - along * along, 0.0))
        near = np.nonzero(perp < 150.0)[0]
        if near.size:
            break
    w = np.exp(-perp[near] / 50.0)
    pick = near[rng.choice(near.size, size=n, p=w / w.sum())]
    pos = doms[pick]
    t = np.linalg.norm(pos - v, axis=1) / C_LIGHT_M_PER_NS + rng.exponential(50.0, n)
    return np.column_stack([pos, t])


def _shower_event(rng, doms, n):
    """Pulses spread uniformly over the DOMs within 300 m of a vertex."""
    while True:
        v = _random_vertex(rng, doms)
        near = np.nonzero(np.linalg.norm(doms - v, axis=1) < 300.0)[0]
        if near.size:
            break
    pos = doms[near[rng.integers(0, near.size, n)]]
    t = np.linalg.norm(pos - v, axis=1) / C_LIGHT_M_PER_NS + rng.exponential(50.0, n)
    return np.column_stack([pos, t])


def _uniform_event(rng, doms, n):
    """Pulses on DOMs drawn uniformly from the whole array."""
    v = _random_vertex(rng, doms)
    pos = doms[rng.integers(0, doms.shape[0], n)]
    t = np.linalg.norm(pos - v, axis=1) / C_LIGHT_M_PER_NS + rng.exponential(50.0, n)
    return np.column_stack([pos, t])


def _c0(seed=0):
    rng = np.random.default_rng(seed)
    cs, fs = [], []
    for n in (37, 200, 512, 1000):
        c = np.empty((n, 4))
        c[:, :3] = rng.normal(0.0, 100.0, (n, 3))
        c[:, 3] = rng.uniform(0.0, 5000.0, n)
        cs.append(c)
        fs.append(_features(rng, n))
    return _pack(cs, fs, 16, "c0: 4 events N={37,200,512,1000}, K=16, voronoi")


def _track_sizes(rng, B):
    n = np.rint(rng.lognormal(np.log(300.0), 1.0, B))
    return np.clip(n, 8, 20000).astype(np.int64)


def _c1(seed=1, B=64):
    rng = np.random.default_rng(seed)
    doms = detector_doms()
    cs, fs = [], []
    for n in _track_sizes(rng, B):
        cs.append(_track_event(rng, doms, int(n)))
        fs.append(_features(rng, int(n)))
    return _pack(cs, fs, 128, f"c1: {B} track events, lognormal N, K=128, voronoi")


def _c2(seed=2, B=256):
    b = _c1(seed, B)
    b.assign_mode, b.k = 1, 32
    b.name = f"c2: {B} track events, lognormal N, K=128, knn k=32"
    return b


def _c3(seed=3, B=8):
    rng = np.random.default_rng(seed)
    doms = detector_doms()
    cs, fs = [], []
    for _ in range(B):
        n = int(rng.integers(50000, 200001))
        cs.append(_shower_event(rng, doms, n))
        fs.append(_features(rng, n))
    return _pack(cs, fs, 128, f"c3: {B} shower events N~U(5e4,2e5), K=128, voronoi, lloyd x3",
                 lloyd_iters=3, charge_col=0)


def _c4(seed=4, B=4096, K=128):
    rng = np.random.default_rng(seed)
    doms = detector_doms()
    cs, fs = [], []
    for n in rng.integers(5, 401, B):
        cs.append(_uniform_event(rng, doms, int(n)))
        fs.append(_features(rng, int(n)))
    return _pack(cs, fs, K, f"c4: {B} small events N~U(5,400), K={K}, voronoi")


WORKLOADS: Dict[str, object] = {"c0": _c0, "c1": _c1, "c2": _c2, "c3": _c3, "c4": _c4}


def make_workload(name: str, **kw) -> Batch:
    """Build one of the named workloads (``c0``..``c4``); kwargs override B/seed/K."""
    return WORKLOADS[name](**kw)


def random_batch(seed: int, sizes, K: int, *, F: int = N_FEATURES, scale=(100.0, 100.0, 100.0, 1000.0),
                 dup_frac: float = 0.0, grid: Optional[float] = None, assign_mode: int = 0, k: int = 0,
                 lloyd_iters: int = 0, charge_col: int = -1, start_local=None) -> Batch:
    """Small random batch for parity tests.

    ``dup_frac`` replaces that fraction of points by copies of other points of
    the same event (exact duplicates, to exercise ties); ``grid`` snaps every
    coordinate to multiples of ``grid`` (more exact ties).
    """
    rng = np.random.default_rng(seed)
    cs, fs = [], []
    for n in sizes:
        n = int(n)
        c = rng.standard_normal((n, 4)) * np.asarray(scale)
        if grid is not None:
            c = np.round(c / grid) * grid
        if dup_frac > 0 and n > 1:
            m = int(dup_frac * n)
            dst = rng.integers(0, n, m)
            src = rng.integers(0, n, m)
            c[dst] = c[src]
        cs.append(c)
        f = rng.standard_normal((n, F))
        if F > 0:
            f[:, 0] = rng.lognormal(0.0, 1.0, n)
        fs.append(f.astype(np.float32))
    b = _pack(cs, fs, K, f"random seed={seed}", assign_mode=assign_mode, k=k,
              lloyd_iters=lloyd_iters, charge_col=charge_col)
    if F != N_FEATURES:
        b.feats = np.ascontiguousarray(
            np.concatenate(fs).astype(np.float32) if len(fs) else np.zeros((0, F), np.float32))
    if start_local is not None:
        b.start_local = np.asarray(start_local, dtype=np.int32)
    return b
