"""Python access to the plain C oracle (``fps_oracle.c``).

TEST INFRASTRUCTURE ONLY: tests/, ``__graft_entry__.smoke()`` and bench.py's
CPU-baseline / reference legs may import this package; the CUDA library and
its binding never do.  The oracle is built with gcc, ``-O2 -ffp-contract=off``
and no fast-math, so every float32 operation is rounded on its own.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "fps_oracle.c")
_LIB = os.path.join(_HERE, "libfps_oracle.so")
CFLAGS = ["-O2", "-std=c11", "-ffp-contract=off", "-fno-fast-math", "-fexcess-precision=standard",
          "-fPIC", "-shared"]

_lib = None


def build(force: bool = False) -> str:
    """Compile the oracle shared library next to its source; return its path."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", *CFLAGS, _SRC, "-o", tmp, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


def bind(path: str):
    """Load an oracle shared library at ``path`` and declare its signatures."""
    lib = ctypes.CDLL(path)
    P = ctypes.c_void_p
    I = ctypes.c_int
    lib.fpso_dist.restype = ctypes.c_float
    lib.fpso_dist.argtypes = [P, P]
    lib.fpso_dist_w.restype = ctypes.c_float
    lib.fpso_dist_w.argtypes = [P, P, P]
    lib.fpso_fps.argtypes = [P, P, I, I, P, P, P, P]
    lib.fpso_assign.argtypes = [P, P, I, P, P, I, P, P]
    lib.fpso_knn.argtypes = [P, P, I, P, P, I, I, P, P]
    lib.fpso_lloyd.argtypes = [P, P, I, I, P, I, I, I, P, P, P]
    lib.fpso_pool_voronoi.argtypes = [P, I, P, I, I, P, P, P]
    lib.fpso_pool_knn.argtypes = [P, I, I, I, I, P, P, P]
    lib.fpso_tokenize.argtypes = [P, P, I, P, I, P, I, I, I, I, I, P, P, P, P, P, P, P]
    lib.fpso_pool_voronoi_backward.argtypes = [P, I, P, I, I, P, P, P]
    lib.fpso_pool_knn_backward.argtypes = [P, I, I, I, I, P, P, ctypes.c_int64, P]
    lib.fpso_pack_tokens.argtypes = [P, I, P, P, I, I, P, P, P]
    lib.fpso_token_summaries.argtypes = [P, P, I, I, P, I, I, P, P, P, P]
    lib.fpso_philox4x32_10.argtypes = [P, P, P]
    lib.fpso_philox4x32_10.restype = None
    lib.fpso_random_starts.argtypes = [P, I, ctypes.c_uint64, ctypes.c_uint32, P]
    lib.fpso_unpack_tokens.argtypes = [P, I, P, I, I, P]
    for f in (lib.fpso_fps, lib.fpso_assign, lib.fpso_knn, lib.fpso_lloyd,
              lib.fpso_pool_voronoi, lib.fpso_pool_knn, lib.fpso_tokenize,
              lib.fpso_pool_voronoi_backward, lib.fpso_pool_knn_backward, lib.fpso_pack_tokens,
              lib.fpso_unpack_tokens, lib.fpso_token_summaries, lib.fpso_random_starts):
        f.restype = I
    return lib


def _load():
    global _lib
    if _lib is None:
        _lib = bind(build())
    return _lib


class use_library:
    """Context manager: route the wrappers below through another oracle build
    (the mutation tests compile altered copies of the oracle to check that the
    pins catch them)."""

    def __init__(self, path: str):
        self.path = path

    def __enter__(self):
        global _lib
        self._saved = _lib
        _lib = bind(self.path)
        return self

    def __exit__(self, *exc):
        global _lib
        _lib = self._saved
        return False


def _f32(a, shape_tail=None):
    a = np.ascontiguousarray(a, dtype=np.float32)
    if shape_tail is not None:
        a = a.reshape((-1,) + tuple(shape_tail))
    return a


def _i64(a):
    return np.ascontiguousarray(a, dtype=np.int64)


def _i32(a):
    return None if a is None else np.ascontiguousarray(a, dtype=np.int32)


def _p(a):
    return None if a is None else a.ctypes.data


def _check(rc, what):
    if rc != 0:
        raise ValueError(f"oracle {what}: invalid arguments")


def dist(p, c) -> np.float32:
    """The float32 squared 4D distance the oracle uses."""
    p = _f32(p).reshape(4)
    c = _f32(c).reshape(4)
    return np.float32(_load().fpso_dist(_p(p), _p(c)))


def _w(axis_scale):
    """Per-axis scale as a float32 [4] array, or None (no scaling)."""
    return None if axis_scale is None else _f32(axis_scale).reshape(4)


def dist_w(p, c, axis_scale) -> np.float32:
    """The distance under a per-axis scale (both points scaled in float32 first)."""
    p = _f32(p).reshape(4)
    c = _f32(c).reshape(4)
    w = _w(axis_scale)
    return np.float32(_load().fpso_dist_w(_p(p), _p(c), _p(w)))


def fps(coords, offsets, K: int, start_local=None, with_sel_dist: bool = False, axis_scale=None):
    coords, offsets = _f32(coords, (4,)), _i64(offsets)
    B = offsets.shape[0] - 1
    start_local = _i32(start_local)
    w = _w(axis_scale)
    idx = np.empty((B, K), np.int32)
    sd = np.empty((B, K), np.float32) if with_sel_dist else None
    _check(_load().fpso_fps(_p(coords), _p(offsets), B, K, _p(start_local), _p(w), _p(idx), _p(sd)), "fps")
    return (idx, sd) if with_sel_dist else idx


def assign(coords, offsets, centroids, K: int, valid=None, axis_scale=None):
    coords, offsets = _f32(coords, (4,)), _i64(offsets)
    B = offsets.shape[0] - 1
    centroids = _f32(centroids).reshape(B, K, 4)
    w = _w(axis_scale)
    tok = np.empty(coords.shape[0], np.int32)
    _check(_load().fpso_assign(_p(coords), _p(offsets), B, _p(centroids), _p(_i32(valid)), K, _p(w), _p(tok)),
           "assign")
    return tok


def knn(coords, offsets, centroids, K: int, k: int, valid=None, axis_scale=None):
    coords, offsets = _f32(coords, (4,)), _i64(offsets)
    B = offsets.shape[0] - 1
    centroids = _f32(centroids).reshape(B, K, 4)
    w = _w(axis_scale)
    out = np.empty((B, K, k), np.int32)
    _check(_load().fpso_knn(_p(coords), _p(offsets), B, _p(centroids), _p(_i32(valid)), K, k, _p(w), _p(out)),
           "knn")
    return out


def lloyd(coords, feats, offsets, K: int, iters: int, centroids, token_id, charge_col: int = -1,
          axis_scale=None):
    coords, offsets = _f32(coords, (4,)), _i64(offsets)
    B = offsets.shape[0] - 1
    feats = _f32(feats)
    F = feats.shape[1] if feats.ndim == 2 else 0
    c = _f32(centroids).reshape(B, K, 4).copy()
    t = _i32(token_id).copy()
    w = _w(axis_scale)
    _check(_load().fpso_lloyd(_p(coords), _p(feats), F, charge_col, _p(offsets), B, K, iters, _p(w), _p(c),
                              _p(t)), "lloyd")
    return c, t


def pool_voronoi(feats, offsets, K: int, token_id):
    feats, offsets = _f32(feats), _i64(offsets)
    B = offsets.shape[0] - 1
    F = feats.shape[1]
    pooled = np.empty((B, K, F), np.float32)
    counts = np.empty((B, K), np.int32)
    _check(_load().fpso_pool_voronoi(_p(feats), F, _p(offsets), B, K, _p(_i32(token_id)), _p(pooled),
                                     _p(counts)), "pool_voronoi")
    return pooled, counts


def pool_knn(feats, knn_idx):
    feats = _f32(feats)
    knn_idx = _i32(knn_idx)
    B, K, k = knn_idx.shape
    F = feats.shape[1]
    pooled = np.empty((B, K, F), np.float32)
    counts = np.empty((B, K), np.int32)
    _check(_load().fpso_pool_knn(_p(feats), F, B, K, k, _p(knn_idx), _p(pooled), _p(counts)), "pool_knn")
    return pooled, counts


def pool_voronoi_backward(grad_pooled, offsets, token_id, counts):
    """Gradient of ``pool_voronoi`` with respect to the features, given the
    gradient of the pooled rows [B, K, F] and the forward's counts [B, K]."""
    grad_pooled, offsets = _f32(grad_pooled), _i64(offsets)
    B, K, F = grad_pooled.shape
    token_id = _i32(token_id)
    out = np.empty((token_id.shape[0], F), np.float32)
    _check(_load().fpso_pool_voronoi_backward(_p(grad_pooled), F, _p(offsets), B, K, _p(token_id),
                                              _p(_i32(counts)), _p(out)), "pool_voronoi_backward")
    return out


def pool_knn_backward(grad_pooled, knn_idx, counts, P: int):
    """Gradient of ``pool_knn`` with respect to the [P, F] features."""
    grad_pooled, knn_idx = _f32(grad_pooled), _i32(knn_idx)
    B, K, F = grad_pooled.shape
    k = knn_idx.shape[2]
    out = np.empty((P, F), np.float32)
    _check(_load().fpso_pool_knn_backward(_p(grad_pooled), F, B, K, k, _p(knn_idx), _p(_i32(counts)), P,
                                          _p(out)), "pool_knn_backward")
    return out


def philox4x32_10(counter, key):
    """One Philox4x32-10 block: four 32-bit words for a 4-word counter and a
    2-word key."""
    c = np.ascontiguousarray(counter, dtype=np.uint32)
    k = np.ascontiguousarray(key, dtype=np.uint32)
    out = np.empty(4, np.uint32)
    _load().fpso_philox4x32_10(_p(c), _p(k), _p(out))
    return out


def random_starts(offsets, seed: int, stream: int = 0):
    """Random local FPS start index per event from Philox4x32-10."""
    offsets = _i64(offsets)
    B = offsets.shape[0] - 1
    out = np.empty(B, np.int32)
    _check(_load().fpso_random_starts(_p(offsets), B, seed, stream, _p(out)), "random_starts")
    return out


def token_summaries(coords, feats, offsets, K: int, token_id, charge_col: int = -1):
    """Charge-weighted summaries per Voronoi token: ``(wsum [B,K], wcoords
    [B,K,4], wfeats [B,K,F])``."""
    coords, feats, offsets = _f32(coords, (4,)), _f32(feats), _i64(offsets)
    B, F = offsets.shape[0] - 1, feats.shape[1]
    wsum = np.empty((B, K), np.float32)
    wc = np.empty((B, K, 4), np.float32)
    wf = np.empty((B, K, F), np.float32)
    _check(_load().fpso_token_summaries(_p(coords), _p(feats), F, charge_col, _p(offsets), B, K,
                                        _p(_i32(token_id)), _p(wsum), _p(wc), _p(wf)), "token_summaries")
    return wsum, wc, wf


def pack_tokens(src, offsets=None, valid=None):
    """Packed layout of padded tokens ``src [B, K, D]``: returns
    ``(dst [N_tok, D], doc_id [N_tok], tok_offsets [B + 1])``."""
    src = _f32(src)
    B, K, D = src.shape
    if valid is None:
        offsets = _i64(offsets)
        n_tok = int(np.minimum(np.diff(offsets), K).sum()) if B else 0
    else:
        valid = _i32(valid)
        n_tok = int(valid.astype(np.int64).sum())
    dst = np.empty((max(n_tok, 1), D), np.float32)
    doc = np.empty(max(n_tok, 1), np.int32)
    tok = np.empty(B + 1, np.int64)
    _check(_load().fpso_pack_tokens(_p(src), D, _p(offsets) if valid is None else None, _p(valid), B, K,
                                    _p(dst), _p(doc), _p(tok)), "pack_tokens")
    return dst[:n_tok], doc[:n_tok], tok


def unpack_tokens(src, tok_offsets, K: int):
    """Padded layout [B, K, D] of packed tokens ``src [N_tok, D]``."""
    src, tok_offsets = _f32(src), _i64(tok_offsets)
    B = tok_offsets.shape[0] - 1
    D = src.shape[1]
    dst = np.empty((B, K, D), np.float32)
    _check(_load().fpso_unpack_tokens(_p(src), D, _p(tok_offsets), B, K, _p(dst)), "unpack_tokens")
    return dst


def tokenize(coords, feats, offsets, K: int, assign_mode: int = 0, k: int = 0, lloyd_iters: int = 0,
             charge_col: int = -1, start_local=None, axis_scale=None) -> dict:
    """The whole tokenizer on one packed batch; returns a dict of numpy outputs.
    ``axis_scale``: optional per-axis scale (wx, wy, wz, wt) of the distance."""
    coords, feats, offsets = _f32(coords, (4,)), _f32(feats), _i64(offsets)
    B = offsets.shape[0] - 1
    P = coords.shape[0]
    F = feats.shape[1]
    out = {
        "centroid_idx": np.empty((B, K), np.int32),
        "token_id": np.empty(P, np.int32),
        "knn_idx": np.empty((B, K, max(k, 1)), np.int32) if assign_mode == 1 else None,
        "centroids": np.empty((B, K, 4), np.float32),
        "pooled": np.empty((B, K, F), np.float32),
        "counts": np.empty((B, K), np.int32),
    }
    w = _w(axis_scale)
    rc = _load().fpso_tokenize(_p(coords), _p(feats), F, _p(offsets), B, _p(_i32(start_local)), K,
                               assign_mode, k, lloyd_iters, charge_col, _p(w), _p(out["centroid_idx"]),
                               _p(out["token_id"]), _p(out["knn_idx"]), _p(out["centroids"]),
                               _p(out["pooled"]), _p(out["counts"]))
    _check(rc, "tokenize")
    return out


def tokenize_batch(batch) -> dict:
    """``tokenize`` on a ``workloads.Batch``."""
    return tokenize(batch.coords, batch.feats, batch.offsets, batch.K, batch.assign_mode, batch.k,
                    batch.lloyd_iters, batch.charge_col, batch.start_local, getattr(batch, "axis_scale", None))
