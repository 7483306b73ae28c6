"""PyTorch-facing binding of the fpstok C ABI (argument marshalling only).

Every function checks dtypes, shapes and devices, allocates outputs and the
workspace with PyTorch, and calls the matching C entry point of libfpstok.so
on the current CUDA stream.  All computation happens in the CUDA kernels.

Inputs are float32 only, as on the pages (graphnet PR #923 "Add Neptune
point-transformer backbone", review thread on the FPS `precision` argument:
both backends always compute in float32, no silent dtype change); any other
dtype raises ``TypeError``.  Events are packed: ``coords[P, 4]`` with
``(x, y, z, t)`` per point (Neptune README, Usage), ``feats[P, F]`` and
``offsets[B + 1]`` (int64) delimiting each event, or per-point ``batch_ids``
converted by :func:`offsets_from_batch_ids`.
"""
from __future__ import annotations

import ctypes
from typing import Dict, Optional, Union

import torch

from . import _lib

_MODES = {"voronoi": _lib.FPS_ASSIGN_VORONOI, "knn": _lib.FPS_ASSIGN_KNN, 0: 0, 1: 1}


def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(device: torch.device) -> ctypes.c_void_p:
    return ctypes.c_void_p(torch.cuda.current_stream(device).cuda_stream)


def _need(t: torch.Tensor, name: str, dtype: torch.dtype, ndim: int, device: Optional[torch.device] = None):
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype} (no implicit conversion)")
    if t.dim() != ndim:
        raise ValueError(f"{name} must have {ndim} dimensions, got shape {tuple(t.shape)}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if device is not None and t.device != device:
        raise ValueError(f"{name} must be on {device}, got {t.device}")


def _cuda_device(t: torch.Tensor) -> torch.device:
    if t.device.type != "cuda":
        raise ValueError("the fpstok path runs on CUDA tensors only (there is no CPU fallback)")
    return t.device


def _workspace(nbytes: int, device: torch.device, workspace: Optional[torch.Tensor]) -> torch.Tensor:
    if workspace is not None:
        if workspace.numel() * workspace.element_size() < nbytes:
            raise ValueError(f"workspace too small: need {nbytes} bytes")
        return workspace
    return torch.empty(max(int(nbytes), 256), dtype=torch.uint8, device=device)


def offsets_from_batch_ids(batch_ids: torch.Tensor, num_events: Optional[int] = None) -> torch.Tensor:
    """int64 offsets [B+1] from sorted per-point event ids (Neptune README, Usage).

    Rejects unsorted ids (events must be contiguous).  On CUDA tensors the
    sortedness check and an unspecified ``num_events`` each read one value
    back from the device.
    """
    _need(batch_ids, "batch_ids", torch.int64, 1)
    if batch_ids.numel() > 1 and bool((batch_ids[1:] < batch_ids[:-1]).any()):
        raise ValueError("batch_ids must be sorted so that every event is contiguous")
    if num_events is None:
        num_events = int(batch_ids.max().item()) + 1 if batch_ids.numel() else 0
    counts = torch.bincount(batch_ids, minlength=num_events)
    off = torch.zeros(num_events + 1, dtype=torch.int64, device=batch_ids.device)
    torch.cumsum(counts, 0, out=off[1:])
    return off


def _axis_scale(axis_scale) -> Optional[ctypes.Array]:
    """Host array of the 4 per-axis weights (x, y, z, t) of the distance, or None."""
    if axis_scale is None:
        return None
    w = [float(v) for v in axis_scale]
    if len(w) != 4:
        raise ValueError("axis_scale must hold 4 weights (x, y, z, t)")
    return (ctypes.c_float * 4)(*w)


class Options:
    """Python view of ``fps_opts``.  ``axis_scale``: optional per-axis weights
    (wx, wy, wz, wt) of the FPS / assignment distance (both points' coordinates
    are multiplied by them in float32 first); None means unscaled."""

    def __init__(self, K: int = 128, assign_mode: Union[str, int] = "voronoi", k: int = 32,
                 lloyd_iters: int = 0, charge_col: int = -1, force_schedule: int = -1,
                 max_event_hint: int = 0, axis_scale=None):
        if assign_mode not in _MODES:
            raise ValueError(f"assign_mode must be 'voronoi' or 'knn', got {assign_mode!r}")
        w = _axis_scale(axis_scale)
        self.c = _lib.FpsOpts(int(K), _MODES[assign_mode], int(k), int(lloyd_iters), int(charge_col),
                              int(force_schedule), int(max_event_hint), w if w is not None else (ctypes.c_float * 4)())

    @property
    def knn(self) -> bool:
        return self.c.assign_mode == _lib.FPS_ASSIGN_KNN


def _prep_offsets(offsets: torch.Tensor, device: torch.device, hint: int):
    """Offsets on the device; the largest event size when they came from the host."""
    _need(offsets, "offsets", torch.int64, 1)
    if offsets.device.type == "cpu":
        if hint == 0 and offsets.numel() > 1:
            hint = int((offsets[1:] - offsets[:-1]).max())
        offsets = offsets.to(device, non_blocking=True)
    elif offsets.device != device:
        raise ValueError("offsets must be on the same device as coords (or on the host)")
    return offsets, hint


def fps_tokenize(coords: torch.Tensor, feats: torch.Tensor, offsets: torch.Tensor, K: int = 128,
                 assign_mode: Union[str, int] = "voronoi", k: int = 32, lloyd_iters: int = 0,
                 charge_col: int = -1, start_local: Optional[torch.Tensor] = None,
                 force_schedule: int = -1, max_event_hint: int = 0,
                 workspace: Optional[torch.Tensor] = None, out: Optional[Dict[str, torch.Tensor]] = None,
                 check_device: bool = False, random_start: bool = False, seed: int = 0,
                 stream_id: int = 0, axis_scale=None) -> Dict[str, torch.Tensor]:
    """The whole tokenizer (C ``fps_tokenize``): FPS fused with Voronoi labels,
    optional charge-weighted Lloyd, then Voronoi mean-pool or kNN gather + pool.

    Returns ``centroid_idx [B,K]``, ``token_id [P]`` (Voronoi labels; also in
    kNN mode), ``knn_idx [B,K,k]`` (kNN mode), ``centroids [B,K,4]``,
    ``pooled [B,K,F]`` and ``counts [B,K]``.  ``offsets`` may live on the host,
    in which case the largest event size is passed to the library as a
    scheduling hint.  ``check_device=True`` synchronises and raises on a
    device-side check failure (bad offsets or start index).  With
    ``random_start`` each event starts at a Philox4x32-10 draw for ``seed``
    and ``stream_id`` (see :func:`random_starts`) instead of ``start_local``.
    ``axis_scale`` = (wx, wy, wz, wt) weights the coordinates in the distance
    (e.g. a time scale); positions and means are returned in input units.
    """
    dev = _cuda_device(coords)
    _need(coords, "coords", torch.float32, 2, dev)
    _need(feats, "feats", torch.float32, 2, dev)
    if coords.shape[1] != 4:
        raise ValueError("coords must be [P, 4] (x, y, z, t)")
    if feats.shape[0] != coords.shape[0]:
        raise ValueError("feats and coords must have the same number of rows")
    offsets, hint = _prep_offsets(offsets, dev, max_event_hint)
    if random_start:
        if start_local is not None:
            raise ValueError("give start_local or random_start, not both")
        start_local = random_starts(offsets, seed, stream_id)
    if start_local is not None:
        _need(start_local, "start_local", torch.int32, 1, dev)
    opts = Options(K, assign_mode, k, lloyd_iters, charge_col, force_schedule, hint, axis_scale)
    P, F = coords.shape[0], feats.shape[1]
    B = offsets.numel() - 1
    lib = _lib.load()
    ws_bytes = lib.fps_workspace_bytes(P, B, F, ctypes.byref(opts.c))
    ws = _workspace(ws_bytes, dev, workspace)
    o = out if out is not None else {}
    o.setdefault("centroid_idx", torch.empty((B, K), dtype=torch.int32, device=dev))
    o.setdefault("token_id", torch.empty(P, dtype=torch.int32, device=dev))
    if opts.knn:
        o.setdefault("knn_idx", torch.empty((B, K, k), dtype=torch.int32, device=dev))
    o.setdefault("centroids", torch.empty((B, K, 4), dtype=torch.float32, device=dev))
    o.setdefault("pooled", torch.empty((B, K, F), dtype=torch.float32, device=dev))
    o.setdefault("counts", torch.empty((B, K), dtype=torch.int32, device=dev))
    st = lib.fps_tokenize(_ptr(coords), _ptr(feats), F, _ptr(offsets), B, P, _ptr(start_local),
                          ctypes.byref(opts.c), _ptr(o["centroid_idx"]), _ptr(o["token_id"]),
                          _ptr(o.get("knn_idx")), _ptr(o["centroids"]), _ptr(o["pooled"]),
                          _ptr(o["counts"]), _ptr(ws), ws.numel(), _stream(dev))
    _lib.check(st, "fps_tokenize")
    if check_device:
        device_status(ws)
    return o


def fps_tokenize_host(coords: torch.Tensor, feats: torch.Tensor, offsets: torch.Tensor, K: int = 128,
                      assign_mode: Union[str, int] = "voronoi", k: int = 32, lloyd_iters: int = 0,
                      charge_col: int = -1, start_local: Optional[torch.Tensor] = None,
                      force_schedule: int = -1, device: Union[str, torch.device] = "cuda",
                      workspace: Optional[torch.Tensor] = None,
                      out: Optional[Dict[str, torch.Tensor]] = None, synchronize: bool = True,
                      axis_scale=None) -> Dict[str, torch.Tensor]:
    """C ``fps_tokenize_host``: host (ideally pinned) inputs and outputs; the
    library stages them through the device workspace on the current stream.
    With ``synchronize`` the results are ready on return."""
    dev = torch.device(device)
    _need(coords, "coords", torch.float32, 2, torch.device("cpu"))
    _need(feats, "feats", torch.float32, 2, torch.device("cpu"))
    _need(offsets, "offsets", torch.int64, 1, torch.device("cpu"))
    if start_local is not None:
        _need(start_local, "start_local", torch.int32, 1, torch.device("cpu"))
    P, F = coords.shape[0], feats.shape[1]
    B = offsets.numel() - 1
    hint = int((offsets[1:] - offsets[:-1]).max()) if B > 0 else 0
    if coords.is_pinned():  # small inputs too: a pageable copy would hold up the overlap of the slices
        if not offsets.is_pinned():
            offsets = offsets.pin_memory()
        if start_local is not None and not start_local.is_pinned():
            start_local = start_local.pin_memory()
    opts = Options(K, assign_mode, k, lloyd_iters, charge_col, force_schedule, hint, axis_scale)
    lib = _lib.load()
    ws = _workspace(lib.fps_host_workspace_bytes(P, B, F, ctypes.byref(opts.c)), dev, workspace)
    pin = coords.is_pinned()
    o = out if out is not None else {}
    o.setdefault("centroid_idx", torch.empty((B, K), dtype=torch.int32, pin_memory=pin))
    o.setdefault("token_id", torch.empty(P, dtype=torch.int32, pin_memory=pin))
    if opts.knn:
        o.setdefault("knn_idx", torch.empty((B, K, k), dtype=torch.int32, pin_memory=pin))
    o.setdefault("centroids", torch.empty((B, K, 4), dtype=torch.float32, pin_memory=pin))
    o.setdefault("pooled", torch.empty((B, K, F), dtype=torch.float32, pin_memory=pin))
    o.setdefault("counts", torch.empty((B, K), dtype=torch.int32, pin_memory=pin))
    stream = _stream(dev)
    st = lib.fps_tokenize_host(_ptr(coords), _ptr(feats), F, _ptr(offsets), B, P, _ptr(start_local),
                               ctypes.byref(opts.c), _ptr(o["centroid_idx"]), _ptr(o["token_id"]),
                               _ptr(o.get("knn_idx")), _ptr(o["centroids"]), _ptr(o["pooled"]),
                               _ptr(o["counts"]), _ptr(ws), ws.numel(), stream)
    _lib.check(st, "fps_tokenize_host")
    if synchronize:
        torch.cuda.current_stream(dev).synchronize()
    return o


def fps_assign(coords: torch.Tensor, offsets: torch.Tensor, centroids: torch.Tensor,
               valid_tokens: Optional[torch.Tensor] = None, workspace: Optional[torch.Tensor] = None,
               out: Optional[torch.Tensor] = None, axis_scale=None) -> torch.Tensor:
    """C ``fps_assign`` (components/fps.py nearest_assign): nearest centroid
    slot of every point, lowest slot on ties; centroids [B, K, 4]."""
    dev = _cuda_device(coords)
    _need(coords, "coords", torch.float32, 2, dev)
    _need(offsets, "offsets", torch.int64, 1, dev)
    _need(centroids, "centroids", torch.float32, 3, dev)
    if valid_tokens is not None:
        _need(valid_tokens, "valid_tokens", torch.int32, 1, dev)
    P, B, K = coords.shape[0], offsets.numel() - 1, centroids.shape[1]
    if centroids.shape[0] != B or centroids.shape[2] != 4:
        raise ValueError("centroids must be [B, K, 4]")
    lib = _lib.load()
    ws = _workspace(lib.fps_assign_workspace_bytes(P, B), dev, workspace)
    tok = out if out is not None else torch.empty(P, dtype=torch.int32, device=dev)
    st = lib.fps_assign(_ptr(coords), _ptr(offsets), B, P, _ptr(centroids), _ptr(valid_tokens), K, _ptr(tok),
                        _axis_scale(axis_scale), _ptr(ws), ws.numel(), _stream(dev))
    _lib.check(st, "fps_assign")
    return tok


def fps_knn(coords: torch.Tensor, offsets: torch.Tensor, centroids: torch.Tensor, k: int,
            valid_tokens: Optional[torch.Tensor] = None, workspace: Optional[torch.Tensor] = None,
            out: Optional[torch.Tensor] = None, axis_scale=None) -> torch.Tensor:
    """C ``fps_knn``: the k nearest points (d, then index) of every valid
    centroid row, global indices, -1 padded; centroids [B, K, 4]."""
    dev = _cuda_device(coords)
    _need(coords, "coords", torch.float32, 2, dev)
    _need(offsets, "offsets", torch.int64, 1, dev)
    _need(centroids, "centroids", torch.float32, 3, dev)
    if valid_tokens is not None:
        _need(valid_tokens, "valid_tokens", torch.int32, 1, dev)
    P, B, K = coords.shape[0], offsets.numel() - 1, centroids.shape[1]
    lib = _lib.load()
    ws = _workspace(lib.fps_knn_workspace_bytes(P, B), dev, workspace)
    res = out if out is not None else torch.empty((B, K, k), dtype=torch.int32, device=dev)
    st = lib.fps_knn(_ptr(coords), _ptr(offsets), B, P, _ptr(centroids), _ptr(valid_tokens), K, k, _ptr(res),
                     _axis_scale(axis_scale), _ptr(ws), ws.numel(), _stream(dev))
    _lib.check(st, "fps_knn")
    return res


def lloyd_refine(coords: torch.Tensor, feats: Optional[torch.Tensor], offsets: torch.Tensor,
                 centroids: torch.Tensor, token_id: torch.Tensor, iters: int, charge_col: int = -1,
                 workspace: Optional[torch.Tensor] = None, axis_scale=None):
    """C ``lloyd_refine``: ``iters`` charge-weighted Lloyd iterations of every
    event with N > K, updating ``centroids`` [B,K,4] and ``token_id`` [P] in
    place.  Returns them."""
    dev = _cuda_device(coords)
    _need(coords, "coords", torch.float32, 2, dev)
    _need(offsets, "offsets", torch.int64, 1, dev)
    _need(centroids, "centroids", torch.float32, 3, dev)
    _need(token_id, "token_id", torch.int32, 1, dev)
    F = 0
    if feats is not None:
        _need(feats, "feats", torch.float32, 2, dev)
        F = feats.shape[1]
    P, B, K = coords.shape[0], offsets.numel() - 1, centroids.shape[1]
    lib = _lib.load()
    ws = _workspace(lib.lloyd_workspace_bytes(P, B, K), dev, workspace)
    st = lib.lloyd_refine(_ptr(coords), _ptr(feats), F, charge_col, _ptr(offsets), B, P, K, iters,
                          _ptr(centroids), _ptr(token_id), _axis_scale(axis_scale), _ptr(ws), ws.numel(),
                          _stream(dev))
    _lib.check(st, "lloyd_refine")
    return centroids, token_id


def segment_pool(feats: torch.Tensor, offsets: Optional[torch.Tensor], K: int,
                 token_id: Optional[torch.Tensor] = None, knn_idx: Optional[torch.Tensor] = None,
                 workspace: Optional[torch.Tensor] = None):
    """C ``segment_pool``: per-token mean of the features, by Voronoi labels
    (``token_id``) or by kNN rows (``knn_idx [B,K,k]``).  Returns
    ``(pooled [B,K,F], counts [B,K])``."""
    dev = _cuda_device(feats)
    _need(feats, "feats", torch.float32, 2, dev)
    P, F = feats.shape
    lib = _lib.load()
    if knn_idx is not None:
        _need(knn_idx, "knn_idx", torch.int32, 3, dev)
        B, K2, k = knn_idx.shape
        if K2 != K:
            raise ValueError("knn_idx must be [B, K, k]")
        mode, nb = _lib.FPS_ASSIGN_KNN, 256
        offp = None
    else:
        if token_id is None or offsets is None:
            raise ValueError("Voronoi pooling needs offsets and token_id")
        _need(offsets, "offsets", torch.int64, 1, dev)
        _need(token_id, "token_id", torch.int32, 1, dev)
        B, k = offsets.numel() - 1, 0
        mode, nb = _lib.FPS_ASSIGN_VORONOI, lib.segment_pool_workspace_bytes(P, B, K, F)
        offp = offsets
    ws = _workspace(nb, dev, workspace)
    pooled = torch.empty((B, K, F), dtype=torch.float32, device=dev)
    counts = torch.empty((B, K), dtype=torch.int32, device=dev)
    st = lib.segment_pool(_ptr(feats), F, _ptr(offp), B, P, K, mode, _ptr(token_id), _ptr(knn_idx), k,
                          _ptr(pooled), _ptr(counts), _ptr(ws), ws.numel(), _stream(feats.device))
    _lib.check(st, "segment_pool")
    return pooled, counts


def segment_pool_backward(grad_pooled: torch.Tensor, counts: torch.Tensor, P: int,
                          offsets: Optional[torch.Tensor] = None, token_id: Optional[torch.Tensor] = None,
                          knn_idx: Optional[torch.Tensor] = None, workspace: Optional[torch.Tensor] = None):
    """C ``segment_pool_backward``: the gradient [P, F] of the pooled rows
    ``grad_pooled [B,K,F]`` with respect to the features, given the forward's
    ``counts [B,K]`` and its Voronoi labels (``offsets`` + ``token_id``) or
    kNN rows (``knn_idx [B,K,k]``)."""
    dev = _cuda_device(grad_pooled)
    _need(grad_pooled, "grad_pooled", torch.float32, 3, dev)
    _need(counts, "counts", torch.int32, 2, dev)
    B, K, F = grad_pooled.shape
    if tuple(counts.shape) != (B, K):
        raise ValueError("counts must be [B, K] like grad_pooled")
    lib = _lib.load()
    if knn_idx is not None:
        _need(knn_idx, "knn_idx", torch.int32, 3, dev)
        if tuple(knn_idx.shape[:2]) != (B, K):
            raise ValueError("knn_idx must be [B, K, k]")
        mode, k, offp = _lib.FPS_ASSIGN_KNN, knn_idx.shape[2], None
        if offsets is not None:  # lets each event's rows be summed in shared memory first
            _need(offsets, "offsets", torch.int64, 1, dev)
            if offsets.numel() != B + 1:
                raise ValueError("offsets must be [B + 1]")
            offp = offsets
    else:
        if token_id is None or offsets is None:
            raise ValueError("the Voronoi backward needs offsets and token_id")
        _need(offsets, "offsets", torch.int64, 1, dev)
        _need(token_id, "token_id", torch.int32, 1, dev)
        if offsets.numel() != B + 1 or token_id.numel() != P:
            raise ValueError("offsets must be [B + 1] and token_id [P]")
        mode, k, offp = _lib.FPS_ASSIGN_VORONOI, 0, offsets
    ws = _workspace(lib.segment_pool_backward_workspace_bytes(P, B, K, F, mode), dev, workspace)
    grad_feats = torch.empty((P, F), dtype=torch.float32, device=dev)
    st = lib.segment_pool_backward(_ptr(grad_pooled), F, _ptr(offp), B, P, K, mode, _ptr(token_id),
                                   _ptr(knn_idx), k, _ptr(counts), _ptr(grad_feats), _ptr(ws), ws.numel(),
                                   _stream(dev))
    _lib.check(st, "segment_pool_backward")
    return grad_feats


def random_starts(offsets: torch.Tensor, seed: int, stream_id: int = 0) -> torch.Tensor:
    """C ``fps_random_starts``: a Philox4x32-10 draw of one local FPS start
    index per event, int32 [B] on the device (for ``start_local``)."""
    dev = _cuda_device(offsets)
    _need(offsets, "offsets", torch.int64, 1, dev)
    B = offsets.numel() - 1
    out = torch.empty(max(B, 0), dtype=torch.int32, device=dev)
    st = _lib.load().fps_random_starts(_ptr(offsets), B, int(seed) & 0xFFFFFFFFFFFFFFFF,
                                       int(stream_id) & 0xFFFFFFFF, _ptr(out), _stream(dev))
    _lib.check(st, "fps_random_starts")
    return out


def token_summaries(coords: torch.Tensor, feats: torch.Tensor, offsets: torch.Tensor, K: int,
                    token_id: torch.Tensor, charge_col: int = -1, workspace: Optional[torch.Tensor] = None):
    """C ``fps_token_summaries``: per Voronoi token the total charge and the
    charge-weighted means of the coordinates and features (unit charge when
    ``charge_col`` is -1).  Returns ``(wsum [B,K], wcoords [B,K,4],
    wfeats [B,K,F])``."""
    dev = _cuda_device(coords)
    _need(coords, "coords", torch.float32, 2, dev)
    _need(feats, "feats", torch.float32, 2, dev)
    _need(offsets, "offsets", torch.int64, 1, dev)
    _need(token_id, "token_id", torch.int32, 1, dev)
    P, F = feats.shape
    if coords.shape != (P, 4) or token_id.numel() != P:
        raise ValueError("coords must be [P, 4] and token_id [P] for feats [P, F]")
    B = offsets.numel() - 1
    lib = _lib.load()
    ws = _workspace(lib.fps_token_summaries_workspace_bytes(B, K, F), dev, workspace)
    wsum = torch.empty((B, K), dtype=torch.float32, device=dev)
    wcoords = torch.empty((B, K, 4), dtype=torch.float32, device=dev)
    wfeats = torch.empty((B, K, F), dtype=torch.float32, device=dev)
    st = lib.fps_token_summaries(_ptr(coords), _ptr(feats), F, charge_col, _ptr(offsets), B, P, K,
                                 _ptr(token_id), _ptr(wsum), _ptr(wcoords), _ptr(wfeats), _ptr(ws), ws.numel(),
                                 _stream(dev))
    _lib.check(st, "fps_token_summaries")
    return wsum, wcoords, wfeats


def pack_tokens(src: torch.Tensor, offsets: Optional[torch.Tensor] = None,
                valid_tokens: Optional[torch.Tensor] = None, workspace: Optional[torch.Tensor] = None):
    """C ``fps_pack_tokens``: the packed layout of padded tokens ``src [B, K, D]``
    (event b keeps ``valid_tokens[b]`` rows, else ``min(N_b, K)`` from the
    point ``offsets``).  Returns ``(dst [N_tok, D], doc_id [N_tok],
    tok_offsets [B + 1])``; reading the packed length synchronises the
    current stream once."""
    dev = _cuda_device(src)
    _need(src, "src", torch.float32, 3, dev)
    B, K, D = src.shape
    if valid_tokens is not None:
        _need(valid_tokens, "valid_tokens", torch.int32, 1, dev)
        if valid_tokens.numel() != B:
            raise ValueError("valid_tokens must be [B]")
    elif offsets is not None:
        _need(offsets, "offsets", torch.int64, 1, dev)
        if offsets.numel() != B + 1:
            raise ValueError("offsets must be [B + 1]")
    else:
        raise ValueError("pack_tokens needs offsets or valid_tokens")
    lib = _lib.load()
    ws = _workspace(lib.fps_pack_workspace_bytes(), dev, workspace)
    dst = torch.empty((max(B * K, 1), D), dtype=torch.float32, device=dev)
    doc_id = torch.empty(max(B * K, 1), dtype=torch.int32, device=dev)
    tok_offsets = torch.empty(B + 1, dtype=torch.int64, device=dev)
    st = lib.fps_pack_tokens(_ptr(src), D, _ptr(offsets), _ptr(valid_tokens), B, K, _ptr(dst), _ptr(doc_id),
                             _ptr(tok_offsets), _ptr(ws), ws.numel(), _stream(dev))
    _lib.check(st, "fps_pack_tokens")
    n_tok = int(tok_offsets[-1].item())
    return dst[:n_tok], doc_id[:n_tok], tok_offsets


def unpack_tokens(src: torch.Tensor, tok_offsets: torch.Tensor, K: int,
                  workspace: Optional[torch.Tensor] = None):
    """C ``fps_unpack_tokens``: packed rows ``src [N_tok, D]`` back to the
    padded layout ``[B, K, D]`` with zero padding."""
    dev = _cuda_device(src)
    _need(src, "src", torch.float32, 2, dev)
    _need(tok_offsets, "tok_offsets", torch.int64, 1, dev)
    B = tok_offsets.numel() - 1
    n_tok, D = src.shape
    lib = _lib.load()
    ws = _workspace(lib.fps_pack_workspace_bytes(), dev, workspace)
    dst = torch.empty((B, K, D), dtype=torch.float32, device=dev)
    st = lib.fps_unpack_tokens(_ptr(src), D, n_tok, _ptr(tok_offsets), B, K, _ptr(dst), _ptr(ws), ws.numel(),
                               _stream(dev))
    _lib.check(st, "fps_unpack_tokens")
    return dst


class _SegmentMean(torch.autograd.Function):
    """Mean-pool with its gradient to the features; both directions are the
    C ``segment_pool`` / ``segment_pool_backward`` calls."""

    @staticmethod
    def forward(ctx, feats, offsets, K, token_id, knn_idx):
        pooled, counts = segment_pool(feats, offsets, K, token_id=token_id, knn_idx=knn_idx)
        ctx.save_for_backward(offsets, token_id, knn_idx, counts)
        ctx.P = feats.shape[0]
        ctx.mark_non_differentiable(counts)
        return pooled, counts

    @staticmethod
    def backward(ctx, grad_pooled, _grad_counts):
        offsets, token_id, knn_idx, counts = ctx.saved_tensors
        g = segment_pool_backward(grad_pooled.contiguous(), counts, ctx.P, offsets=offsets, token_id=token_id,
                                  knn_idx=knn_idx)
        return g, None, None, None, None


def segment_mean(feats: torch.Tensor, offsets: Optional[torch.Tensor], K: int,
                 token_id: Optional[torch.Tensor] = None, knn_idx: Optional[torch.Tensor] = None):
    """``segment_pool`` that autograd differentiates with respect to
    ``feats``.  Returns ``(pooled [B,K,F], counts [B,K])``."""
    return _SegmentMean.apply(feats, offsets, K, token_id, knn_idx)


def device_status(workspace: torch.Tensor) -> None:
    """Reads the device-side status word of a workspace (synchronises the
    current stream) and raises ``FpsError`` if a check failed."""
    lib = _lib.load()
    detail = ctypes.c_int(0)
    st = lib.fps_device_status(_ptr(workspace), _stream(workspace.device), ctypes.byref(detail))
    if st != _lib.FPS_OK:
        err = _lib.FpsError(st, f"device check (reason {detail.value})")
        err.detail = detail.value
        raise err


def launch_count() -> int:
    """Kernels launched by libfpstok in this process."""
    return int(_lib.load().fps_launch_count())


def set_stage_events(events) -> None:
    """Record ``events[2s]`` / ``events[2s+1]`` (torch.cuda.Event, already
    created) around internal stage s of the following calls; None disables."""
    lib = _lib.load()
    if not events:
        lib.fps_set_stage_events(None, 0)
        return
    arr = (ctypes.c_void_p * len(events))(*[ctypes.c_void_p(e.cuda_event) for e in events])
    lib.fps_set_stage_events(arr, len(events))
