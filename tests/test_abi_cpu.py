"""CPU-only checks of the C ABI: the library loads, exports every function the
header declares, and rejects bad arguments on the host before any launch
(none of these calls reach the GPU)."""
import ctypes
import os
import re

import pytest

import farthest_point_sampling_b200 as fps
from farthest_point_sampling_b200 import _lib

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "fpstok.h")


def header_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    names = re.findall(r"^[A-Za-z_][\w \*]*?\b(\w+)\s*\(", text, flags=re.M)
    return sorted(set(n for n in names if n not in ("if", "while")))


def test_header_parses():
    names = header_functions()
    assert "fps_tokenize" in names and "segment_pool" in names and len(names) >= 15


def test_library_exports_every_declared_symbol():
    lib = fps.load_library()
    for name in header_functions():
        assert hasattr(lib, name), name
    declared = {n for n, _, _ in _lib.SIGNATURES}
    assert declared == set(header_functions())


def test_status_strings():
    lib = fps.load_library()
    for code in range(6):
        assert lib.fps_status_string(code)
    assert lib.fps_status_string(0) == b"ok"


def _tok(lib, opts, P=100, B=2, F=6, ws_bytes=1 << 20, ws=None, **kw):
    args = dict(coords=16, feats=16, F=F, offsets=16, B=B, P=P, start=None, cidx=16, tok=16, knn=16,
                cents=16, pooled=16, counts=16, ws=256 if ws is None else ws, ws_bytes=ws_bytes)
    args.update(kw)
    P_ = ctypes.c_void_p
    return lib.fps_tokenize(P_(args["coords"]), P_(args["feats"]), args["F"], P_(args["offsets"]), args["B"],
                            args["P"], P_(args["start"]) if args["start"] else None,
                            ctypes.byref(opts.c) if opts is not None else None,
                            P_(args["cidx"]), P_(args["tok"]), P_(args["knn"]) if args["knn"] else None,
                            P_(args["cents"]), P_(args["pooled"]), P_(args["counts"]), P_(args["ws"]),
                            args["ws_bytes"], None)


def test_host_side_argument_errors():
    lib = fps.load_library()
    O = fps.Options
    assert _tok(lib, None) == _lib.FPS_ERR_ARG
    assert _tok(lib, O(K=0)) == _lib.FPS_ERR_ARG
    assert _tok(lib, O(K=257)) == _lib.FPS_ERR_TOO_LARGE
    assert _tok(lib, O(K=16, assign_mode="knn", k=0)) == _lib.FPS_ERR_ARG
    assert _tok(lib, O(K=16, assign_mode="knn", k=17)) == _lib.FPS_ERR_TOO_LARGE
    assert _tok(lib, O(K=16, lloyd_iters=-1)) == _lib.FPS_ERR_ARG
    assert _tok(lib, O(K=16, charge_col=6)) == _lib.FPS_ERR_ARG
    assert _tok(lib, O(K=16), F=0) == _lib.FPS_ERR_ARG
    assert _tok(lib, O(K=16), F=65) == _lib.FPS_ERR_TOO_LARGE
    assert _tok(lib, O(K=16), P=1 << 31) == _lib.FPS_ERR_TOO_LARGE
    assert _tok(lib, O(K=16), B=-1) == _lib.FPS_ERR_ARG
    assert _tok(lib, O(K=16, force_schedule=5)) == _lib.FPS_ERR_ARG
    assert _tok(lib, O(K=16), coords=8) == _lib.FPS_ERR_ARG  # misaligned float4 rows
    assert _tok(lib, O(K=16), tok=0) == _lib.FPS_ERR_ARG  # Voronoi needs token_id
    assert _tok(lib, O(K=16, assign_mode="knn", k=4), knn=0) == _lib.FPS_ERR_ARG
    assert _tok(lib, O(K=16), ws_bytes=16) == _lib.FPS_ERR_WORKSPACE
    assert _tok(lib, O(K=16), ws=0) == _lib.FPS_ERR_WORKSPACE
    assert _tok(lib, O(K=16), ws=128) == _lib.FPS_ERR_WORKSPACE  # misaligned workspace
    assert _tok(lib, O(K=16), B=0) == _lib.FPS_OK  # empty batch: nothing to launch


def test_standalone_argument_errors():
    lib = fps.load_library()
    P_ = ctypes.c_void_p
    x = P_(256)
    assert lib.fps_assign(x, x, 2, 100, x, None, 0, x, None, x, 1 << 20, None) == _lib.FPS_ERR_ARG
    assert lib.fps_assign(x, x, 2, 100, x, None, 300, x, None, x, 1 << 20, None) == _lib.FPS_ERR_TOO_LARGE
    assert lib.fps_assign(x, x, 2, 100, x, None, 8, x, None, x, 8, None) == _lib.FPS_ERR_WORKSPACE
    assert lib.fps_knn(x, x, 2, 100, x, None, 8, 0, x, None, x, 1 << 20, None) == _lib.FPS_ERR_ARG
    assert lib.fps_knn(x, x, 2, 100, x, None, 8, 129, x, None, x, 1 << 20, None) == _lib.FPS_ERR_TOO_LARGE
    assert lib.lloyd_refine(x, None, 0, 0, x, 2, 100, 8, 1, x, x, None, x, 1 << 20, None) == _lib.FPS_ERR_ARG
    assert lib.lloyd_refine(x, x, 6, 0, x, 2, 100, 8, -1, x, x, None, x, 1 << 20, None) == _lib.FPS_ERR_ARG
    # a non-finite axis weight is an argument error, found before anything is launched
    bad = (ctypes.c_float * 4)(1.0, 1.0, 1.0, float("inf"))
    assert lib.fps_assign(x, x, 2, 100, x, None, 8, x, bad, x, 1 << 20, None) == _lib.FPS_ERR_ARG
    assert lib.fps_knn(x, x, 2, 100, x, None, 8, 4, x, bad, x, 1 << 20, None) == _lib.FPS_ERR_ARG
    assert lib.lloyd_refine(x, None, 0, -1, x, 2, 100, 8, 1, x, x, bad, x, 1 << 20, None) == _lib.FPS_ERR_ARG
    nan_opts = fps.Options(K=16, axis_scale=(1.0, float("nan"), 1.0, 1.0))
    assert _tok(lib, nan_opts) == _lib.FPS_ERR_ARG
    assert lib.segment_pool(x, 6, x, 2, 100, 8, 2, x, None, 0, x, x, x, 1 << 20, None) == _lib.FPS_ERR_ARG
    assert lib.segment_pool(x, 0, x, 2, 100, 8, 0, x, None, 0, x, x, x, 1 << 20, None) == _lib.FPS_ERR_ARG
    assert lib.segment_pool(x, 6, x, 2, 100, 8, 1, None, x, 0, x, x, x, 1 << 20, None) == _lib.FPS_ERR_ARG
    # segment_pool_backward(grad, F, offsets, B, P, K, mode, token_id, knn_idx, k, counts, grad_feats, ws, n, s)
    bw = lib.segment_pool_backward
    assert bw(x, 6, x, 2, 100, 8, 2, x, None, 0, x, x, x, 1 << 20, None) == _lib.FPS_ERR_ARG  # bad mode
    assert bw(x, 0, x, 2, 100, 8, 0, x, None, 0, x, x, x, 1 << 20, None) == _lib.FPS_ERR_ARG  # F = 0
    assert bw(x, 65, x, 2, 100, 8, 0, x, None, 0, x, x, x, 1 << 20, None) == _lib.FPS_ERR_TOO_LARGE
    assert bw(x, 6, x, 2, 100, 300, 0, x, None, 0, x, x, x, 1 << 20, None) == _lib.FPS_ERR_TOO_LARGE
    assert bw(x, 6, None, 2, 100, 8, 0, x, None, 0, x, x, x, 1 << 20, None) == _lib.FPS_ERR_ARG  # no offsets
    assert bw(x, 6, x, 2, 100, 8, 0, None, None, 0, x, x, x, 1 << 20, None) == _lib.FPS_ERR_ARG  # no labels
    assert bw(x, 6, x, 2, 100, 8, 0, x, None, 0, None, x, x, 1 << 20, None) == _lib.FPS_ERR_ARG  # no counts
    assert bw(x, 6, None, 2, 100, 8, 1, None, None, 4, x, x, x, 1 << 20, None) == _lib.FPS_ERR_ARG  # no rows
    assert bw(x, 6, None, 2, 100, 8, 1, None, x, 129, x, x, x, 1 << 20, None) == _lib.FPS_ERR_TOO_LARGE
    need = lib.segment_pool_backward_workspace_bytes(100, 2, 8, 6, 1)
    assert need >= 2 * 100 * 6 * 8
    assert bw(x, 6, None, 2, 100, 8, 1, None, x, 4, x, x, x, need - 1, None) == _lib.FPS_ERR_WORKSPACE
    assert bw(x, 6, x, 2, 0, 8, 0, x, None, 0, x, x, None, 0, None) == _lib.FPS_OK  # nothing to do
    # fps_pack_tokens(src, D, offsets, valid, B, K, dst, doc_id, tok_offsets, ws, n, s)
    pk, upk = lib.fps_pack_tokens, lib.fps_unpack_tokens
    wsb = lib.fps_pack_workspace_bytes()
    assert pk(x, 0, x, None, 2, 8, x, x, x, x, wsb, None) == _lib.FPS_ERR_ARG  # D = 0
    assert pk(x, 4, None, None, 2, 8, x, x, x, x, wsb, None) == _lib.FPS_ERR_ARG  # no offsets, no counts
    assert pk(x, 4, x, None, 2, 0, x, x, x, x, wsb, None) == _lib.FPS_ERR_ARG  # K = 0
    assert pk(x, 1 << 24, x, None, 2, 256, x, x, x, x, wsb, None) == _lib.FPS_ERR_TOO_LARGE
    assert pk(x, 4, x, None, 2, 8, x, x, x, None, wsb, None) == _lib.FPS_ERR_WORKSPACE
    assert upk(x, 4, -1, x, 2, 8, x, x, wsb, None) == _lib.FPS_ERR_ARG  # n_tok < 0
    assert upk(x, 4, 10, None, 2, 8, x, x, wsb, None) == _lib.FPS_ERR_ARG  # no tok_offsets
    assert upk(x, 4, 10, x, 0, 8, x, x, wsb, None) == _lib.FPS_OK  # B = 0
    # fps_token_summaries(coords, feats, F, charge_col, offsets, B, P, K, token_id, wsum, wc, wf, ws, n, s)
    ts = lib.fps_token_summaries
    nts = lib.fps_token_summaries_workspace_bytes(2, 8, 6)
    assert nts >= 2 * 8 * 11 * 8
    assert ts(x, x, 6, 6, x, 2, 100, 8, x, x, x, x, x, nts, None) == _lib.FPS_ERR_ARG  # charge_col >= F
    assert ts(x, x, 6, -2, x, 2, 100, 8, x, x, x, x, x, nts, None) == _lib.FPS_ERR_ARG
    assert ts(x, x, 6, 0, x, 2, 100, 300, x, x, x, x, x, nts, None) == _lib.FPS_ERR_TOO_LARGE
    assert ts(x, x, 6, 0, x, 2, 100, 8, None, x, x, x, x, nts, None) == _lib.FPS_ERR_ARG  # no token ids
    assert ts(x, x, 6, 0, x, 2, 100, 8, x, x, x, x, x, nts - 1, None) == _lib.FPS_ERR_WORKSPACE


def test_workspace_sizes_grow_with_problem():
    lib = fps.load_library()
    o = fps.Options(K=128)
    small = lib.fps_workspace_bytes(1000, 4, 6, ctypes.byref(o.c))
    big = lib.fps_workspace_bytes(1_000_000, 4096, 6, ctypes.byref(o.c))
    lloyd = lib.fps_workspace_bytes(1_000_000, 4096, 6, ctypes.byref(fps.Options(K=128, lloyd_iters=3).c))
    assert 0 < small < big < lloyd
    assert lib.fps_host_workspace_bytes(1000, 4, 6, ctypes.byref(o.c)) > small
    assert lib.fps_max_event_points() >= 200_000 - 4000


def test_binding_rejects_cpu_tensors_and_dtypes():
    torch = pytest.importorskip("torch")
    c = torch.zeros((10, 4))
    with pytest.raises(ValueError):
        fps.fps_tokenize(c, torch.zeros((10, 6)), torch.tensor([0, 10]), K=4)
    with pytest.raises(TypeError):
        fps.offsets_from_batch_ids(torch.zeros(5, dtype=torch.int32))
    # every other entry point refuses host tensors too: there is no CPU path
    off = torch.tensor([0, 10])
    tok = torch.zeros(10, dtype=torch.int32)
    calls = [
        lambda: fps.segment_pool_backward(torch.zeros((1, 4, 6)), torch.zeros((1, 4), dtype=torch.int32), 10,
                                          offsets=off, token_id=tok),
        lambda: fps.segment_mean(torch.zeros((10, 6)), off, 4, token_id=tok),
        lambda: fps.token_summaries(c, torch.zeros((10, 6)), off, 4, tok),
        lambda: fps.random_starts(off, 1),
        lambda: fps.pack_tokens(torch.zeros((1, 4, 6)), offsets=off),
        lambda: fps.unpack_tokens(torch.zeros((4, 6)), torch.tensor([0, 4]), 4),
        lambda: fps.segment_pool(torch.zeros((10, 6)), off, 4, token_id=tok),
    ]
    for call in calls:
        with pytest.raises(ValueError, match="CUDA"):
            call()


def test_offsets_from_batch_ids():
    torch = pytest.importorskip("torch")
    ids = torch.tensor([0, 0, 1, 1, 1, 3], dtype=torch.int64)
    assert fps.offsets_from_batch_ids(ids).tolist() == [0, 2, 5, 5, 6]
    assert fps.offsets_from_batch_ids(ids, num_events=5).tolist() == [0, 2, 5, 5, 6, 6]
    with pytest.raises(ValueError):
        fps.offsets_from_batch_ids(torch.tensor([0, 1, 0], dtype=torch.int64))
