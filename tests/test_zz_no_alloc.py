"""The allocation-free tokenizer entry point, fps_tokenize_static.

It serves callers that cannot allocate device memory (a plugin inside a host
program that owns all GPU memory, or a caller that cannot accept the
synchronisation cudaMalloc can cause): it keeps its scratch in a static device
array instead of a caller-provided workspace.  These tests call it through the
C ABI three times in a row, with different batches so that every call after
the first starts from the scratch contents the previous one left (a kNN batch
with Lloyd, a Voronoi batch, then the kNN batch again), and check every output
against the workspace-taking fps_tokenize within the tolerances the other
parity tests use, and the Voronoi batch also against the CPU oracle.  The
device status word of the static path is read back after a call with a start
index outside its event.  This file is collected last on purpose.
"""
import ctypes

import numpy as np
import pytest

import oracle
import workloads
from parity import ATOL, RTOL

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

if not torch.cuda.is_available():  # pragma: no cover
    pytest.skip("needs a CUDA device", allow_module_level=True)

import farthest_point_sampling_b200 as fps  # noqa: E402
from farthest_point_sampling_b200 import _lib  # noqa: E402


def _call_static(lib, b, out, dev, start=None):
    c = torch.from_numpy(b.coords).to(dev)
    f = torch.from_numpy(b.feats).to(dev)
    o = torch.from_numpy(b.offsets).to(dev)
    opts = fps.Options(K=b.K, assign_mode=b.assign_mode, k=max(b.k, 1), lloyd_iters=b.lloyd_iters,
                       charge_col=b.charge_col)
    p = lambda t: None if t is None else ctypes.c_void_p(t.data_ptr())  # noqa: E731
    stream = ctypes.c_void_p(torch.cuda.current_stream(dev).cuda_stream)
    st = None if start is None else torch.tensor(start, dtype=torch.int32, device=dev)
    rc = lib.fps_tokenize_static(p(c), p(f), b.F, p(o), b.B, b.P, p(st), ctypes.byref(opts.c),
                                 p(out["centroid_idx"]), p(out["token_id"]), p(out.get("knn_idx")),
                                 p(out["centroids"]), p(out["pooled"]), p(out["counts"]), stream)
    torch.cuda.synchronize(dev)
    return rc


def _reference(b, dev):
    c = torch.from_numpy(b.coords).to(dev)
    f = torch.from_numpy(b.feats).to(dev)
    o = torch.from_numpy(b.offsets).to(dev)
    out = fps.fps_tokenize(c, f, o, K=b.K, assign_mode=b.assign_mode, k=max(b.k, 1), lloyd_iters=b.lloyd_iters,
                           charge_col=b.charge_col)
    torch.cuda.synchronize(dev)
    return {k: v.cpu().numpy() for k, v in out.items()}


def _garbage_outputs(ref, dev):
    out = {}
    for k, v in ref.items():
        t = torch.from_numpy(v).to(dev)
        t.fill_(-7)  # results must not depend on what the buffers held
        out[k] = t
    return out


def test_static_entry_point_matches_workspace_entry_point_twice():
    dev = torch.device("cuda:0")
    lib = fps.load_library()
    # a kNN batch with Lloyd first, then a Voronoi batch, then the kNN batch
    # again, so every later call reuses scratch the one before dirtied (the
    # kNN and Lloyd words included)
    knn = workloads.random_batch(901, [0, 5, 100, 129, 700, 5000, 30000], 64, assign_mode=1, k=16,
                                 lloyd_iters=2, charge_col=0)
    batches = [knn, workloads.make_workload("c1"), knn]
    for b in batches:
        ref = _reference(b, dev)
        out = _garbage_outputs(ref, dev)
        assert _call_static(lib, b, out, dev) == _lib.FPS_OK
        got = {k: v.cpu().numpy() for k, v in out.items()}
        for k in ("centroid_idx", "token_id", "counts") + (("knn_idx",) if b.assign_mode == 1 else ()):
            np.testing.assert_array_equal(got[k], ref[k], err_msg=k)
        for k in ("centroids", "pooled"):
            err = np.abs(got[k].astype(np.float64) - ref[k])
            assert np.all(err <= RTOL * np.abs(ref[k]) + ATOL), k
        assert lib.fps_static_device_status(None, None) == _lib.FPS_OK
        if b.assign_mode == 0:  # the Voronoi batch also straight against the CPU oracle
            want = oracle.tokenize_batch(b)
            for k in ("centroid_idx", "token_id", "counts"):
                np.testing.assert_array_equal(got[k], want[k], err_msg=f"oracle {k}")
            for k in ("centroids", "pooled"):
                err = np.abs(got[k].astype(np.float64) - want[k])
                assert np.all(err <= RTOL * np.abs(want[k]) + ATOL), f"oracle {k}"


def test_static_entry_point_reports_device_errors():
    dev = torch.device("cuda:0")
    lib = fps.load_library()
    b = workloads.random_batch(902, [300, 40, 500], 16)
    ref = _reference(b, dev)
    out = _garbage_outputs(ref, dev)
    # event 2 starts at local index 600 of its 500 points: the binning kernel
    # skips it and records the reason in the static array's status word
    assert _call_static(lib, b, out, dev, start=[0, 0, 600]) == _lib.FPS_OK
    detail = ctypes.c_int(0)
    assert lib.fps_static_device_status(None, ctypes.byref(detail)) == _lib.FPS_ERR_DEVICE
    assert detail.value == 2  # FPS_DEV_BAD_START
    # the word is cleared by the read, and a good call leaves it clear
    assert lib.fps_static_device_status(None, None) == _lib.FPS_OK
    assert _call_static(lib, b, out, dev) == _lib.FPS_OK
    assert lib.fps_static_device_status(None, None) == _lib.FPS_OK
    np.testing.assert_array_equal(out["centroid_idx"].cpu().numpy(), ref["centroid_idx"])


def test_static_entry_point_rejects_batches_beyond_its_scratch():
    lib = fps.load_library()
    opts = fps.Options(K=128)
    P, B = 20_000_000, 200_000  # needs far more than the static scratch
    assert lib.fps_workspace_bytes(P, B, 6, ctypes.byref(opts.c)) > (8 << 20)
    x = ctypes.c_void_p(256)
    rc = lib.fps_tokenize_static(x, x, 6, x, B, P, None, ctypes.byref(opts.c), x, x, None, x, x, x, None)
    assert rc == _lib.FPS_ERR_TOO_LARGE
