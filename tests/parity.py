"""Helpers shared by the GPU parity tests: run a batch through the CUDA path
(C ABI via the binding) and compare it with the CPU oracle."""
from __future__ import annotations

import numpy as np
import torch

import oracle

RTOL = 1e-5  # pooled means and Lloyd centroids: max relative error
ATOL = 1e-6  # absolute floor


def to_dev(batch, device="cuda"):
    c = torch.from_numpy(batch.coords).to(device)
    f = torch.from_numpy(batch.feats).to(device)
    o = torch.from_numpy(batch.offsets).to(device)
    s = None if batch.start_local is None else torch.from_numpy(batch.start_local).to(device)
    return c, f, o, s


def run_gpu(batch, force_schedule=-1, host_offsets=False, **kw):
    import farthest_point_sampling_b200 as fps

    c, f, o, s = to_dev(batch)
    if host_offsets:
        o = torch.from_numpy(batch.offsets)
    kw.setdefault("axis_scale", getattr(batch, "axis_scale", None))
    out = fps.fps_tokenize(c, f, o, K=batch.K, assign_mode=batch.assign_mode, k=max(batch.k, 1),
                           lloyd_iters=batch.lloyd_iters, charge_col=batch.charge_col, start_local=s,
                           force_schedule=force_schedule, check_device=True, **kw)
    torch.cuda.synchronize()
    return {k: v.cpu().numpy() for k, v in out.items()}


def assert_float_close(got, want, what):
    got = np.asarray(got, np.float64)
    want = np.asarray(want, np.float64)
    err = np.abs(got - want)
    bad = err > RTOL * np.abs(want) + ATOL
    assert not bad.any(), f"{what}: {bad.sum()} values outside tolerance, worst {err.max():.3g}"


def compare(batch, gpu, ora=None):
    """Element-by-element comparison of a GPU run with the oracle."""
    if ora is None:
        ora = oracle.tokenize_batch(batch)
    K = batch.K
    w = getattr(batch, "axis_scale", None)
    np.testing.assert_array_equal(gpu["centroid_idx"], ora["centroid_idx"], err_msg="centroid_idx")
    sizes = batch.sizes()
    valid = np.minimum(sizes, K).astype(np.int32)
    if batch.lloyd_iters == 0:
        np.testing.assert_array_equal(gpu["centroids"], ora["centroids"], err_msg="centroids")
        np.testing.assert_array_equal(gpu["token_id"], ora["token_id"], err_msg="token_id")
    else:
        assert_float_close(gpu["centroids"], ora["centroids"], "lloyd centroids")
        # the final labels are the exact nearest centroids of the GPU's centroids
        want = oracle.assign(batch.coords, batch.offsets, gpu["centroids"], K, valid=valid, axis_scale=w)
        pt = np.repeat(sizes <= K, sizes)
        want[pt] = ora["token_id"][pt]
        np.testing.assert_array_equal(gpu["token_id"], want, err_msg="token_id after Lloyd")
    if batch.assign_mode == 1:
        if batch.lloyd_iters == 0:
            np.testing.assert_array_equal(gpu["knn_idx"], ora["knn_idx"], err_msg="knn_idx")
        else:
            want = oracle.knn(batch.coords, batch.offsets, gpu["centroids"], K, batch.k, valid=valid, axis_scale=w)
            big = sizes > K
            np.testing.assert_array_equal(gpu["knn_idx"][big], want[big], err_msg="knn_idx after Lloyd")
            np.testing.assert_array_equal(gpu["knn_idx"][~big], ora["knn_idx"][~big])
        want_p, want_c = oracle.pool_knn(batch.feats, gpu["knn_idx"])
    else:
        want_p, want_c = oracle.pool_voronoi(batch.feats, batch.offsets, K, gpu["token_id"])
    np.testing.assert_array_equal(gpu["counts"], want_c, err_msg="counts")
    assert_float_close(gpu["pooled"], want_p, "pooled")
    np.testing.assert_array_equal(gpu["counts"], ora["counts"], err_msg="counts vs oracle pipeline")
    assert_float_close(gpu["pooled"], ora["pooled"], "pooled vs oracle pipeline")
    return ora
