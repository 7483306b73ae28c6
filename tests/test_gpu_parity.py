"""GPU parity: the CUDA path (through the C ABI) against the CPU oracle.

Indices, labels and kNN ids are compared bit for bit; pooled means and Lloyd
centroids within 1e-5 relative with a 1e-6 absolute floor.
"""
import numpy as np
import pytest

import oracle
import workloads
from parity import ATOL, RTOL, assert_float_close, compare, run_gpu, to_dev

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

if not torch.cuda.is_available():  # pragma: no cover - the gpu marker is deselected on CPU hosts
    pytest.skip("needs a CUDA device", allow_module_level=True)

import farthest_point_sampling_b200 as fps  # noqa: E402


@pytest.fixture(scope="module", autouse=True)
def _lib_loaded():
    fps.load_library()


# ------------------------------------------------------------- the five workloads

@pytest.mark.parametrize("name", ["c0", "c1", "c2", "c3", "c4"])
def test_workload_parity(name):
    b = workloads.make_workload(name)
    compare(b, run_gpu(b))


@pytest.mark.parametrize("K", [32, 64, 256])
def test_c4_k_sweep(K):
    b = workloads.make_workload("c4", K=K)
    compare(b, run_gpu(b))


def test_c1_host_offsets_hint():
    b = workloads.make_workload("c1")
    compare(b, run_gpu(b, host_offsets=True))


# ------------------------------------------------------------- sizes, tiles, ragged tails

EDGE_SIZES = [0, 1, 2, 15, 16, 17, 31, 32, 33, 63, 64, 65, 127, 128, 129, 447, 448, 449, 1000, 2559, 2560,
              2561, 3071, 3072, 3073, 4095, 12287, 12288, 12289, 30001, 98305]


@pytest.mark.parametrize("K", [1, 2, 16, 128, 256])
def test_edge_sizes(K):
    b = workloads.random_batch(100 + K, EDGE_SIZES, K, charge_col=0)
    compare(b, run_gpu(b))


@pytest.mark.parametrize("F", [1, 7, 12, 40, 64])
def test_fused_pooling_feature_counts(F):
    """The pooling the warp and register-CTA schedules fuse into FPS, across
    feature counts: with few features the warp copies the event's whole
    feature block into shared memory (447 points x 7 features still fit, 448
    do not), with more it stages a few features per pass; the register CTA
    pools in place only while its feature rows fit, else the pool kernel
    takes its events.  Event sizes around the warp and CTA capacities and
    around 16-byte boundaries of the feature block."""
    sizes = [129, 130, 131, 250, 383, 446, 447, 448, 449, 900, 2559, 2560, 5, 0, 300, 301]
    b = workloads.random_batch(900 + F, sizes, 128, F=F)
    compare(b, run_gpu(b))
    b = workloads.random_batch(950 + F, [447, 448] * 40 + [200] * 40, 128, F=F)
    compare(b, run_gpu(b))


@pytest.mark.parametrize("kind", ["dup", "grid", "allsame"])
def test_ties_and_duplicates(kind):
    sizes = [40, 200, 700, 3000, 15000]
    if kind == "dup":
        b = workloads.random_batch(7, sizes, 32, dup_frac=0.5)
    elif kind == "grid":
        b = workloads.random_batch(8, sizes, 32, grid=200.0)
    else:
        b = workloads.random_batch(9, sizes, 32)
        for e in range(b.B):
            o0, o1 = b.offsets[e], b.offsets[e + 1]
            b.coords[o0:o1] = b.coords[o0]
    compare(b, run_gpu(b))


@pytest.mark.parametrize("force", [-1, 0])
def test_warp_events_with_few_distinct_points(force):
    """Warp-schedule events with fewer distinct points than K: the arg-max
    reaches a zero maximum, after which the remaining centroids are the
    lowest-index unselected points.  The warp loop runs without an exit test
    and runs such an event again with one; every third event is one point
    repeated.  300 events, so that the automatic schedule is the warp one."""
    rng = np.random.default_rng(31)
    sizes = [int(n) for n in rng.integers(129, 449, 300)]
    b = workloads.random_batch(32, sizes, 128, dup_frac=0.7)
    for e in range(0, b.B, 3):
        o0, o1 = b.offsets[e], b.offsets[e + 1]
        b.coords[o0:o1] = b.coords[o0]
    compare(b, run_gpu(b, force_schedule=force))


@pytest.mark.parametrize("name", ["c4", "mixed"])
def test_warp_only_batches_with_a_size_hint(name):
    """Host offsets give the library the largest event size; when every FPS
    event fits the warp schedule, the warp kernel alone follows the binning,
    as a programmatic dependent launch on the caller's stream.  The 4096-event
    workload, and a batch with empty, tiny, N = K and N = K + 1 events between
    the warp-size ones."""
    if name == "c4":
        b = workloads.make_workload("c4")
    else:
        rng = np.random.default_rng(41)
        sizes = [int(n) for n in rng.integers(129, 449, 300)]
        for i, n in enumerate([0, 1, 5, 127, 128, 129, 0, 448, 3]):
            sizes.insert(i * 31, n)
        b = workloads.random_batch(42, sizes, 128, dup_frac=0.02)
    compare(b, run_gpu(b, host_offsets=True))


@pytest.mark.parametrize("force", [0, 1, 2, 3, 4])
def test_forced_schedules_agree(force):
    sizes = [129, 300, 448, 449, 2000, 2560, 2561, 12288, 12289, 40000, 98304, 98305]
    b = workloads.random_batch(11, sizes, 128, dup_frac=0.05)
    ora = oracle.tokenize_batch(b)
    compare(b, run_gpu(b, force_schedule=force), ora)


def test_start_local():
    sizes = [5, 300, 2000, 20000]
    rng = np.random.default_rng(3)
    starts = [int(rng.integers(0, n)) for n in sizes]
    b = workloads.random_batch(12, sizes, 64, start_local=starts)
    compare(b, run_gpu(b))


def test_time_shift_invariance_gpu():
    b = workloads.random_batch(13, [300, 3000, 20000], 64)
    rng = np.random.default_rng(4)
    t = np.round(rng.uniform(0, 2 ** 14, b.P) * 256) / 256
    b.coords[:, 3] = t.astype(np.float32)
    base = run_gpu(b)["centroid_idx"]
    b.coords[:, 3] = (t + 4096.5).astype(np.float32)
    np.testing.assert_array_equal(run_gpu(b)["centroid_idx"], base)


# ------------------------------------------------------------- kNN and Lloyd

@pytest.mark.parametrize("k", [1, 5, 32, 33, 64, 100, 128])
def test_knn_sizes(k):
    b = workloads.random_batch(20 + k, [0, 3, 100, 128, 129, 500, 5000, 13000], 128, assign_mode=1, k=k,
                               dup_frac=0.1)
    compare(b, run_gpu(b))


@pytest.mark.parametrize("iters,charge", [(1, 0), (3, 0), (2, -1), (4, 0)])
def test_lloyd_pipeline(iters, charge):
    b = workloads.random_batch(30 + iters, [50, 129, 600, 5000, 20000, 60000], 64, lloyd_iters=iters,
                               charge_col=charge)
    compare(b, run_gpu(b))


def test_knn_after_lloyd():
    b = workloads.random_batch(41, [20, 300, 4000], 32, assign_mode=1, k=16, lloyd_iters=2, charge_col=0)
    compare(b, run_gpu(b))


def test_lloyd_step_by_step():
    """Each GPU Lloyd iteration against one oracle iteration from the GPU's state."""
    b = workloads.make_workload("c3")
    c, f, o, _ = to_dev(b)
    out = fps.fps_tokenize(c, f, o, K=b.K)
    cent, tok = out["centroids"], out["token_id"]
    for _ in range(3):
        prev_c, prev_t = cent.cpu().numpy(), tok.cpu().numpy()
        fps.lloyd_refine(c, f, o, cent, tok, iters=1, charge_col=0)
        want_c, _ = oracle.lloyd(b.coords, b.feats, b.offsets, b.K, 1, prev_c, prev_t, charge_col=0)
        got_c = cent.cpu().numpy()
        assert_float_close(got_c, want_c, "one Lloyd step")
        want_t = oracle.assign(b.coords, b.offsets, got_c, b.K)
        np.testing.assert_array_equal(tok.cpu().numpy(), want_t)


# ------------------------------------------------------------- standalone entry points

def _fps_state(b):
    c, f, o, _ = to_dev(b)
    ora = oracle.tokenize_batch(b)
    cent = torch.from_numpy(ora["centroids"]).cuda()
    return c, f, o, ora, cent


def test_standalone_assign():
    b = workloads.random_batch(50, [0, 10, 100, 2047, 2048, 2049, 9000], 32)
    c, f, o, ora, cent = _fps_state(b)
    valid = np.minimum(b.sizes(), 32).astype(np.int32)
    valid[3] = 5  # fewer valid rows than tokens
    got = fps.fps_assign(c, o, cent, torch.from_numpy(valid).cuda()).cpu().numpy()
    want = oracle.assign(b.coords, b.offsets, ora["centroids"], 32, valid=valid)
    np.testing.assert_array_equal(got, want)
    got = fps.fps_assign(c, o, cent).cpu().numpy()
    np.testing.assert_array_equal(got, oracle.assign(b.coords, b.offsets, ora["centroids"], 32))


def test_standalone_knn():
    b = workloads.random_batch(51, [0, 10, 100, 2000], 32)
    c, f, o, ora, cent = _fps_state(b)
    for k in (1, 7, 32):
        got = fps.fps_knn(c, o, cent, k).cpu().numpy()
        want = oracle.knn(b.coords, b.offsets, ora["centroids"], 32, k)
        np.testing.assert_array_equal(got, want)


def test_standalone_pool():
    b = workloads.random_batch(52, [0, 10, 100, 511, 512, 513, 2047, 2048, 2049, 9000], 32, F=5)
    c, f, o, ora, cent = _fps_state(b)
    tok = torch.from_numpy(ora["token_id"]).cuda()
    pooled, counts = fps.segment_pool(f, o, 32, token_id=tok)
    wp, wc = oracle.pool_voronoi(b.feats, b.offsets, 32, ora["token_id"])
    np.testing.assert_array_equal(counts.cpu().numpy(), wc)
    assert_float_close(pooled.cpu().numpy(), wp, "segment_pool voronoi")
    knn = oracle.knn(b.coords, b.offsets, ora["centroids"], 32, 9)
    pooled, counts = fps.segment_pool(f, None, 32, knn_idx=torch.from_numpy(knn).cuda())
    wp, wc = oracle.pool_knn(b.feats, knn)
    np.testing.assert_array_equal(counts.cpu().numpy(), wc)
    assert_float_close(pooled.cpu().numpy(), wp, "segment_pool knn")


def _host_run(b, **kw):
    out = fps.fps_tokenize_host(torch.from_numpy(b.coords).pin_memory(), torch.from_numpy(b.feats).pin_memory(),
                                torch.from_numpy(b.offsets), K=b.K, assign_mode=b.assign_mode, k=max(b.k, 1),
                                lloyd_iters=b.lloyd_iters, charge_col=b.charge_col, **kw)
    return {k: v.numpy() for k, v in out.items()}


def test_host_entry_point():
    b = workloads.make_workload("c1")
    compare(b, _host_run(b))


@pytest.mark.parametrize("name", ["c4", "c2", "c3"])
def test_host_entry_point_in_slices(name):
    # batches of 65,536 points or more go through in slices of consecutive
    # events (copies in, compute and copies out overlapping): the slices'
    # global indices, kNN rows and Lloyd centroids must come back as one batch
    b = workloads.make_workload(name)
    assert b.P >= 65536
    compare(b, _host_run(b))


def test_host_entry_point_start_indices_and_host_checks():
    b = workloads.random_batch(64, [40000, 30000, 20, 5000, 9000], 32, start_local=[7, 29999, 0, 4, 8])
    st = torch.from_numpy(b.start_local)
    compare(b, _host_run(b, start_local=st))
    bad = st.clone()
    bad[1] = 30000  # outside its event: refused on the host, nothing runs
    with pytest.raises(fps.FpsError):
        _host_run(b, start_local=bad)
    off = torch.from_numpy(b.offsets).clone()
    off[2] = off[1] - 1  # decreasing offsets
    with pytest.raises(fps.FpsError):
        fps.fps_tokenize_host(torch.from_numpy(b.coords).pin_memory(), torch.from_numpy(b.feats).pin_memory(), off,
                              K=b.K)


# ------------------------------------------------------------- degenerate inputs and errors

def test_empty_batch_and_empty_events():
    c = torch.zeros((0, 4), device="cuda")
    f = torch.zeros((0, 6), device="cuda")
    out = fps.fps_tokenize(c, f, torch.zeros(1, dtype=torch.int64, device="cuda"), K=8)
    assert out["centroid_idx"].shape == (0, 8)
    b = workloads.random_batch(60, [0, 0, 0], 8)
    compare(b, run_gpu(b))


def test_device_errors_are_reported_without_fault():
    b = workloads.random_batch(61, [100, 200], 16, start_local=[5, 500])
    c, f, o, s = to_dev(b)
    with pytest.raises(fps.FpsError) as ei:
        fps.fps_tokenize(c, f, o, K=16, start_local=s, check_device=True)
    assert ei.value.detail == 2
    bad = torch.tensor([0, 100, 50, 300], dtype=torch.int64, device="cuda")
    c2 = torch.zeros((300, 4), device="cuda")
    f2 = torch.zeros((300, 6), device="cuda")
    with pytest.raises(fps.FpsError) as ei:
        fps.fps_tokenize(c2, f2, bad, K=16, check_device=True)
    assert ei.value.detail == 1
    # the context is still usable
    b = workloads.make_workload("c0")
    compare(b, run_gpu(b))


def test_dtype_is_not_converted():
    b = workloads.make_workload("c0")
    c, f, o, _ = to_dev(b)
    with pytest.raises(TypeError):
        fps.fps_tokenize(c.double(), f, o, K=16)
    with pytest.raises(TypeError):
        fps.fps_tokenize(c.half(), f, o, K=16)


def test_many_small_events_use_the_warp_schedule():
    # more FPS events than SMs: the warp schedule, in decreasing size order
    b = workloads.random_batch(70, np.random.default_rng(70).integers(129, 449, 700), 128)
    compare(b, run_gpu(b))


def test_no_host_sync_and_launch_count():
    b = workloads.make_workload("c1")
    c, f, o, _ = to_dev(b)
    fps.fps_tokenize(c, f, o, K=128)  # warm: workspace and outputs through the caching allocator
    torch.cuda.synchronize()
    before = fps.launch_count()
    torch.cuda.set_sync_debug_mode("error")
    try:
        fps.fps_tokenize(c, f, o, K=128)
    finally:
        torch.cuda.set_sync_debug_mode("default")
    n = fps.launch_count() - before
    assert 3 <= n <= 10, n
    torch.cuda.synchronize()


def test_cuda_graph_capture_and_replay():
    """One fps_tokenize call captured into a CUDA graph (the internal helper
    streams join the capture) and replayed on new inputs of the same shape."""
    dev = torch.device("cuda")
    b1 = workloads.make_workload("c1")
    b2 = workloads.random_batch(77, b1.sizes(), b1.K)  # same shapes, other values
    c, f, o, _ = to_dev(b1)
    out = fps.fps_tokenize(c, f, o, K=b1.K)  # first call on the device happens before capture
    ws = torch.empty(1 << 22, dtype=torch.uint8, device=dev)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.graph(g, stream=side):
        fps.fps_tokenize(c, f, o, K=b1.K, workspace=ws, out=out)
    for b in (b1, b2):
        c.copy_(torch.from_numpy(b.coords))
        f.copy_(torch.from_numpy(b.feats))
        g.replay()
        torch.cuda.synchronize()
        compare(b, {k: v.cpu().numpy() for k, v in out.items()})
