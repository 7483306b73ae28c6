"""Parity of the mean-pool backward (C ``segment_pool_backward``) with the oracle.

The Voronoi gradient is a float64 quotient rounded once, so it is compared
bit for bit.  The kNN gradient of an event whose rows name only its own
points, and whose points fit the kernel's shared buffer, is summed in row
order like the oracle's and compared bit for bit too; otherwise float64
shares meet in an order the atomics choose and the comparison uses the float
tolerance (1e-5 relative, 1e-6 absolute floor).  Labels, kNN rows and counts come from the oracle or from
seeded numpy draws, never from the CUDA path.
"""
import numpy as np
import pytest

import oracle
import workloads

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

if not torch.cuda.is_available():  # pragma: no cover - the gpu marker is deselected on CPU hosts
    pytest.skip("needs a CUDA device", allow_module_level=True)

import farthest_point_sampling_b200 as fps  # noqa: E402
from farthest_point_sampling_b200 import _lib  # noqa: E402
from parity import assert_float_close  # noqa: E402


def _dev(a):
    return torch.from_numpy(np.ascontiguousarray(a)).cuda()


def _random_labels(seed, sizes, K, unassigned=0.05):
    """Random token ids in 0..min(N,K)-1 per event, a share of them -1, and
    the matching counts."""
    rng = np.random.default_rng(seed)
    offsets = np.concatenate([[0], np.cumsum(sizes)]).astype(np.int64)
    tok = np.concatenate([rng.integers(0, max(min(int(n), K), 1), int(n)) for n in sizes] or [np.zeros(0)])
    tok = tok.astype(np.int32)
    tok[rng.random(tok.shape[0]) < unassigned] = -1
    counts = np.zeros((len(sizes), K), np.int32)
    ev = np.repeat(np.arange(len(sizes)), sizes)
    np.add.at(counts, (ev[tok >= 0], tok[tok >= 0]), 1)
    return offsets, tok, counts


@pytest.mark.parametrize("F", [1, 6, 7, 64])
def test_voronoi_backward_bitexact(F):
    # sizes span several 1024-point tiles, empty events and a ragged tail
    sizes = [0, 1, 37, 255, 256, 257, 1023, 1024, 1025, 0, 0, 2049, 3, 4097, 700]
    K = 32
    offsets, tok, counts = _random_labels(60 + F, sizes, K)
    rng = np.random.default_rng(70 + F)
    G = rng.normal(0, 3, (len(sizes), K, F)).astype(np.float32)
    want = oracle.pool_voronoi_backward(G, offsets, tok, counts)
    got = fps.segment_pool_backward(_dev(G), _dev(counts), len(tok), offsets=_dev(offsets), token_id=_dev(tok))
    np.testing.assert_array_equal(got.cpu().numpy(), want)


@pytest.mark.parametrize("F", [1, 6, 7])
def test_voronoi_backward_unaligned_output(F):
    """Through the C ABI into an output that starts 4 bytes past a 16-byte
    boundary (the binding allocates aligned outputs): every element in place,
    nothing written outside."""
    import ctypes

    from farthest_point_sampling_b200 import api
    sizes = [300, 1025, 7, 0, 2048, 5]
    K = 32
    offsets, tok, counts = _random_labels(80 + F, sizes, K)
    rng = np.random.default_rng(81 + F)
    G = rng.normal(0, 3, (len(sizes), K, F)).astype(np.float32)
    want = oracle.pool_voronoi_backward(G, offsets, tok, counts)
    lib = fps.load_library()
    P, B = len(tok), len(sizes)
    buf = torch.full((P * F + 4,), 7.0, dtype=torch.float32, device="cuda")
    out = buf[1:1 + P * F]
    assert out.data_ptr() % 16 == 4
    nb = lib.segment_pool_backward_workspace_bytes(P, B, K, F, 0)
    ws = torch.empty(max(nb, 256), dtype=torch.uint8, device="cuda")
    g, c, o, t = _dev(G), _dev(counts), _dev(offsets), _dev(tok)
    st = lib.segment_pool_backward(api._ptr(g), F, api._ptr(o), B, P, K, 0, api._ptr(t), None, 0, api._ptr(c),
                                   ctypes.c_void_p(out.data_ptr()), api._ptr(ws), ws.numel(),
                                   api._stream(torch.device("cuda")))
    assert st == 0
    fps.device_status(ws)
    np.testing.assert_array_equal(out.cpu().numpy().reshape(P, F), want)
    assert buf[0].item() == 7.0 and buf[-3:].cpu().tolist() == [7.0, 7.0, 7.0]


def test_voronoi_backward_from_the_tokenizer_labels():
    b = workloads.make_workload("c1")
    ora = oracle.tokenize_batch(b)
    rng = np.random.default_rng(71)
    G = rng.normal(0, 1, ora["pooled"].shape).astype(np.float32)
    want = oracle.pool_voronoi_backward(G, b.offsets, ora["token_id"], ora["counts"])
    got = fps.segment_pool_backward(_dev(G), _dev(ora["counts"]), b.coords.shape[0], offsets=_dev(b.offsets),
                                    token_id=_dev(ora["token_id"]))
    np.testing.assert_array_equal(got.cpu().numpy(), want)


def test_voronoi_backward_full_size():
    """About a million points in 8 events (the large-event workload's sizes),
    every element checked."""
    b = workloads.make_workload("c3")
    sizes = np.diff(b.offsets)
    offsets, tok, counts = _random_labels(72, sizes, b.K, unassigned=0.0)
    rng = np.random.default_rng(73)
    G = rng.normal(0, 1, (len(sizes), b.K, b.feats.shape[1])).astype(np.float32)
    want = oracle.pool_voronoi_backward(G, offsets, tok, counts)
    got = fps.segment_pool_backward(_dev(G), _dev(counts), len(tok), offsets=_dev(offsets), token_id=_dev(tok))
    np.testing.assert_array_equal(got.cpu().numpy(), want)


def test_voronoi_backward_zero_count_cells():
    """Counts that disagree with the labels: a zero count gives no gradient."""
    sizes = [300, 200]
    offsets, tok, counts = _random_labels(74, sizes, 8)
    counts[0, 3] = 0
    counts[1, :] = 0
    G = np.ones((2, 8, 3), np.float32)
    want = oracle.pool_voronoi_backward(G, offsets, tok, counts)
    got = fps.segment_pool_backward(_dev(G), _dev(counts), len(tok), offsets=_dev(offsets), token_id=_dev(tok))
    np.testing.assert_array_equal(got.cpu().numpy(), want)
    assert np.all(want[300:] == 0) and np.all(want[:300][tok[:300] == 3] == 0)


@pytest.mark.parametrize("k", [1, 9, 32, 33, 100])
def test_knn_backward(k):
    b = workloads.random_batch(75, [0, 5, 40, 300, 1500, 5000], 32, F=5)
    ora = oracle.tokenize(b.coords, b.feats, b.offsets, 32)
    knn = oracle.knn(b.coords, b.offsets, ora["centroids"], 32, k)
    counts = (knn >= 0).sum(2).astype(np.int32)
    rng = np.random.default_rng(76 + k)
    G = rng.normal(0, 2, (len(b.offsets) - 1, 32, 5)).astype(np.float32)
    want = oracle.pool_knn_backward(G, knn, counts, b.coords.shape[0])
    got = fps.segment_pool_backward(_dev(G), _dev(counts), b.coords.shape[0], knn_idx=_dev(knn))
    assert_float_close(got.cpu().numpy(), want, f"segment_pool_backward knn k={k}")
    # with offsets every event here fits in shared memory: its entries are
    # grouped by point and summed in row order, exactly as the oracle sums
    got = fps.segment_pool_backward(_dev(G), _dev(counts), b.coords.shape[0], knn_idx=_dev(knn),
                                    offsets=_dev(b.offsets))
    np.testing.assert_array_equal(got.cpu().numpy(), want)


def test_knn_backward_rows_outside_their_event():
    """Rows may name any point: entries outside their event take the global path."""
    rng = np.random.default_rng(81)
    sizes = [50, 3000, 0, 400]
    offsets = np.concatenate([[0], np.cumsum(sizes)]).astype(np.int64)
    P, B, K, k = int(offsets[-1]), len(sizes), 16, 8
    knn = rng.integers(-1, P, (B, K, k)).astype(np.int32)
    counts = (knn >= 0).sum(2).astype(np.int32)
    G = rng.normal(0, 1, (B, K, 3)).astype(np.float32)
    want = oracle.pool_knn_backward(G, knn, counts, P)
    for offp in (None, _dev(offsets)):
        got = fps.segment_pool_backward(_dev(G), _dev(counts), P, knn_idx=_dev(knn), offsets=offp)
        assert_float_close(got.cpu().numpy(), want, "segment_pool_backward knn, rows across events")


def test_knn_backward_full_size():
    """The kNN workload (256 events, k = 32) with kNN rows from the oracle."""
    b = workloads.make_workload("c2")
    ora = oracle.tokenize_batch(b)
    knn = ora["knn_idx"]
    G = np.random.default_rng(77).normal(0, 1, ora["pooled"].shape).astype(np.float32)
    want = oracle.pool_knn_backward(G, knn, ora["counts"], b.coords.shape[0])
    for offp in (None, _dev(b.offsets)):
        got = fps.segment_pool_backward(_dev(G), _dev(ora["counts"]), b.coords.shape[0], knn_idx=_dev(knn),
                                        offsets=offp)
        assert_float_close(got.cpu().numpy(), want, "segment_pool_backward knn (full size)")


def test_segment_mean_autograd():
    b = workloads.random_batch(78, [0, 20, 600, 3000], 16, F=6)
    ora = oracle.tokenize(b.coords, b.feats, b.offsets, 16)
    feats = _dev(b.feats).requires_grad_(True)
    pooled, counts = fps.segment_mean(feats, _dev(b.offsets), 16, token_id=_dev(ora["token_id"]))
    np.testing.assert_array_equal(counts.cpu().numpy(), ora["counts"])
    G = np.random.default_rng(79).normal(0, 1, pooled.shape).astype(np.float32)
    (pooled * _dev(G)).sum().backward()
    want = oracle.pool_voronoi_backward(G, b.offsets, ora["token_id"], ora["counts"])
    np.testing.assert_array_equal(feats.grad.cpu().numpy(), want)

    knn = oracle.knn(b.coords, b.offsets, ora["centroids"], 16, 4)
    feats.grad = None
    pooled, counts = fps.segment_mean(feats, _dev(b.offsets), 16, knn_idx=_dev(knn))
    (pooled * _dev(G)).sum().backward()
    want = oracle.pool_knn_backward(G, knn, counts.cpu().numpy(), b.coords.shape[0])
    assert_float_close(feats.grad.cpu().numpy(), want, "segment_mean knn backward")


def test_bad_token_is_reported_and_skipped():
    sizes = [100, 100]
    offsets, tok, counts = _random_labels(80, sizes, 8, unassigned=0.0)
    tok[150] = 8  # outside 0..K-1: the kernel's own range check skips it
    G = np.ones((2, 8, 2), np.float32)
    nb = fps.load_library().segment_pool_backward_workspace_bytes(200, 2, 8, 2, _lib.FPS_ASSIGN_VORONOI)
    ws = torch.empty(max(nb, 256), dtype=torch.uint8, device="cuda")
    got = fps.segment_pool_backward(_dev(G), _dev(counts), 200, offsets=_dev(offsets), token_id=_dev(tok),
                                    workspace=ws)
    with pytest.raises(_lib.FpsError):
        fps.device_status(ws)
    got = got.cpu().numpy()
    assert np.all(got[150] == 0)
    ok = np.arange(200) != 150
    tok[150] = -1
    want = oracle.pool_voronoi_backward(G, offsets, tok, counts)
    np.testing.assert_array_equal(got[ok], want[ok])
