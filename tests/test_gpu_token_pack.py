"""Parity of the packed token layout (C ``fps_pack_tokens`` / ``fps_unpack_tokens``)
with the oracle: a copy and a scan, so every output is compared bit for bit."""
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


def _dev(a):
    return torch.from_numpy(np.ascontiguousarray(a)).cuda()


def _check(src, offsets=None, valid=None):
    want = oracle.pack_tokens(src, offsets=offsets, valid=valid)
    got = fps.pack_tokens(_dev(src), offsets=None if offsets is None else _dev(offsets),
                          valid_tokens=None if valid is None else _dev(valid))
    for g, w in zip(got, want):
        np.testing.assert_array_equal(g.cpu().numpy(), w)
    K = src.shape[1]
    back = fps.unpack_tokens(got[0], got[2], K).cpu().numpy()
    np.testing.assert_array_equal(back, oracle.unpack_tokens(want[0], want[2], K))


@pytest.mark.parametrize("D", [1, 4, 6, 33])
def test_pack_random_sizes(D):
    rng = np.random.default_rng(100 + D)
    sizes = np.concatenate([[0, 1, 16, 17], rng.integers(0, 60, 3000)])  # > one 1024-event scan tile
    offsets = np.concatenate([[0], np.cumsum(sizes)]).astype(np.int64)
    src = rng.normal(0, 1, (len(sizes), 16, D)).astype(np.float32)
    _check(src, offsets=offsets)
    _check(src, valid=rng.integers(0, 17, len(sizes)).astype(np.int32))


def test_pack_tokenizer_output():
    """The tokenizer's pooled rows and centroids of the small-event workload
    (4096 events, K = 128), tokens from the oracle."""
    b = workloads.make_workload("c4")
    ora = oracle.tokenize_batch(b)
    _check(ora["pooled"], offsets=b.offsets)
    _check(ora["centroids"], offsets=b.offsets)


def test_pack_edge_cases():
    _check(np.ones((1, 1, 1), np.float32), offsets=np.array([0, 5]))
    _check(np.ones((3, 4, 2), np.float32), offsets=np.array([0, 0, 0, 0]))  # no tokens at all
    _check(np.arange(24, dtype=np.float32).reshape(2, 4, 3), valid=np.array([4, 0], np.int32))


def test_pack_bad_count_is_reported():
    src = np.ones((2, 4, 2), np.float32)
    nb = fps.load_library().fps_pack_workspace_bytes()
    ws = torch.empty(max(nb, 256), dtype=torch.uint8, device="cuda")
    dst, doc, tok = fps.pack_tokens(_dev(src), valid_tokens=_dev(np.array([2, 9], np.int32)), workspace=ws)
    with pytest.raises(_lib.FpsError):
        fps.device_status(ws)
    assert tok.cpu().tolist() == [0, 2, 6]  # the count above K is clamped to K
