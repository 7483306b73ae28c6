"""Parity of the charge-weighted token summaries (C ``fps_token_summaries``)
with the oracle.  The float64 sums meet in an order the tiles and atomics
choose, so the float outputs are compared within the float tolerance (1e-5
relative, 1e-6 absolute floor); a zero total charge (empty cell) is exact."""
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


def _check(b, K, tok, charge_col):
    want = oracle.token_summaries(b.coords, b.feats, b.offsets, K, tok, charge_col=charge_col)
    got = fps.token_summaries(_dev(b.coords), _dev(b.feats), _dev(b.offsets), K, _dev(tok), charge_col=charge_col)
    for name, g, w in zip(("wsum", "wcoords", "wfeats"), got, want):
        g = g.cpu().numpy()
        assert_float_close(g, w, f"token_summaries {name} (charge_col={charge_col})")
        assert np.array_equal(g == 0, w == 0) or name != "wsum"


@pytest.mark.parametrize("charge_col", [-1, 0])
def test_summaries_tokenizer_labels(charge_col):
    for name in ("c1", "c4"):
        b = workloads.make_workload(name)
        ora = oracle.tokenize_batch(b)
        _check(b, b.K, ora["token_id"], charge_col)


def test_summaries_large_events():
    """The large-event workload's sizes (8 events of 50k-200k points) with
    seeded random labels: every tile adds into the same few accumulators."""
    b = workloads.make_workload("c3")
    rng = np.random.default_rng(110)
    tok = rng.integers(-1, b.K, b.coords.shape[0]).astype(np.int32)
    _check(b, b.K, tok, 0)


@pytest.mark.parametrize("F", [1, 6, 7])
def test_summaries_many_tiny_events(F):
    """Events of 0-6 points: every CTA's range holds hundreds of whole events
    (summed one event at a time and written directly), and the events cut by
    a range boundary are finished from the partial sums."""
    rng = np.random.default_rng(111 + F)
    sizes = rng.integers(0, 7, 5000)
    b = workloads.random_batch(112 + F, sizes, 4, F=F)
    tok = np.concatenate([rng.integers(-1, 4, int(n)) for n in sizes]).astype(np.int32)
    _check(b, 4, tok, 0 if F > 1 else -1)


@pytest.mark.parametrize("F", [9, 12, 64])
def test_summaries_wide_rows(F):
    """More than 8 features: the rows are read from global memory per value
    group instead of being staged, in groups of 8 features per thread."""
    rng = np.random.default_rng(120 + F)
    b = workloads.random_batch(121 + F, [0, 3, 700, 1024, 1025, 5000, 20000, 1], 16, F=F)
    tok = np.concatenate([rng.integers(-1, 16, int(n)) for n in b.sizes()]).astype(np.int32)
    _check(b, 16, tok, 0)
    _check(b, 16, tok, -1)


def test_summaries_mixed_sizes():
    b = workloads.random_batch(113, [0, 1, 100, 1023, 1024, 1025, 5000, 3, 0, 40000], 32, F=5)
    ora = oracle.tokenize(b.coords, b.feats, b.offsets, 32)
    _check(b, 32, ora["token_id"], 0)
    _check(b, 32, ora["token_id"], -1)


def test_summaries_bad_token_is_reported():
    b = workloads.random_batch(114, [50, 60], 8, F=3)
    tok = np.zeros(110, np.int32)
    tok[7] = 8
    nb = fps.load_library().fps_token_summaries_workspace_bytes(2, 8, 3)
    ws = torch.empty(max(nb, 256), dtype=torch.uint8, device="cuda")
    fps.token_summaries(_dev(b.coords), _dev(b.feats), _dev(b.offsets), 8, _dev(tok), charge_col=0, workspace=ws)
    with pytest.raises(_lib.FpsError):
        fps.device_status(ws)
