"""Parity of the random FPS start points (C ``fps_random_starts``, Philox4x32-10
on the device) with the oracle's generator, bit for bit, and of the tokenizer
run from those starts."""
import numpy as np
import pytest

import oracle
import workloads

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

if not torch.cuda.is_available():  # pragma: no cover - the gpu marker is deselected on CPU hosts
    pytest.skip("needs a CUDA device", allow_module_level=True)

import farthest_point_sampling_b200 as fps  # noqa: E402
from parity import compare, run_gpu  # noqa: E402


@pytest.mark.parametrize("seed,stream", [(0, 0), (1, 0), (0x123456789ABCDEF, 7), (2**64 - 1, 2**32 - 1)])
def test_random_starts_match_oracle(seed, stream):
    rng = np.random.default_rng(130)
    sizes = np.concatenate([[0, 1, 2, 3, 2**20], rng.integers(0, 100000, 3000)])
    offsets = np.concatenate([[0], np.cumsum(sizes)]).astype(np.int64)
    got = fps.random_starts(torch.from_numpy(offsets).cuda(), seed, stream).cpu().numpy()
    np.testing.assert_array_equal(got, oracle.random_starts(offsets, seed, stream))


def test_tokenizer_from_random_starts():
    b = workloads.make_workload("c1")
    starts = oracle.random_starts(b.offsets, 42, 3)
    b.start_local = starts
    ora = oracle.tokenize_batch(b)
    got = fps.fps_tokenize(torch.from_numpy(b.coords).cuda(), torch.from_numpy(b.feats).cuda(),
                           torch.from_numpy(b.offsets).cuda(), K=b.K, random_start=True, seed=42, stream_id=3)
    compare(b, {k: v.cpu().numpy() for k, v in got.items()}, ora)
