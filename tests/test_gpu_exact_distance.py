"""Exact float32 distance arithmetic on every GPU path.

The distance is ((dx*dx + dy*dy) + dz*dz) + dt*dt with every operation
rounded to nearest on its own (Neptune README, "How it works", step 1: FPS
over the 4D (x, y, z, t) pulses; the fixed order and the absence of fused
multiply-adds are this implementation's reading).  For offsets (a, b, z, t)
and (b, a, z, t) from the same point the two distances are exactly equal,
because a float32 sum of two terms does not depend on their order, whereas a
multiply fused into that sum rounds differently for the two orders in a good
fraction of cases.  Ties resolve to the lowest index or slot, so any fused
evaluation shows up as a different index than the oracle's.
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
from parity import compare, run_gpu  # noqa: E402


def _offsets(rng, m):
    a, b, z, t = (rng.normal(0, 150, m).astype(np.float32) for _ in range(4))
    return np.stack([a, b, z, t], 1), np.stack([b, a, z, t], 1)


def _swap_tie_batch(seed, m=600):
    """m events [origin, o1, o2] with o2 the x/y swap of o1: d(o1) == d(o2)."""
    rng = np.random.default_rng(seed)
    o1, o2 = _offsets(rng, m)
    coords = np.zeros((3 * m, 4), np.float32)
    coords[1::3] = o1
    coords[2::3] = o2
    b = workloads.random_batch(seed, [3] * m, 2)
    b.coords[:] = coords
    return b


@pytest.mark.parametrize("force", [-1, 0, 1, 2, 3, 4])
def test_fps_ties_under_swapped_offsets(force):
    b = _swap_tie_batch(900)
    ora = oracle.tokenize_batch(b)
    # the oracle's tie rule: the second centroid is the lower of the two tied points
    np.testing.assert_array_equal(ora["centroid_idx"][:, 1], b.offsets[:-1] + 1)
    compare(b, run_gpu(b, force_schedule=force), ora)


def test_fps_ties_in_both_lanes():
    """The tied pair sits in the second packed slot of the warp schedule too."""
    rng = np.random.default_rng(901)
    m = 300
    o1, o2 = _offsets(rng, m)
    n = 70  # points 0..69: origin at 0, filler far below, tied pair at 33 and 66
    coords = np.zeros((m * n, 4), np.float32)
    for e in range(m):
        ev = coords[e * n:(e + 1) * n]
        ev[1:] = rng.normal(0, 1e-3, (n - 1, 4))
        ev[33] = o1[e]
        ev[66] = o2[e]
    b = workloads.random_batch(901, [n] * m, 2)
    b.coords[:] = coords
    ora = oracle.tokenize_batch(b)
    np.testing.assert_array_equal(ora["centroid_idx"][:, 1], b.offsets[:-1] + 33)
    compare(b, run_gpu(b), ora)


def test_nearest_centroid_ties_under_swapped_offsets():
    """fps_assign (the search Lloyd refinement also uses) with tied centroid
    pairs at slots (1, 2) and (3, 4) of K = 5 (odd: one padded slot)."""
    rng = np.random.default_rng(902)
    m, K = 2000, 5
    o1, o2 = _offsets(rng, m)
    p1, p2 = _offsets(rng, m)
    cent = np.zeros((m, K, 4), np.float32)
    cent[:, 0] = 1e6  # far away
    cent[:, 1], cent[:, 2] = o1, o2
    cent[:, 3], cent[:, 4] = p1, p2
    near34 = np.array([oracle.dist(np.zeros(4, np.float32), p1[e]) < oracle.dist(np.zeros(4, np.float32), o1[e])
                       for e in range(m)])
    coords = np.zeros((m, 4), np.float32)  # one point per event, at the origin
    offsets = np.arange(m + 1, dtype=np.int64)
    want = oracle.assign(coords, offsets, cent, K, valid=np.full(m, K, np.int32))
    np.testing.assert_array_equal(want, np.where(near34, 3, 1))
    got = fps.fps_assign(torch.from_numpy(coords).cuda(), torch.from_numpy(offsets).cuda(),
                         torch.from_numpy(cent).cuda(), torch.full((m,), K, dtype=torch.int32, device="cuda"))
    np.testing.assert_array_equal(got.cpu().numpy(), want)
