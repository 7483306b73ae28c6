"""The multiply-high divisions the side kernels use instead of integer division.

The pool backward, the kNN backward and the token summaries take q = e / d as
(e * ceil(2^32 / d)) >> 32 for a runtime divisor d >= 2 (F features, k
neighbours, G feature groups).  With m = ceil(2^32 / d) and delta = m*d - 2^32
(0 <= delta < d) the error of e*m / 2^32 against e / d is e*delta / (d*2^32),
which stays below 1/d (so the floor is unchanged) whenever e*delta < 2^32.
These tests check the identity exhaustively over the ranges the kernels use
and the bound for the larger ones.
"""
import numpy as np
import pytest


def mulhi_div(e, d):
    m = ((1 << 32) + d - 1) // d
    return (e.astype(np.uint64) * np.uint64(m)) >> np.uint64(32)


@pytest.mark.parametrize("d", range(2, 65))
def test_tile_element_division(d):
    """Voronoi gather: e < 1024 * F, F <= 64."""
    e = np.arange(1024 * d, dtype=np.uint64)
    assert np.array_equal(mulhi_div(e, d), e // np.uint64(d))


def test_knn_row_division():
    """kNN backward: entry e of K*k <= 2^15 entries, row e / k, k <= 128."""
    e = np.arange(1 << 15, dtype=np.uint64)
    for k in range(2, 129):
        assert np.array_equal(mulhi_div(e, k), e // np.uint64(k)), k


def test_bound_covers_the_shared_buffers():
    """Indices divided by F or by the feature-group count G (both <= 64) stay
    below 2^21 in the kernels; the bound holds to 2^26.  (The divisor k <= 128
    only divides entries below 2^15, covered exhaustively above.)"""
    for d in range(2, 65):
        m = ((1 << 32) + d - 1) // d
        delta = m * d - (1 << 32)
        assert 0 <= delta < d
        assert ((1 << 26) - 1) * delta < (1 << 32)
    rng = np.random.default_rng(0)
    e = rng.integers(0, 1 << 26, 200000).astype(np.uint64)
    for d in (2, 3, 7, 8, 9, 63, 64):
        assert np.array_equal(mulhi_div(e, d), e // np.uint64(d))
