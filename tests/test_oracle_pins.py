"""Pins for the CPU oracle: hand-worked fixtures, brute force, closed forms, invariants.

None of these compare the oracle with itself or with the CUDA path.  The
``pin_*`` functions are also re-run against deliberately broken copies of the
oracle (``test_oracle_mutations.py``) to show each plausible slip is caught.
"""
import os

import numpy as np
import pytest

import bruteforce as bf
import oracle
import workloads

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def read_fps_fixture(name):
    coords, meta, mode = [], {}, None
    with open(os.path.join(GOLDEN, name)) as fh:
        for line in fh:
            line = line.split("#", 1)[0].strip()
            if not line:
                continue
            key, *rest = line.split()
            if key == "coords":
                mode = "coords"
                continue
            if key in ("N", "K", "start", "expected", "sel_dist", "scale", "unscaled_expected"):
                mode = None
                meta[key] = rest
                continue
            if mode == "coords":
                coords.append([float(v) for v in line.split()])
    return (np.array(coords, np.float32), int(meta["K"][0]), int(meta["start"][0]),
            np.array([int(v) for v in meta["expected"]]), np.array([float(v) for v in meta["sel_dist"]],
                                                                    np.float32))


FPS_FIXTURES = ["fps_collinear9.txt", "fps_hypercube16.txt", "fps_duplicates.txt"]


# ---------------------------------------------------------------- distance

def pin_dist_golden():
    rows = np.loadtxt(os.path.join(GOLDEN, "dist_order.txt"), dtype=np.float64, comments="#")
    for r in rows:
        got = oracle.dist(r[0:4], r[4:8])
        assert got == np.float32(r[8]), (r, got)
        assert oracle.dist(r[4:8], r[0:4]) == got  # a-b = -(b-a) exactly


def pin_dist_error_bound():
    rng = np.random.default_rng(11)
    for _ in range(2000):
        p = (rng.standard_normal(4) * rng.choice([1e-3, 1.0, 100.0, 5000.0], 4)).astype(np.float32)
        c = (rng.standard_normal(4) * rng.choice([1e-3, 1.0, 100.0, 5000.0], 4)).astype(np.float32)
        exact = float(np.sum((p.astype(np.float64) - c.astype(np.float64)) ** 2))
        got = float(oracle.dist(p, c))
        # 4 subtractions, 4 products, 3 sums: relative error below 8 units of 2^-24
        assert abs(got - exact) <= 8 * 2.0 ** -24 * exact + 1e-30, (p, c, got, exact)


def test_dist_golden():
    pin_dist_golden()


def test_dist_error_bound():
    pin_dist_error_bound()


# ---------------------------------------------------------------- FPS

def pin_fps_fixtures():
    for name in FPS_FIXTURES:
        pts, K, start, expected, seld = read_fps_fixture(name)
        idx, sd = oracle.fps(pts, [0, len(pts)], K, start_local=[start], with_sel_dist=True)
        assert idx[0].tolist() == expected.tolist(), (name, idx[0])
        assert np.array_equal(sd[0], seld), (name, sd[0])


def _tiny_batches():
    for seed in range(60):
        rng = np.random.default_rng(1000 + seed)
        K = int(rng.integers(1, 17))
        sizes = rng.integers(0, 65, int(rng.integers(1, 6)))
        kw = {}
        if seed % 3 == 1:
            kw["dup_frac"] = 0.4
        if seed % 3 == 2:
            kw["grid"] = 50.0
        b = workloads.random_batch(seed, sizes, K, **kw)
        starts = np.array([rng.integers(0, max(int(n), 1)) for n in sizes], np.int32)
        yield b, K, starts


def pin_fps_bruteforce():
    for b, K, starts in _tiny_batches():
        got = oracle.fps(b.coords, b.offsets, K, start_local=starts)
        want = bf.fps(b.coords, b.offsets, K, start_local=starts)
        assert np.array_equal(got, want), (b.sizes(), K)


def pin_fps_invariants():
    for b, K, starts in _tiny_batches():
        idx, sd = oracle.fps(b.coords, b.offsets, K, start_local=starts, with_sel_dist=True)
        for e in range(b.B):
            o0, o1 = b.offsets[e], b.offsets[e + 1]
            n = o1 - o0
            row = idx[e]
            valid = row[row >= 0]
            assert len(valid) == min(n, K)
            assert np.all(row[len(valid):] == -1)
            assert len(set(valid.tolist())) == len(valid)  # distinct
            assert np.all((valid >= o0) & (valid < o1))  # inside the event
            if n <= K:
                assert np.array_equal(valid, np.arange(o0, o1))  # one token per pulse
            else:
                assert valid[0] == o0 + starts[e]
                s = sd[e, 1:]
                assert np.all(np.diff(s) <= 0)  # selection distance never grows


def test_fps_fixtures():
    pin_fps_fixtures()


def test_fps_bruteforce():
    pin_fps_bruteforce()


def test_fps_invariants():
    pin_fps_invariants()


def test_fps_time_shift_invariance():
    # t on a 2^-8 ns grid, |t| < 2^15 before and after the shift: every shifted
    # value is exact in f32, so each difference (and distance) is unchanged.
    rng = np.random.default_rng(5)
    sizes = [300, 129, 1000]
    b = workloads.random_batch(5, sizes, 64)
    t = np.round(rng.uniform(0, 2 ** 14, b.P) * 256) / 256
    b.coords[:, 3] = t.astype(np.float32)
    base = oracle.fps(b.coords, b.offsets, 64)
    for shift in (1024.0, -8192.25, 12345.5):
        c2 = b.coords.copy()
        c2[:, 3] = (t + shift).astype(np.float32)
        assert np.array_equal((c2[:, 3].astype(np.float64) - shift), t)  # shift exact
        assert np.array_equal(oracle.fps(c2, b.offsets, 64), base)


def test_fps_edge_cases():
    pts = np.random.default_rng(0).standard_normal((10, 4)).astype(np.float32)
    # empty batch, empty event, N=1, N=K, N=K+1, K=1
    assert oracle.fps(np.zeros((0, 4)), [0], 4).shape == (0, 4)
    idx = oracle.fps(pts[:0], [0, 0], 4)
    assert idx.tolist() == [[-1, -1, -1, -1]]
    assert oracle.fps(pts[:1], [0, 1], 4).tolist() == [[0, -1, -1, -1]]
    assert oracle.fps(pts[:4], [0, 4], 4).tolist() == [[0, 1, 2, 3]]
    row = oracle.fps(pts[:5], [0, 5], 4)[0]
    assert row[0] == 0 and len(set(row.tolist())) == 4
    assert oracle.fps(pts, [0, 10], 1, start_local=[7]).tolist() == [[7]]
    with pytest.raises(ValueError):
        oracle.fps(pts, [0, 10], 4, start_local=[10])
    with pytest.raises(ValueError):
        oracle.fps(pts, [0, 6, 5], 4)


# ---------------------------------------------------------------- assign

def _centroids(b, idx):
    return np.where(idx[..., None] >= 0, b.coords[np.maximum(idx, 0)], 0).astype(np.float32)


def pin_assign_bruteforce():
    for b, K, starts in _tiny_batches():
        idx = bf.fps(b.coords, b.offsets, K, start_local=starts)
        cents = _centroids(b, idx)
        valid = np.minimum(b.sizes(), K).astype(np.int32)
        got = oracle.assign(b.coords, b.offsets, cents, K, valid=valid)
        want = bf.assign(b.coords, b.offsets, cents, valid)
        assert np.array_equal(got, want)


def test_assign_bruteforce():
    pin_assign_bruteforce()


def test_assign_invariants():
    b = workloads.make_workload("c0")
    idx = oracle.fps(b.coords, b.offsets, b.K)
    cents = _centroids(b, idx)
    tok = oracle.assign(b.coords, b.offsets, cents, b.K)
    for e in range(b.B):
        o0, o1 = b.offsets[e], b.offsets[e + 1]
        # every centroid lands in its own cell (c0 has no duplicate points)
        assert np.array_equal(tok[idx[e]], np.arange(b.K))
        counts = np.bincount(tok[o0:o1], minlength=b.K)
        assert counts.sum() == o1 - o0
        # the label's distance is the minimum over all centroids
        D = bf.pair_dist(b.coords[o0:o1], cents[e])
        assert np.array_equal(D[np.arange(o1 - o0), tok[o0:o1]], D.min(1))


# ---------------------------------------------------------------- kNN

def pin_knn_bruteforce():
    for b, K, starts in _tiny_batches():
        idx = bf.fps(b.coords, b.offsets, K, start_local=starts)
        cents = _centroids(b, idx)
        valid = np.minimum(b.sizes(), K).astype(np.int32)
        for k in (1, 3, 8):
            got = oracle.knn(b.coords, b.offsets, cents, K, k, valid=valid)
            want = bf.knn(b.coords, b.offsets, cents, valid, k)
            assert np.array_equal(got, want)


def test_knn_bruteforce():
    pin_knn_bruteforce()


def test_knn_row0_is_centroid():
    b = workloads.make_workload("c0")
    idx = oracle.fps(b.coords, b.offsets, b.K)
    got = oracle.knn(b.coords, b.offsets, _centroids(b, idx), b.K, 5)
    assert np.array_equal(got[:, :, 0], idx)


# ---------------------------------------------------------------- pool

def pin_pool_bruteforce():
    for b, K, starts in _tiny_batches():
        idx = bf.fps(b.coords, b.offsets, K, start_local=starts)
        cents = _centroids(b, idx)
        valid = np.minimum(b.sizes(), K).astype(np.int32)
        tok = bf.assign(b.coords, b.offsets, cents, valid)
        pooled, counts = oracle.pool_voronoi(b.feats, b.offsets, K, tok)
        wp, wc = bf.pool_voronoi(b.feats, b.offsets, K, tok)
        assert np.array_equal(counts, wc)
        np.testing.assert_allclose(pooled, wp, rtol=1e-6, atol=1e-7)


def test_pool_bruteforce():
    pin_pool_bruteforce()


def test_pool_closed_forms():
    rng = np.random.default_rng(3)
    offsets = np.array([0, 50, 50, 130])
    tok = np.concatenate([rng.integers(0, 4, 50), rng.integers(0, 4, 80)]).astype(np.int32)
    # constant features pool to the constant
    f = np.full((130, 3), 2.5, np.float32)
    pooled, counts = oracle.pool_voronoi(f, offsets, 4, tok)
    assert np.all(pooled[counts > 0] == 2.5) and np.all(pooled[counts == 0] == 0)
    assert counts[0].sum() == 50 and counts[1].sum() == 0 and counts[2].sum() == 80
    # one-hot of a 2-valued feature pools to the fraction of each value
    v = rng.integers(0, 2, 130)
    f = np.stack([v == 0, v == 1], 1).astype(np.float32)
    pooled, counts = oracle.pool_voronoi(f, offsets, 4, tok)
    for e, (o0, o1) in enumerate([(0, 50), (50, 50), (50, 130)]):
        for j in range(4):
            m = tok[o0:o1] == j
            if m.any():
                assert pooled[e, j, 1] == np.float32(v[o0:o1][m].sum() / m.sum())
    # kNN pool: counts are the number of valid entries
    knn_idx = np.array([[[0, 1, -1], [2, -1, -1]]], np.int32)
    f = np.arange(12, dtype=np.float32).reshape(4, 3)
    pooled, counts = oracle.pool_knn(f, knn_idx)
    assert counts.tolist() == [[2, 1]]
    assert pooled[0, 0].tolist() == [1.5, 2.5, 3.5] and pooled[0, 1].tolist() == [6, 7, 8]


# ---------------------------------------------------------------- Lloyd

# ---------------------------------------------------------------- pool backward
#
# The pool is linear in the features, so its vector-Jacobian product G -> dX is
# its transpose: <G, pool(X)> = <dX, X> for every X and G (the adjoint
# identity).  The forward side uses the numpy brute force, not the oracle.

def _knn_pool_np(feats, knn_idx):
    B, K, k = knn_idx.shape
    out = np.zeros((B, K, feats.shape[1]))
    for b in range(B):
        for j in range(K):
            rows = [i for i in knn_idx[b, j] if i >= 0]
            if rows:
                out[b, j] = feats[rows].astype(np.float64).mean(0)
    return out


def _backward_cases():
    for b, K, starts in list(_tiny_batches())[:24]:
        idx = bf.fps(b.coords, b.offsets, K, start_local=starts)
        cents = _centroids(b, idx)
        valid = np.minimum(b.sizes(), K).astype(np.int32)
        tok = bf.assign(b.coords, b.offsets, cents, valid)
        yield b, K, valid, cents, tok


def pin_pool_backward_adjoint():
    rng = np.random.default_rng(77)
    for b, K, valid, cents, tok in _backward_cases():
        B, F = len(b.offsets) - 1, b.feats.shape[1]
        G = rng.normal(0, 1, (B, K, F)).astype(np.float32)
        X = rng.normal(0, 1, b.feats.shape).astype(np.float32)
        # Voronoi
        wp, wc = bf.pool_voronoi(X, b.offsets, K, tok)
        dX = oracle.pool_voronoi_backward(G, b.offsets, tok, wc)
        lhs = float((G.astype(np.float64) * wp).sum())
        rhs = float((dX.astype(np.float64) * X).sum())
        scale = float(np.abs(G).sum() * np.abs(X).max()) + 1e-30
        assert abs(lhs - rhs) <= 1e-6 * scale, (lhs, rhs)
        # a point outside every cell gets no gradient
        assert np.all(dX[tok < 0] == 0)
        # kNN
        k = 3
        knn_idx = bf.knn(b.coords, b.offsets, cents, valid, k)
        kp = _knn_pool_np(X, knn_idx)
        kc = (knn_idx >= 0).sum(2).astype(np.int32)
        dX = oracle.pool_knn_backward(G, knn_idx, kc, X.shape[0])
        lhs = float((G.astype(np.float64) * kp).sum())
        rhs = float((dX.astype(np.float64) * X).sum())
        assert abs(lhs - rhs) <= 1e-6 * scale, (lhs, rhs)


def test_pool_backward_adjoint():
    pin_pool_backward_adjoint()


def test_pool_backward_autograd():
    """Reverse-mode autograd of a float64 torch scatter-mean, elementwise."""
    torch = pytest.importorskip("torch")
    rng = np.random.default_rng(78)
    for b, K, valid, cents, tok in list(_backward_cases())[:10]:
        B, F = len(b.offsets) - 1, b.feats.shape[1]
        G = rng.normal(0, 1, (B, K, F)).astype(np.float32)
        ev = np.repeat(np.arange(B), np.diff(b.offsets))
        X = torch.tensor(b.feats, dtype=torch.float64, requires_grad=True)
        keep = torch.from_numpy(tok >= 0)
        cell = torch.from_numpy(ev * K + np.maximum(tok, 0)).long()
        sums = torch.zeros(B * K, F, dtype=torch.float64).index_add(0, cell[keep], X[keep])
        cnt = torch.zeros(B * K, dtype=torch.float64).index_add(0, cell[keep], torch.ones(int(keep.sum()),
                                                                                            dtype=torch.float64))
        pooled = sums / cnt.clamp(min=1).unsqueeze(1)
        (pooled * torch.from_numpy(G.reshape(B * K, F)).double()).sum().backward()
        want = X.grad.numpy().astype(np.float32)
        got = oracle.pool_voronoi_backward(G, b.offsets, tok, cnt.numpy().astype(np.int32).reshape(B, K))
        np.testing.assert_array_equal(got, want)

        knn_idx = bf.knn(b.coords, b.offsets, cents, valid, 4)
        X.grad = None
        flat = torch.from_numpy(knn_idx.reshape(B * K, 4)).long()
        m = (flat >= 0).double()
        rows = X[flat.clamp(min=0)] * m.unsqueeze(2)
        kc = m.sum(1)
        pooled = rows.sum(1) / kc.clamp(min=1).unsqueeze(1)
        (pooled * torch.from_numpy(G.reshape(B * K, F)).double()).sum().backward()
        want = X.grad.numpy()
        got = oracle.pool_knn_backward(G, knn_idx, kc.numpy().astype(np.int32).reshape(B, K), X.shape[0])
        np.testing.assert_allclose(got, want, rtol=1e-6, atol=1e-7)


def test_pool_backward_closed_forms():
    # G = 1 on every row: each assigned point gets 1 / (size of its cell), and
    # the gradients of one cell sum to 1 per feature
    offsets = np.array([0, 5, 5, 9])
    tok = np.array([0, 0, 1, 0, -1, 2, 2, 2, 0], np.int32)
    counts = np.array([[3, 1, 0], [0, 0, 0], [1, 0, 3]], np.int32)
    G = np.ones((3, 3, 2), np.float32)
    dX = oracle.pool_voronoi_backward(G, offsets, tok, counts)
    np.testing.assert_array_equal(dX[:, 0], np.float32([1 / 3, 1 / 3, 1, 1 / 3, 0, 1 / 3, 1 / 3, 1 / 3, 1]))
    # kNN: a point gathered by two rows sums both rows' shares
    knn_idx = np.array([[[0, 1], [1, -1]]], np.int32)
    dX = oracle.pool_knn_backward(np.float32([[[2, 0], [3, 1]]]), knn_idx, np.int32([[2, 1]]), 3)
    assert dX.tolist() == [[1, 0], [4, 1], [0, 0]]


# ---------------------------------------------------------------- random starts
#
# Known-answer vectors of Philox4x32-10 as published with the generator
# (Salmon et al., SC 2011, and its reference distribution): counter, key,
# expected output.
PHILOX_KAT = [
    ([0, 0, 0, 0], [0, 0], [0x6627e8d5, 0xe169c58d, 0xbc57ac4c, 0x9b00dbd8]),
    ([0xffffffff] * 4, [0xffffffff] * 2, [0x408f276d, 0x41c83b0e, 0xa20bc7c6, 0x6d5451fd]),
    ([0x243f6a88, 0x85a308d3, 0x13198a2e, 0x03707344], [0xa4093822, 0x299f31d0],
     [0xd16cfe09, 0x94fdcceb, 0x5001e420, 0x24126ea1]),
]


def pin_random_starts():
    for ctr, key, want in PHILOX_KAT:
        assert oracle.philox4x32_10(ctr, key).tolist() == want
    rng = np.random.default_rng(120)
    sizes = np.concatenate([[0, 1, 2, 3], rng.integers(1, 5000, 4000)])
    offsets = np.concatenate([[0], np.cumsum(sizes)])
    st = oracle.random_starts(offsets, seed=0x123456789ABCDEF, stream=7)
    # the multiply-shift of the first Philox word, recomputed in Python integers
    for b in range(6):
        u = int(oracle.philox4x32_10([b, 7, 0, 0], [0x89ABCDEF, 0x1234567])[0])
        assert st[b] == (u * int(sizes[b])) >> 32
    assert np.all((st >= 0) & ((st < sizes) | (sizes == 0)))
    # roughly uniform: the start's position within its event
    frac = st[sizes > 100] / sizes[sizes > 100]
    hist = np.histogram(frac, bins=10, range=(0, 1))[0]
    assert hist.min() > 0.7 * hist.mean()
    # another seed or stream gives other starts
    assert not np.array_equal(st, oracle.random_starts(offsets, seed=1, stream=7))
    assert not np.array_equal(st, oracle.random_starts(offsets, seed=0x123456789ABCDEF, stream=8))


def test_random_starts():
    pin_random_starts()


# ---------------------------------------------------------------- token summaries

def pin_token_summaries():
    for b, K, valid, cents, tok in list(_backward_cases())[:16]:
        B = len(b.offsets) - 1
        ev = np.repeat(np.arange(B), np.diff(b.offsets))
        # unit charge: the total is the count, the means the plain means
        wsum, wc, wf = oracle.token_summaries(b.coords, b.feats, b.offsets, K, tok, charge_col=-1)
        pooled, counts = bf.pool_voronoi(b.feats, b.offsets, K, tok)
        assert np.array_equal(wsum, counts.astype(np.float32))
        np.testing.assert_allclose(wf, pooled, rtol=1e-6, atol=1e-7)
        cm, _ = bf.pool_voronoi(b.coords, b.offsets, K, tok)
        np.testing.assert_allclose(wc, cm, rtol=1e-6, atol=1e-5)
        # charge column 0: numpy's weighted average per cell
        wsum, wc, wf = oracle.token_summaries(b.coords, b.feats, b.offsets, K, tok, charge_col=0)
        q = b.feats[:, 0].astype(np.float64)
        for e in range(B):
            for j in range(K):
                m = (ev == e) & (tok == j)
                W = q[m].sum()
                assert np.isclose(wsum[e, j], W, rtol=1e-6, atol=1e-7)
                if m.any() and W > 0:
                    np.testing.assert_allclose(wc[e, j], np.average(b.coords[m].astype(np.float64), 0, q[m]),
                                               rtol=1e-6, atol=1e-5)
                    np.testing.assert_allclose(wf[e, j], np.average(b.feats[m].astype(np.float64), 0, q[m]),
                                               rtol=1e-5, atol=1e-6)
                else:
                    assert not wc[e, j].any() and not wf[e, j].any()


def test_token_summaries():
    pin_token_summaries()


# ---------------------------------------------------------------- packed tokens

def pin_pack_tokens():
    rng = np.random.default_rng(90)
    for b, K, starts in list(_tiny_batches())[:30]:
        B = len(b.offsets) - 1
        D = int(rng.integers(1, 6))
        src = rng.normal(0, 1, (B, K, D)).astype(np.float32)
        n = np.diff(b.offsets)
        v = np.minimum(n, K)
        dst, doc, tok = oracle.pack_tokens(src, offsets=b.offsets)
        # closed forms: the packed length, the scan, the event ids
        assert dst.shape == (v.sum(), D)
        assert np.array_equal(tok, np.concatenate([[0], np.cumsum(v)]))
        assert np.array_equal(doc, np.repeat(np.arange(B), v))
        # numpy's boolean-mask gather of the same rows, in row-major order
        mask = np.arange(K)[None, :] < v[:, None]
        assert np.array_equal(dst, src[mask])
        # unpack inverts it and zeroes the padding
        back = oracle.unpack_tokens(dst, tok, K)
        assert np.array_equal(back, np.where(mask[:, :, None], src, 0))
        # caller-given counts
        vv = rng.integers(0, K + 1, B).astype(np.int32)
        dst, doc, tok = oracle.pack_tokens(src, valid=vv)
        mask = np.arange(K)[None, :] < vv[:, None]
        assert np.array_equal(dst, src[mask]) and np.array_equal(doc, np.repeat(np.arange(B), vv))


def test_pack_tokens():
    pin_pack_tokens()


def pin_lloyd_closed_form():
    rng = np.random.default_rng(7)
    n, K = 40, 3
    pts = (rng.standard_normal((n, 4)) * [100, 100, 100, 1000]).astype(np.float32)
    q = rng.lognormal(0, 1, n).astype(np.float32)
    feats = np.stack([q, rng.standard_normal(n).astype(np.float32)], 1)
    lab = rng.integers(0, K, n).astype(np.int32)
    cents = pts[[0, 1, 2]].copy()
    got_c, got_t = oracle.lloyd(pts, feats, [0, n], K, 1, cents[None], lab, charge_col=0)
    want_c = bf.lloyd_update(pts, q, lab, cents)
    np.testing.assert_allclose(got_c[0], want_c, rtol=2e-7, atol=0)
    # the re-assignment is the all-pairs nearest centroid of the new centroids
    assert np.array_equal(got_t, bf.assign(pts, [0, n], got_c, [K]))
    # unit charge (charge_col = -1) gives the plain mean of each cell
    got_c, _ = oracle.lloyd(pts, feats, [0, n], K, 1, cents[None], lab, charge_col=-1)
    for j in range(K):
        np.testing.assert_allclose(got_c[0, j], pts[lab == j].astype(np.float64).mean(0), rtol=2e-7)


def test_lloyd_closed_form():
    pin_lloyd_closed_form()


def test_lloyd_keeps_empty_and_nonpositive_cells():
    rng = np.random.default_rng(8)
    n, K = 12, 4
    pts = rng.standard_normal((n, 4)).astype(np.float32)
    q = np.ones(n, np.float32)
    q[lab_neg := np.arange(4, 8)] = -1.0  # cell 1 has weight -4
    lab = np.array([0] * 4 + [1] * 4 + [2] * 4, np.int32)  # cell 3 empty
    cents = (np.arange(16, dtype=np.float32).reshape(4, 4) * 10)
    got_c, _ = oracle.lloyd(pts, q[:, None], [0, n], K, 1, cents[None], lab, charge_col=0)
    assert np.array_equal(got_c[0, 1], cents[1]) and np.array_equal(got_c[0, 3], cents[3])
    assert not np.array_equal(got_c[0, 0], cents[0])
    del lab_neg


def test_lloyd_objective_nonincreasing():
    b = workloads.random_batch(21, [600, 900], 16, charge_col=0)
    idx = oracle.fps(b.coords, b.offsets, 16)
    cents = _centroids(b, idx)
    tok = oracle.assign(b.coords, b.offsets, cents, 16)
    q = b.feats[:, 0].astype(np.float64)

    def objective(c, t):
        e = np.repeat(np.arange(b.B), b.sizes())
        diff = b.coords.astype(np.float64) - c[e, t].astype(np.float64)
        return float(np.sum(q * np.sum(diff * diff, 1)))

    prev = objective(cents, tok)
    for _ in range(5):
        cents, tok = oracle.lloyd(b.coords, b.feats, b.offsets, 16, 1, cents, tok, charge_col=0)
        cur = objective(cents, tok)
        assert cur <= prev * (1 + 1e-6)
        prev = cur


def test_lloyd_skips_passthrough_events():
    b = workloads.random_batch(4, [10, 40], 16)
    idx = oracle.fps(b.coords, b.offsets, 16)
    cents = _centroids(b, idx)
    tok = oracle.assign(b.coords, b.offsets, cents, 16)
    c2, t2 = oracle.lloyd(b.coords, b.feats, b.offsets, 16, 2, cents, tok)
    assert np.array_equal(c2[0], cents[0]) and np.array_equal(t2[:10], tok[:10])


# ---------------------------------------------------------------- whole tokenizer

def test_tokenize_composition():
    for mode, k, iters in ((0, 0, 0), (1, 4, 0), (0, 0, 2), (1, 6, 1)):
        b = workloads.random_batch(30 + mode, [0, 5, 16, 17, 90, 200], 16, assign_mode=mode, k=k,
                                   lloyd_iters=iters, charge_col=0)
        out = oracle.tokenize_batch(b)
        idx = bf.fps(b.coords, b.offsets, 16)
        assert np.array_equal(out["centroid_idx"], idx)
        valid = np.minimum(b.sizes(), 16)
        tok = out["token_id"]
        for e in range(b.B):
            o0, o1 = b.offsets[e], b.offsets[e + 1]
            n = o1 - o0
            assert np.all(out["centroids"][e, valid[e]:] == 0)
            if n <= 16:  # passthrough: token j is point j, pooled = own features
                assert np.array_equal(tok[o0:o1], np.arange(n))
                assert np.array_equal(out["pooled"][e, :n], b.feats[o0:o1])
                assert np.all(out["counts"][e, :n] == 1) and np.all(out["counts"][e, n:] == 0)
                if mode == 1:
                    assert np.array_equal(out["knn_idx"][e, :n, 0], np.arange(o0, o1))
                    assert np.all(out["knn_idx"][e, :n, 1:] == -1)
        big = b.sizes() > 16
        if iters == 0:
            assert np.array_equal(out["centroids"][big], b.coords[idx[big]])
        want_tok = bf.assign(b.coords, b.offsets, out["centroids"], valid)
        m = np.repeat(big, b.sizes())
        assert np.array_equal(tok[m], want_tok[m])
        if mode == 0:
            assert out["counts"].sum() == b.P
            wp, wc = bf.pool_voronoi(b.feats, b.offsets, 16, tok)
            assert np.array_equal(out["counts"], wc)
            np.testing.assert_allclose(out["pooled"], wp, rtol=1e-6, atol=1e-7)
        else:
            want = bf.knn(b.coords, b.offsets, out["centroids"], valid, k)
            assert np.array_equal(out["knn_idx"][big], want[big])
            assert np.all(out["counts"][big] == min(k, 17))


# ------------------------------------------------------------------ per-axis scale

def _prescaled(coords, w):
    """coords with every coordinate multiplied by its axis weight in float32."""
    return (np.asarray(coords, np.float32) * np.asarray(w, np.float32)[None, :]).astype(np.float32)


def pin_axis_scale():
    """The per-axis scale multiplies both points' coordinates, axis by axis, in
    float32 before the distance; only the metric changes."""
    # hand-worked fixture: the time scale reorders FPS
    path = os.path.join(GOLDEN, "fps_time_scale.txt")
    meta = {}
    coords = []
    with open(path) as fh:
        mode = None
        for line in fh:
            line = line.split("#", 1)[0].strip()
            if not line:
                continue
            key, *rest = line.split()
            if key == "coords":
                mode = "coords"
                continue
            if mode == "coords" and key not in ("expected", "sel_dist", "unscaled_expected"):
                coords.append([float(v) for v in line.split()])
                continue
            mode = None
            meta[key] = rest
    pts = np.array(coords, np.float32)
    K = int(meta["K"][0])
    w = np.array([float(v) for v in meta["scale"]], np.float32)
    idx, sd = oracle.fps(pts, [0, len(pts)], K, start_local=[int(meta["start"][0])], with_sel_dist=True,
                         axis_scale=w)
    assert idx[0].tolist() == [int(v) for v in meta["expected"]]
    assert sd[0].tolist() == [float(v) for v in meta["sel_dist"]]
    assert oracle.fps(pts, [0, len(pts)], K).tolist()[0] == [int(v) for v in meta["unscaled_expected"]]

    # unit scale gives the same bits as no scale, through the whole tokenizer
    for mode, k, it in ((0, 0, 2), (1, 7, 1)):
        b = workloads.random_batch(71 + mode, [3, 40, 200, 513], 32, assign_mode=mode, k=k, lloyd_iters=it,
                                   charge_col=0)
        a = oracle.tokenize_batch(b)
        b.axis_scale = (1.0, 1.0, 1.0, 1.0)
        u = oracle.tokenize_batch(b)
        for key in a:
            if a[key] is not None:
                assert np.array_equal(a[key], u[key]), key

    # any scale: FPS, assignment and kNN equal the unscaled functions on
    # coordinates (and centroids) scaled beforehand in float32
    b = workloads.random_batch(73, [150, 300, 77], 24)
    w = np.array([1.0, 1.0, 1.0, 0.3], np.float32)
    sc = _prescaled(b.coords, w)
    idx = oracle.fps(b.coords, b.offsets, b.K, axis_scale=w)
    assert np.array_equal(idx, oracle.fps(sc, b.offsets, b.K))
    cents = np.where(idx[..., None] >= 0, b.coords[np.maximum(idx, 0)], 0).astype(np.float32)
    tok = oracle.assign(b.coords, b.offsets, cents, b.K, axis_scale=w)
    assert np.array_equal(tok, oracle.assign(sc, b.offsets, _prescaled(cents.reshape(-1, 4), w), b.K))
    kn = oracle.knn(b.coords, b.offsets, cents, b.K, 6, axis_scale=w)
    assert np.array_equal(kn, oracle.knn(sc, b.offsets, _prescaled(cents.reshape(-1, 4), w), b.K, 6))

    # power-of-two scales are exact in float32 and float64: the whole tokenizer
    # (Lloyd included) equals the unscaled one on pre-scaled coordinates, with
    # the centroids in the caller's units (divided back exactly)
    w2 = np.array([0.5, 2.0, 1.0, 0.125], np.float32)
    b = workloads.random_batch(74, [5, 260, 1000], 32, lloyd_iters=2, charge_col=0)
    b.axis_scale = tuple(float(v) for v in w2)
    got = oracle.tokenize_batch(b)
    want = oracle.tokenize(_prescaled(b.coords, w2), b.feats, b.offsets, b.K, lloyd_iters=2, charge_col=0)
    for key in ("centroid_idx", "token_id", "counts", "pooled"):
        assert np.array_equal(got[key], want[key]), key
    assert np.array_equal(got["centroids"] * w2, want["centroids"])

    # a zero time weight ignores time: FPS equals FPS with t zeroed
    b = workloads.random_batch(75, [90, 500], 16)
    z = b.coords.copy()
    z[:, 3] = 0.0
    assert np.array_equal(oracle.fps(b.coords, b.offsets, b.K, axis_scale=[1, 1, 1, 0]),
                          oracle.fps(z, b.offsets, b.K))


def test_axis_scale():
    pin_axis_scale()
