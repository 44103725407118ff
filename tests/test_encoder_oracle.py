"""Pins of the encoder oracle (CPU): k-means, index assignment, sidecar
selection and the full encode, each checked against something other than
its own formula -- exact integer brute force on dyadic inputs, the midpoint
rule, scikit-learn's Lloyd k-means, Lloyd's monotone objective, weights drawn
exactly from a codebook, hand-worked cases in tests/golden/tiny_kmeans.txt --
and planted mistakes that those pins must catch.
"""
import numpy as np
import pytest

import oracle

enc = oracle.hxq_encoder_oracle


def _dyadic(rng, shape, lo=-64, hi=64, scale=2.0 ** -6):
    """Small multiples of 2^-6: fp32 differences, squares and sums of two
    squares of these are exact, so fp32 decisions equal exact ones."""
    return (rng.integers(lo, hi, size=shape) * scale).astype(np.float32)


def _exact_nearest(points_int, cents_int):
    """Nearest centroid with Python integers (the dyadic grid scaled to
    integers); ties to the lowest index."""
    out = []
    for p in points_int:
        best, bi = None, -1
        for i, c in enumerate(cents_int):
            d = sum((a - b) * (a - b) for a, b in zip(p, c))
            if best is None or d < best:
                best, bi = d, i
        out.append(bi)
    return np.array(out, dtype=np.int64)


@pytest.mark.parametrize("dim", [1, 2])
def test_assign_exact_integer_bruteforce(dim):
    rng = np.random.default_rng(3 + dim)
    pts = _dyadic(rng, (300, dim))
    # few distinct centroid values, some repeated: exact ties must go to the lowest index
    cents = _dyadic(rng, (12, dim), -16, 16, 2.0 ** -4)
    cents[7] = cents[2]
    cents[11] = cents[5]
    got = enc.assign(pts if dim == 2 else pts[:, 0], cents if dim == 2 else cents[:, 0])
    to_int = lambda a: [tuple(int(v) for v in row) for row in np.rint(a.astype(np.float64) * 64)]
    want = _exact_nearest(to_int(pts), to_int(cents))
    assert np.array_equal(got, want)
    assert not np.isin(got, [7, 11]).any()  # the later copy of a tie never wins


def test_assign_midpoint_rule_1d():
    """Sorted distinct centroids in 1D: the nearest is found by comparing
    with the midpoints between neighbours (a point on a midpoint goes left,
    to the lower index)."""
    rng = np.random.default_rng(5)
    cents = np.unique(_dyadic(rng, 40, -512, 512, 2.0 ** -7))
    pts = _dyadic(rng, 5000, -600, 600, 2.0 ** -8)
    mids = (cents[:-1].astype(np.float64) + cents[1:]) / 2
    want = np.searchsorted(mids, pts.astype(np.float64), side="left")
    assert np.array_equal(enc.assign(pts, cents), want)


def _blobs(rng, centers, per, sigma):
    c = np.asarray(centers, np.float64)
    pts = np.repeat(c, per, axis=0) + rng.normal(0, sigma, size=(c.shape[0] * per, c.shape[1]))
    return pts[rng.permutation(pts.shape[0])].astype(np.float32)


@pytest.mark.parametrize("dim", [1, 2])
def test_kmeans_matches_sklearn_lloyd(dim):
    from sklearn.cluster import KMeans
    rng = np.random.default_rng(11 + dim)
    k = 6
    centers = rng.uniform(-1, 1, size=(k, dim)) * 4
    pts = _blobs(rng, centers, 400, 0.25)
    init = pts[rng.choice(pts.shape[0], k, replace=False)]
    for iters in (1, 3, 20):
        c, lab = enc.kmeans(pts, init, iters)
        km = KMeans(n_clusters=k, init=init.astype(np.float64), n_init=1, max_iter=iters, tol=0.0,
                    algorithm="lloyd").fit(pts.astype(np.float64))
        assert np.array_equal(lab, km.labels_), f"iters {iters}"
        assert np.allclose(c, km.cluster_centers_, rtol=0, atol=1e-6), f"iters {iters}"


@pytest.mark.parametrize("dim", [1, 2])
def test_kmeans_objective_never_increases(dim):
    rng = np.random.default_rng(21 + dim)
    pts = rng.normal(0, 0.02, size=(4000, dim)).astype(np.float32)
    c = pts[rng.choice(pts.shape[0], 64, replace=False)].copy()
    prev = enc.inertia(pts, c, enc.assign(pts, c))
    for _ in range(8):
        c = enc.kmeans_update(pts, enc.assign(pts, c), c)
        cur = enc.inertia(pts, c, enc.assign(pts, c))
        assert cur <= prev * (1 + 1e-9)
        prev = cur


def test_kmeans_recovers_separated_clusters_and_stays_there():
    rng = np.random.default_rng(31)
    centers = np.array([[-3.0, 1.0], [0.0, -2.0], [2.5, 2.5], [4.0, -4.0]])
    pts = _blobs(rng, centers, 500, 0.05)
    c, lab = enc.kmeans(pts, centers + 0.7, 10)
    assert np.allclose(c, centers, atol=0.02)
    assert np.array_equal(np.bincount(lab, minlength=4), [500] * 4)
    c2, lab2 = enc.kmeans(pts, c, 3)  # a fixed point of Lloyd's rounds
    assert np.array_equal(c2, c) and np.array_equal(lab2, lab)


def test_kmeans_update_empty_cluster_keeps_position():
    pts = np.array([[0.0], [0.25], [4.0], [4.5]], np.float32)
    c = np.array([[0.0], [4.0], [100.0]], np.float32)
    new = enc.kmeans_update(pts, enc.assign(pts, c), c)
    assert np.array_equal(new[:, 0], np.array([0.125, 4.25, 100.0], np.float32))


@pytest.mark.parametrize("mode", [0, 1])
def test_encode_recovers_weights_drawn_from_the_codebook(mode):
    rng = np.random.default_rng(41 + mode)
    N, K = 24, 40
    if mode == 0:
        cb = np.sort(rng.normal(0, 0.02, 256)).astype(np.float32)
        idx = rng.integers(0, 256, size=N * K)
        W = cb[idx].reshape(N, K)
    else:
        cb = rng.normal(0, 0.02, 8192).astype(np.float32)
        idx = rng.integers(0, 4096, size=N * K // 2)
        W = cb.reshape(4096, 2)[idx].reshape(N, K)
    indices, pos, val = enc.encode(W, mode, cb, 0.0)
    want = idx.astype(np.uint8) if mode == 0 else oracle.pack12(idx)
    assert np.array_equal(indices, want)
    assert pos.size == 0 and val.size == 0
    assert np.array_equal(oracle.decode(mode, cb, indices, pos, val, N, K), W)


@pytest.mark.parametrize("mode", [0, 1])
def test_sidecar_planted_outliers_dyadic(mode):
    """Codebook on a coarse dyadic grid, weights on it plus planted offsets:
    an error exactly at the threshold stays out, one above it goes in."""
    rng = np.random.default_rng(51 + mode)
    N, K = 8, 32
    tau = np.float32(2.0 ** -5)
    if mode == 0:
        cb = (np.arange(256) - 128).astype(np.float32) * 2.0 ** -3
        idx = rng.integers(0, 256, size=N * K)
        W_hat = cb[idx].reshape(N, K)
    else:
        g = (np.arange(64) - 32).astype(np.float32) * 2.0 ** -3
        cb = np.stack(np.meshgrid(g, g, indexing="ij"), -1).reshape(-1).astype(np.float32)  # 64 x 64 grid
        idx = rng.integers(0, 4096, size=N * K // 2)
        W_hat = cb.reshape(4096, 2)[idx].reshape(N, K)
    W = W_hat.copy()
    flat = W.reshape(-1)
    at_tau = np.array([3, 77, 130])
    above = np.array([5, 64, 200, 255])
    small = np.array([9, 100])
    flat[at_tau] += tau               # exactly the threshold: not stored
    flat[above] -= np.float32(3 * 2.0 ** -6)  # 0.046875 > tau, still nearest to its own entry
    flat[small] += np.float32(2.0 ** -7)
    indices, pos, val = enc.encode(W, mode, cb, float(tau))
    assert np.array_equal(pos, np.sort(above))
    assert np.array_equal(val, flat[np.sort(above)])
    W_rec = oracle.decode(mode, cb, indices, pos, val, N, K)
    assert np.max(np.abs(W_rec - W)) <= tau
    assert np.array_equal(W_rec.reshape(-1)[pos], flat[pos])


@pytest.mark.parametrize("mode", [0, 1])
def test_encode_decode_roundtrip_within_threshold(mode):
    rng = np.random.default_rng(61 + mode)
    N, K = 16, 64
    W = rng.normal(0, 0.02, size=(N, K)).astype(np.float32)
    pts = W.reshape(-1, 1 if mode == 0 else 2)
    k = 256 if mode == 0 else 4096
    init = pts[rng.choice(pts.shape[0], min(k, pts.shape[0]), replace=False)]
    if init.shape[0] < k:  # 2D with fewer pairs than entries: pad with far points that stay empty
        init = np.concatenate([init, np.full((k - init.shape[0], 2), 1e3, np.float32)])
    cb, _ = enc.kmeans(pts, init, 4)
    tau = 0.004
    indices, pos, val = enc.encode(W, mode, cb.reshape(-1), tau)
    W_rec = oracle.decode(mode, cb.reshape(-1), indices, pos, val, N, K)
    assert np.all(np.abs(W_rec - W) <= np.float32(tau))
    assert np.array_equal(W_rec.reshape(-1)[pos], W.reshape(-1)[pos])


# ----------------------------------------------------------------- planted mistakes

def _pins_pass():
    try:
        for dim in (1, 2):
            test_assign_exact_integer_bruteforce(dim)
            test_kmeans_matches_sklearn_lloyd(dim)
        test_assign_midpoint_rule_1d()
        test_kmeans_update_empty_cluster_keeps_position()
        for mode in (0, 1):
            test_encode_recovers_weights_drawn_from_the_codebook(mode)
            test_sidecar_planted_outliers_dyadic(mode)
        test_hand_worked_encoder_cases()
    except AssertionError:
        return False
    return True


@pytest.mark.parametrize("mutant", ["ties_last", "swap_pair_components", "update_skips_last_point",
                                    "empty_to_zero", "threshold_inclusive", "sidecar_stores_delta",
                                    "sidecar_colmajor"])
def test_encoder_planted_mistakes_are_caught(monkeypatch, mutant):
    assert _pins_pass()
    orig_dist, orig_update, orig_select = enc.distances_f32, enc.kmeans_update, enc.sidecar_select
    if mutant == "ties_last":
        def assign_last(points, centroids):
            d = orig_dist(points, centroids)
            return d.shape[1] - 1 - np.argmin(d[:, ::-1], axis=1)
        monkeypatch.setattr(enc, "assign", assign_last)
    elif mutant == "swap_pair_components":
        def dist_swapped(points, centroids):
            c = enc._as_points(centroids)
            return orig_dist(points, c[:, ::-1] if c.shape[1] == 2 else c)
        monkeypatch.setattr(enc, "distances_f32", dist_swapped)
    elif mutant == "update_skips_last_point":
        monkeypatch.setattr(enc, "kmeans_update",
                            lambda p, lab, c: orig_update(enc._as_points(p)[:-1], np.asarray(lab)[:-1], c))
    elif mutant == "empty_to_zero":
        def update_zero(p, lab, c):
            new = orig_update(p, lab, c)
            new[np.bincount(np.asarray(lab), minlength=len(new)) == 0] = 0
            return new
        monkeypatch.setattr(enc, "kmeans_update", update_zero)
    elif mutant == "threshold_inclusive":
        def select_ge(W, W_hat, t):
            w, wh = np.asarray(W, np.float32).reshape(-1), np.asarray(W_hat, np.float32).reshape(-1)
            pos = np.nonzero(np.abs(w - wh) >= np.float32(t))[0].astype(np.int64)
            return pos, w[pos]
        monkeypatch.setattr(enc, "sidecar_select", select_ge)
    elif mutant == "sidecar_stores_delta":
        def select_delta(W, W_hat, t):
            pos, _ = orig_select(W, W_hat, t)
            return pos, (np.asarray(W, np.float32).reshape(-1) - np.asarray(W_hat, np.float32).reshape(-1))[pos]
        monkeypatch.setattr(enc, "sidecar_select", select_delta)
    elif mutant == "sidecar_colmajor":
        def select_colmajor(W, W_hat, t):
            Wa = np.asarray(W, np.float32)
            pos, val = orig_select(Wa.T, np.asarray(W_hat, np.float32).T, t)
            return pos, val
        monkeypatch.setattr(enc, "sidecar_select", select_colmajor)
    assert not _pins_pass(), f"planted mistake {mutant} was not caught"


# ----------------------------------------------------------------- hand-worked fixtures

def _golden_cases():
    import os
    path = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden", "tiny_kmeans.txt")
    cases = []
    for raw in open(path):
        line = raw.split("#", 1)[0].strip()
        if not line:
            continue
        kind, rest = line.split(":", 1)
        cases.append((kind.strip(), [f.split() for f in rest.split("|")]))
    return cases


def _arr(tokens, dim=1):
    a = np.array([float(t) for t in tokens], np.float32)
    return a.reshape(-1, dim) if dim == 2 else a


def test_hand_worked_encoder_cases():
    cases = _golden_cases()
    assert {k for k, _ in cases} == {"kmeans", "assign", "sidecar"}
    for kind, f in cases:
        name = f[0][0]
        if kind == "kmeans":
            dim = int(f[1][0])
            c, lab = enc.kmeans(_arr(f[2], dim), _arr(f[3], dim), int(f[4][0]))
            assert np.array_equal(c, _arr(f[5], dim)), name
            assert np.array_equal(lab, [int(t) for t in f[6]]), name
        elif kind == "assign":
            dim = int(f[1][0])
            assert np.array_equal(enc.assign(_arr(f[2], dim), _arr(f[3], dim)), [int(t) for t in f[4]]), name
        else:
            cb, w, t = _arr(f[1]), _arr(f[2]), float(f[3][0])
            lab = enc.assign(w, cb)
            assert np.array_equal(lab, [int(v) for v in f[4]]), name
            pos, val = enc.sidecar_select(w, cb[lab], t)
            assert np.array_equal(pos, [int(v) for v in f[5]]), name
            assert np.array_equal(val, _arr(f[6])), name


# ---- the exact mean rounded once to fp32 (reading: exact sum / count, one
# rounding to nearest even)

def _nearest_f32_brute(fr):
    """Round the Fraction fr to fp32 by comparing it exactly with its two fp32
    neighbours (ties to the even significand)."""
    from fractions import Fraction
    if fr == 0:
        return np.float32(0.0)
    lo = np.float32(float(fr))  # near fr; step to the two neighbours around fr
    while Fraction(float(lo)) > fr:
        lo = np.nextafter(lo, np.float32(-np.inf))
    while Fraction(float(np.nextafter(lo, np.float32(np.inf)))) <= fr:
        lo = np.nextafter(lo, np.float32(np.inf))
    hi = np.nextafter(lo, np.float32(np.inf))
    if Fraction(float(lo)) == fr:
        return lo
    dl, dh = fr - Fraction(float(lo)), Fraction(float(hi)) - fr
    if dl != dh:
        return lo if dl < dh else hi
    return lo if (int(np.float32(lo).view(np.uint32)) & 1) == 0 else hi


def test_round_rational_matches_brute_force():
    from fractions import Fraction
    rng = np.random.default_rng(11)
    cases = [(1, 3), (-1, 3), (2, 3), (7, 10), (1, 1 << 150), (3, 1 << 150), (5, 1 << 150), (1, 1 << 151),
             (-(1 << 24) - 1, 2), ((1 << 24) + 1, 2), ((1 << 25) + 2, 4), ((1 << 25) + 6, 4)]
    for _ in range(3000):
        den = int(rng.integers(1, 1 << 40))
        num = int(rng.integers(-(1 << 62), 1 << 62)) >> int(rng.integers(0, 60))
        cases.append((num, den << int(rng.integers(0, 140))))
    for num, den in cases:
        got = enc.round_rational_f32(num, den)
        want = _nearest_f32_brute(Fraction(num, den))
        assert got.view(np.uint32) == want.view(np.uint32), (num, den, got, want)


def test_round_rational_equals_float32_of_exact_float64():
    """Where the rational is exactly a float64, one rounding of that float64
    to fp32 (numpy's cast) is the right answer."""
    rng = np.random.default_rng(12)
    x = rng.normal(0, 1, 20000) * np.exp2(rng.integers(-140, 100, 20000))
    for v in x.tolist():
        n, d = float(v).as_integer_ratio()
        assert enc.round_rational_f32(n, d).view(np.uint32) == np.float32(v).view(np.uint32)


def test_kmeans_update_is_exact_mean_rounded_once():
    """Against Fraction arithmetic, on sets built so that a float64 running
    sum is inexact: a huge value and many tiny ones in one cluster, exact
    ties at fp32 midpoints."""
    from fractions import Fraction
    rng = np.random.default_rng(13)
    pts = np.concatenate([rng.normal(0, 0.02, 4000), [3.0e4], rng.normal(0, 1e-9, 3000),
                          [np.float32(1.0), np.float32(1.0) + np.float32(2.0 ** -23)]]).astype(np.float32)
    lab = np.concatenate([rng.integers(0, 5, 4000), [5], np.full(3000, 5), [6, 6]])
    c = np.zeros(7, np.float32)
    new = enc.kmeans_update(pts, lab, c)
    for j in range(7):
        sel = pts[lab == j]
        want = _nearest_f32_brute(sum((Fraction(float(v)) for v in sel), Fraction(0)) / len(sel))
        assert new[j].view(np.uint32) == want.view(np.uint32), j
    # 1 and 1 + 2^-23 average to a midpoint: ties to the even significand (1.0)
    assert new[6] == np.float32(1.0)


def test_kmeans_update_float64_running_sum_is_caught():
    """A planted mistake: the mean as a float64 running sum over the count,
    then one cast to fp32. For {10, 2^-22, 7 * 2^-60, 2^-22} the exact mean
    is 2.5 + 2^-23 + 7 * 2^-62, just above the midpoint between 2.5 and the
    next fp32 value, so it rounds up; the float64 sum drops the 7 * 2^-60,
    lands on the midpoint and ties down to 2.5."""
    pts = np.array([10.0, 2.0 ** -22, 7 * 2.0 ** -60, 2.0 ** -22], dtype=np.float32)
    exact = enc.kmeans_update(pts, np.zeros(4, np.int64), np.zeros(1, np.float32))[0]
    assert exact == np.nextafter(np.float32(2.5), np.float32(3.0))
    running = np.float64(0.0)
    for v in pts.tolist():
        running += np.float64(v)
    assert np.float32(running / 4) == np.float32(2.5)
