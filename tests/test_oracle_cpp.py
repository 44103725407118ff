"""The plain C++ oracle (oracle/hxq_oracle_ref.cpp) against the hand-worked
golden layers and against the numpy oracle: two independently written CPU
oracles of the same definition must decode identically, bit for bit, and
agree on the forward to float64 rounding (their sums run in different
orders); on dyadic layers with integer activations both are exact, so they
agree exactly. Their encoder sides (assignment, Lloyd rounds, sidecar
selection) take the same fp32 decisions and sum the means in the same
order, so they agree bit for bit."""
import numpy as np
import pytest

import golden_io
import oracle
import synthetic
from oracle import hxq_oracle_cpp as cpp


@pytest.mark.parametrize("name", ["tiny_scalar.txt", "tiny_vq2d.txt"])
def test_cpp_oracle_golden_layers(name):
    layer, x, W, y, s = golden_io.tiny_layer(name)
    Wc = cpp.decode(layer["mode"], layer["codebook"], layer["indices"], layer["sidecar_pos"],
                    layer["sidecar_val"], layer["N"], layer["K"])
    assert np.array_equal(Wc, W.astype(np.float32))
    bits = synthetic.f32_to_bf16_bits(x.astype(np.float32))
    yc, sc = cpp.forward(bits, Wc)
    assert np.array_equal(yc, y) and np.array_equal(sc, s)


@pytest.mark.parametrize("mode,N,K,ns", [(0, 130, 72, 40), (0, 3, 8, 0), (1, 129, 136, 60), (1, 7, 64, 7)])
@pytest.mark.parametrize("M", [1, 5])
def test_cpp_oracle_matches_numpy_oracle(mode, N, K, ns, M):
    layer = synthetic.make_layer(mode, N, K, 900 + N, sidecar_count=ns)
    x = synthetic.activations(M, K, 901)
    args = (mode, layer["codebook"], layer["indices"], layer["sidecar_pos"], layer["sidecar_val"], N, K)
    Wn = oracle.decode(*args)
    Wc = cpp.decode(*args)
    assert np.array_equal(Wc, Wn)
    yn, sn = oracle.forward(x, Wn), oracle.abs_scale(x, Wn)
    yc, sc = cpp.forward(x, Wc)
    tol = 1e-12 * sn
    assert np.all(np.abs(yc - yn) <= tol) and np.all(np.abs(sc - sn) <= tol)


@pytest.mark.parametrize("mode", [0, 1])
def test_cpp_oracle_dyadic_exact_agreement(mode):
    rng = np.random.default_rng(910 + mode)
    N, K, M = 40, 64, 3
    if mode == 0:
        cb = (rng.integers(-64, 64, 256) * 2.0 ** -6).astype(np.float32)
        idx = rng.integers(0, 256, N * K).astype(np.uint8)
    else:
        cb = (rng.integers(-64, 64, 8192) * 2.0 ** -6).astype(np.float32)
        idx = oracle.pack12(rng.integers(0, 4096, N * K // 2))
    pos = rng.choice(N * K, 30, replace=False).astype(np.int64)
    val = (rng.integers(-32, 32, 30) * 2.0 ** -3).astype(np.float32)
    x = synthetic.f32_to_bf16_bits(rng.integers(-8, 8, (M, K)).astype(np.float32))
    Wn = oracle.decode(mode, cb, idx, pos, val, N, K)
    Wc = cpp.decode(mode, cb, idx, pos, val, N, K)
    assert np.array_equal(Wc, Wn)
    yc, sc = cpp.forward(x, Wc)
    assert np.array_equal(yc, oracle.forward(x, Wn)) and np.array_equal(sc, oracle.abs_scale(x, Wn))


def test_cpp_oracle_rejects_bad_layers():
    cb = np.zeros(8192, np.float32)
    idx = np.zeros(64, np.uint8)
    with pytest.raises(ValueError):
        cpp.decode(0, cb, idx, [3, 3], [1.0, 2.0], 8, 8)       # repeated position
    with pytest.raises(ValueError):
        cpp.decode(0, cb, idx, [64], [1.0], 8, 8)              # out of range
    with pytest.raises(ValueError):
        cpp.decode(2, cb, idx, [], [], 8, 8)                   # unknown mode
    with pytest.raises(ValueError):
        cpp.decode(1, cb, idx, [], [], 2, 6)                   # 2D needs K % 4 == 0


# ----------------------------------------------------------------- encoder side

enc = oracle.hxq_encoder_oracle


@pytest.mark.parametrize("dim,k,n", [(1, 256, 20000), (2, 512, 8000), (2, 4096, 6000)])
def test_cpp_encoder_matches_numpy_encoder(dim, k, n):
    rng = np.random.default_rng(920 + dim + k)
    pts = rng.normal(0, 0.02, size=(n, dim)).astype(np.float32)
    init = pts[rng.choice(n, k, replace=False)].copy()
    init[k // 3] = init[1]  # an exact tie
    assert np.array_equal(cpp.assign(pts, init), enc.assign(pts, init))
    # float64 means in the same (point) order: the same fp32 centroids, bit for bit
    c_c, lab_c = cpp.kmeans(pts, init, 4)
    c_n, lab_n = enc.kmeans(pts, init, 4)
    assert np.array_equal(c_c, c_n) and np.array_equal(lab_c, lab_n)


def test_cpp_sidecar_select_matches_numpy():
    rng = np.random.default_rng(930)
    W = rng.normal(0, 0.02, size=(64, 96)).astype(np.float32)
    W_hat = (np.rint(W * 256) / 256).astype(np.float32)
    for t in (0.0, 0.0005, 0.001, 0.00195312):
        pc, vc = cpp.sidecar_select(W, W_hat, t)
        pn, vn = enc.sidecar_select(W, W_hat, t)
        assert np.array_equal(pc, pn) and np.array_equal(vc, vn)


def test_cpp_encoder_hand_worked_cases():
    import os
    path = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden", "tiny_kmeans.txt")
    for raw in open(path):
        line = raw.split("#", 1)[0].strip()
        if not line.startswith("kmeans:"):
            continue
        f = [x.split() for x in line.split(":", 1)[1].split("|")]
        dim = int(f[1][0])
        arr = lambda t: np.array([float(v) for v in t], np.float32).reshape(-1, dim)
        c, lab = cpp.kmeans(arr(f[2]), arr(f[3]), int(f[4][0]))
        assert np.array_equal(c, arr(f[5])) and np.array_equal(lab, [int(v) for v in f[6]]), f[0]


@pytest.mark.parametrize("mode,N,K,ns", [(0, 130, 72, 40), (1, 129, 136, 60), (0, 300, 64, 300)])
@pytest.mark.parametrize("threads", [1, 3])
def test_cpp_forward_rows_equals_forward(mode, N, K, ns, threads):
    """The row-range forward used to time the oracle on the host cores takes
    the same steps as decode + forward (the same k-order float64 sums), so
    any row range, on any number of threads, matches them exactly."""
    layer = synthetic.make_layer(mode, N, K, 70 + N, sidecar_count=ns)
    x = synthetic.activations(2, K, 71)
    W = cpp.decode(mode, layer["codebook"], layer["indices"], layer["sidecar_pos"], layer["sidecar_val"], N, K)
    y, _ = cpp.forward(x, W)
    for r0, r1 in [(0, N), (1, N - 1), (N // 2, N // 2 + 1)]:
        got = cpp.forward_rows(layer, x, r0, r1, threads)
        assert np.array_equal(got, y[:, r0:r1])
    with pytest.raises(ValueError):
        cpp.forward_rows(layer, x, 3, 2)


def test_cpp_exact_mean_matches_numpy_over_wide_magnitudes():
    """The two oracles form the exact mean independently (C++: base-2^32
    digit sums and long division; numpy: Python integers and a rational
    rounding) and must agree bit for bit, on clusters spanning about 80
    binades and on the planted midpoint case."""
    rng = np.random.default_rng(3)
    for trial in range(20):
        n, k, dim = int(rng.integers(1, 20000)), int(rng.integers(1, 50)), int(rng.integers(1, 3))
        pts = (rng.normal(0, 0.02, size=(n, dim)) * np.exp2(rng.integers(-40, 40, size=(n, dim)))).astype(np.float32)
        lab = rng.integers(0, k, size=n)
        c = rng.normal(size=(k, dim)).astype(np.float32)
        a, b = enc.kmeans_update(pts, lab, c), cpp.kmeans_update(pts, lab, c)
        assert np.array_equal(a.view(np.uint32), b.view(np.uint32)), trial
    pts = np.array([10.0, 2.0 ** -22, 7 * 2.0 ** -60, 2.0 ** -22], np.float32)
    got = cpp.kmeans_update(pts, np.zeros(4, np.int64), np.zeros(1, np.float32))[0, 0]
    assert got == np.nextafter(np.float32(2.5), np.float32(3.0))


def test_cpp_threaded_assign_equals_plain():
    rng = np.random.default_rng(4)
    for dim in (1, 2):
        pts = rng.normal(0, 0.02, size=(30001, dim)).astype(np.float32)
        cents = rng.normal(0, 0.02, size=(77, dim)).astype(np.float32)
        assert np.array_equal(cpp.assign(pts, cents, threads=5), cpp.assign(pts, cents))
