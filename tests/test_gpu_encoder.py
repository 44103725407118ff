"""GPU encoder (hxq_assign, hxq_kmeans, hxq_encode) against the encoder
oracle, through the C ABI.

Bar: bit-exact throughout. Index assignment and everything decided from it
(indices, packed bytes, sidecar positions and values, counts), and the
k-means centroids -- the exact mean of each cluster's fp32 coordinates,
rounded once to fp32 -- after one round and after ten, at the bench's full
layer shapes too, and bitwise repeatable run to run.
"""
import os

import numpy as np
import pytest

import oracle
import synthetic

pytestmark = pytest.mark.gpu

enc = oracle.hxq_encoder_oracle


def _dev(a):
    import torch
    return torch.from_numpy(np.ascontiguousarray(a)).cuda()


def _labels(t):
    import torch
    return (t.cpu().to(torch.int32) & 0xFFFF).numpy().astype(np.int64)


def _ulps(a, b):
    """Distance in fp32 units in the last place, elementwise."""
    a = np.asarray(a, np.float32).astype(np.float64)
    b = np.asarray(b, np.float32).astype(np.float64)
    return np.abs(a - b) / np.spacing(np.maximum(np.abs(a), np.abs(b)).astype(np.float32)).astype(np.float64)


@pytest.mark.parametrize("dim,k,n", [(1, 256, 100003), (1, 7, 5000), (2, 4096, 50001), (2, 300, 1)])
def test_assign_bit_exact(hxq, dim, k, n):
    import torch
    rng = np.random.default_rng(100 + dim + k)
    pts = rng.normal(0, 0.02, size=(n, dim)).astype(np.float32)
    cents = rng.normal(0, 0.02, size=(k, dim)).astype(np.float32)
    if k > 10:  # exact ties: a later copy of a centroid never wins
        cents[k - 1] = cents[3]
        cents[k - 2] = cents[1]
    lab = torch.empty(n, dtype=torch.int16, device="cuda")
    hxq.hxq_assign(_dev(pts), n, dim, _dev(cents), k, lab)
    torch.cuda.synchronize()
    want = enc.assign(pts if dim == 2 else pts[:, 0], cents if dim == 2 else cents[:, 0])
    assert np.array_equal(_labels(lab), want)


def test_assign_dyadic_ties(hxq):
    """Points and centroids on a coarse dyadic grid: many exact ties."""
    import torch
    rng = np.random.default_rng(7)
    pts = (rng.integers(-40, 40, size=(20000, 2)) * 2.0 ** -5).astype(np.float32)
    cents = (rng.integers(-8, 8, size=(64, 2)) * 2.0 ** -3).astype(np.float32)
    lab = torch.empty(pts.shape[0], dtype=torch.int16, device="cuda")
    hxq.hxq_assign(_dev(pts), pts.shape[0], 2, _dev(cents), 64, lab)
    torch.cuda.synchronize()
    assert np.array_equal(_labels(lab), enc.assign(pts, cents))


@pytest.mark.parametrize("dim,k,n", [(1, 256, 200000), (2, 4096, 120000), (2, 16, 999)])
def test_kmeans_one_round(hxq, dim, k, n):
    import torch
    rng = np.random.default_rng(200 + dim)
    pts = rng.normal(0, 0.02, size=(n, dim)).astype(np.float32)
    init = pts[rng.choice(n, k, replace=False)].copy()
    init[-1] = 50.0  # far away: a centroid with no points stays
    c_dev = _dev(init)
    lab = torch.empty(n, dtype=torch.int16, device="cuda")
    hxq.hxq_kmeans(_dev(pts), n, dim, k, 1, c_dev, lab)
    torch.cuda.synchronize()
    got = c_dev.cpu().numpy()
    want = enc.kmeans_update(pts, enc.assign(pts, init), init)
    assert np.array_equal(got.view(np.uint32), want.view(np.uint32)), f"max {np.max(_ulps(got, want))} ulp"
    assert np.array_equal(got[-1], init[-1])
    # the returned labels are the assignment to the returned centroids
    assert np.array_equal(_labels(lab), enc.assign(pts, got))


@pytest.mark.parametrize("dim,k", [(1, 256), (2, 1024)])
def test_kmeans_rounds_match_oracle_and_repeat(hxq, dim, k):
    import torch
    rng = np.random.default_rng(300 + dim)
    n = 60000
    pts = rng.normal(0, 0.02, size=(n, dim)).astype(np.float32)
    init = pts[rng.choice(n, k, replace=False)].copy()
    runs = []
    for _ in range(2):
        c_dev = _dev(init)
        lab = torch.empty(n, dtype=torch.int16, device="cuda")
        hxq.hxq_kmeans(_dev(pts), n, dim, k, 10, c_dev, lab)
        torch.cuda.synchronize()
        runs.append((c_dev.cpu().numpy(), _labels(lab)))
    assert np.array_equal(runs[0][0], runs[1][0]) and np.array_equal(runs[0][1], runs[1][1]), "not repeatable"
    c_or, lab_or = enc.kmeans(pts, init, 10)
    c_gpu, lab_gpu = runs[0]
    assert np.array_equal(c_gpu.view(np.uint32), c_or.view(np.uint32)), f"max {np.max(_ulps(c_gpu, c_or))} ulp"
    assert np.array_equal(lab_gpu, lab_or)


def test_kmeans_wide_magnitudes_exact(hxq):
    """Clusters whose points span many binades (1e-9 .. 1e-1): a float64
    running sum would drop low bits here; the exact means do not."""
    import torch
    rng = np.random.default_rng(310)
    n = 50000
    pts = (rng.normal(0, 0.02, n) * np.exp2(rng.integers(-22, 1, n))).astype(np.float32)
    init = np.sort(pts[rng.choice(n, 64, replace=False)]).copy()
    c_dev = _dev(init)
    hxq.hxq_kmeans(_dev(pts), n, 1, 64, 3, c_dev, None)
    torch.cuda.synchronize()
    c_or, _ = enc.kmeans(pts, init, 3)
    assert np.array_equal(c_dev.cpu().numpy().view(np.uint32), c_or.view(np.uint32))


@pytest.mark.parametrize("shape", ["scalar", "vq2d"])
def test_kmeans_bench_shapes_ten_rounds_exact(hxq, shape):
    """The bench's encoder layers (Mamba2 in_proj 8512 x 2048 scalars, k =
    256; 11008 x 4096 as 22.5M pairs, k = 4096), ten Lloyd rounds from the
    bench's seeded start, checked round by round: every label of the GPU
    assignment against the plain C++ oracle's (all host threads), and every
    new centroid against the oracle's exact-mean update from those labels,
    bit for bit; one ten-round call then ends on the same centroids."""
    import sys
    import torch
    sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
    import bench
    from oracle import hxq_oracle_cpp as cpp
    mode, N, K, k, tau, dim, W, init = bench.encoder_layer(shape)
    pts = W.reshape(-1, dim)
    n = pts.shape[0]
    pts_dev = _dev(pts.reshape(-1) if dim == 1 else pts)
    c = (init if dim == 2 else init[:, 0]).copy()
    lab = torch.empty(n, dtype=torch.int16, device="cuda")
    threads = os.cpu_count() or 1
    for r in range(10):
        hxq.hxq_assign(pts_dev, n, dim, _dev(c), k, lab)
        torch.cuda.synchronize()
        lab_gpu = _labels(lab)
        lab_or = cpp.assign(pts if dim == 2 else pts[:, 0], c, threads)
        assert np.array_equal(lab_gpu, lab_or), f"round {r}: {np.sum(lab_gpu != lab_or)} labels differ"
        c_dev = _dev(c)
        hxq.hxq_kmeans(pts_dev, n, dim, k, 1, c_dev, None)
        torch.cuda.synchronize()
        c_gpu = c_dev.cpu().numpy()
        c_or = enc.kmeans_update(pts, lab_or, c.reshape(k, dim)).reshape(c.shape)
        assert np.array_equal(c_gpu.view(np.uint32), c_or.view(np.uint32)), \
            f"round {r}: {np.sum(c_gpu != c_or)} centroids differ, max {np.max(_ulps(c_gpu, c_or))} ulp"
        c = c_gpu
    c_dev = _dev(init if dim == 2 else init[:, 0])
    hxq.hxq_kmeans(pts_dev, n, dim, k, 10, c_dev, None)
    torch.cuda.synchronize()
    assert np.array_equal(c_dev.cpu().numpy().view(np.uint32), c.view(np.uint32))


def _encode_gpu(hxq, W, mode, cb, tau, cap):
    import torch
    N, K = W.shape
    nbytes = N * K if mode == 0 else 3 * N * K // 4
    idx = torch.empty(nbytes, dtype=torch.uint8, device="cuda")
    pos = torch.full((max(cap, 1),), -1, dtype=torch.int64, device="cuda")
    val = torch.zeros(max(cap, 1), dtype=torch.float32, device="cuda")
    cnt = torch.zeros(1, dtype=torch.int64, device="cuda")
    hxq.hxq_encode(_dev(W), mode, N, K, _dev(cb), tau, idx, pos, val, cap, cnt)
    torch.cuda.synchronize()
    return idx.cpu().numpy(), pos.cpu().numpy(), val.cpu().numpy(), int(cnt.item())


@pytest.mark.parametrize("mode,N,K,tau", [(0, 1000, 1024, 0.0009), (0, 37, 200, 0.0009), (1, 600, 512, 0.012),
                                        (1, 9, 72, 0.003), (0, 41, 13, 0.0003), (0, 7, 1, 0.0),
                                        (1, 33, 12, 0.003)])
def test_encode_bit_exact(hxq, mode, N, K, tau):
    rng = np.random.default_rng(400 + mode + N)
    W = rng.normal(0, 0.02, size=(N, K)).astype(np.float32)
    if mode == 0:
        cb = np.sort(rng.normal(0, 0.02, 256)).astype(np.float32)
    else:
        cb = rng.normal(0, 0.02, 8192).astype(np.float32)
    idx_o, pos_o, val_o = enc.encode(W, mode, cb, tau)
    assert pos_o.size > 0
    idx, pos, val, n = _encode_gpu(hxq, W, mode, cb, tau, pos_o.size + 10)
    assert np.array_equal(idx, idx_o)
    assert n == pos_o.size
    assert np.array_equal(pos[:n], pos_o) and np.array_equal(val[:n], val_o)
    assert np.all(pos[n:] == -1)  # nothing written past the count


def test_encode_sidecar_capacity(hxq):
    """Room for fewer entries than exceed the threshold: the count is the
    full one and the lowest positions are written."""
    rng = np.random.default_rng(500)
    W = rng.normal(0, 0.02, size=(300, 256)).astype(np.float32)
    cb = np.sort(rng.normal(0, 0.02, 256)).astype(np.float32)
    _, pos_o, val_o = enc.encode(W, 0, cb, 0.0005)
    cap = pos_o.size // 3
    _, pos, val, n = _encode_gpu(hxq, W, 0, cb, 0.0005, cap)
    assert n == pos_o.size
    assert np.array_equal(pos[:cap], pos_o[:cap]) and np.array_equal(val[:cap], val_o[:cap])
    _, _, _, n0 = _encode_gpu(hxq, W, 0, cb, 0.0005, 0)  # count only
    assert n0 == pos_o.size


@pytest.mark.parametrize("mode", [0, 1])
def test_gpu_encoded_layer_runs_forward(hxq, mode):
    """k-means, encode and create on the GPU: the handle decodes to the
    oracle's decoding of the same buffers, stays within the threshold of W,
    and its forward matches the oracle."""
    import torch
    rng = np.random.default_rng(600 + mode)
    N, K = 512, 1024
    W = rng.normal(0, 0.02, size=(N, K)).astype(np.float32)
    dim, k = (1, 256) if mode == 0 else (2, 4096)
    pts = W.reshape(-1, dim)
    init = pts[rng.choice(pts.shape[0], k, replace=False)]
    Wd = _dev(W)
    cent, _ = hxq.kmeans(Wd.view(-1) if dim == 1 else Wd.view(-1, 2), _dev(init if dim == 2 else init[:, 0]), 5)
    tau = 0.002
    idx, pos, val = hxq.encode(Wd, mode, cent.reshape(-1), tau)
    lin = hxq.HelixLinear(cent.reshape(-1), idx, mode, pos, val, N, K)
    W_gpu = lin.decode().cpu().numpy()
    torch.cuda.synchronize()
    cb, idx_h, pos_h, val_h = (t.cpu().numpy() for t in (cent.reshape(-1), idx, pos, val))
    W_or = oracle.decode(mode, cb, idx_h, pos_h, val_h, N, K)
    assert np.array_equal(W_gpu, W_or)
    assert np.all(np.abs(W_or - W) <= np.float32(tau))
    x = synthetic.activations(4, K, 601)
    y = lin.forward(_dev(x.view(np.int16))).cpu().numpy()
    assert np.all(np.abs(y - oracle.forward(x, W_or)) <= 1e-5 * oracle.abs_scale(x, W_or))
    lin.close()


def test_encoder_rejects_bad_arguments(hxq):
    import torch
    p = torch.zeros(64, dtype=torch.float32, device="cuda")
    c = torch.zeros(8, dtype=torch.float32, device="cuda")
    lab = torch.zeros(64, dtype=torch.int16, device="cuda")
    L = hxq.lib
    assert L.hxq_assign(p.data_ptr(), 64, 3, c.data_ptr(), 8, lab.data_ptr(), None) == hxq.HXQ_EINVAL
    assert L.hxq_assign(p.data_ptr(), 64, 1, c.data_ptr(), 4097, lab.data_ptr(), None) == hxq.HXQ_EINVAL
    assert L.hxq_assign(p.data_ptr(), 0, 1, c.data_ptr(), 8, lab.data_ptr(), None) == hxq.HXQ_EINVAL
    assert L.hxq_kmeans(p.data_ptr(), 64, 1, 8, -1, c.data_ptr(), None, None) == hxq.HXQ_EINVAL
    cnt = torch.zeros(1, dtype=torch.int64, device="cuda")
    idx = torch.zeros(64, dtype=torch.uint8, device="cuda")
    enc_ = L.hxq_encode
    assert enc_(p.data_ptr(), 0, 8, 8, c.data_ptr(), float("nan"), idx.data_ptr(), None, None, 0,
                cnt.data_ptr(), None) == hxq.HXQ_EINVAL
    assert enc_(p.data_ptr(), 0, 8, 8, c.data_ptr(), -1.0, idx.data_ptr(), None, None, 0,
                cnt.data_ptr(), None) == hxq.HXQ_EINVAL
    assert enc_(p.data_ptr(), 0, 8, 8, c.data_ptr(), 0.1, idx.data_ptr(), None, None, 5,
                cnt.data_ptr(), None) == hxq.HXQ_EINVAL
    assert enc_(p.data_ptr(), 2, 8, 8, c.data_ptr(), 0.1, idx.data_ptr(), None, None, 0,
                cnt.data_ptr(), None) == hxq.HXQ_EINVAL
    assert enc_(p.data_ptr(), 1, 4, 10, c.data_ptr(), 0.1, idx.data_ptr(), None, None, 0,
                cnt.data_ptr(), None) == hxq.HXQ_EINVAL
