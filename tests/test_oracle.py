"""Pins for the CPU oracle: it is checked against things other than itself.

* hand-worked golden vectors (tests/golden/) for the 12-bit packing, the bf16
  rounding and two tiny layers (one per mode);
* exact integer brute force (dyadic codebooks, integer activations);
* pure-Python loops with correctly rounded sums on tiny random layers;
* the invariants: constant codebook, one-hot activation, Cartesian-product
  2D codebook equal to the scalar decode of the matching index pair;
* torch's bf16 conversion as an independent library routine for rounding;
* planted mistakes: plausible bugs substituted into the oracle must fail at
  least one of the pins above.
"""
import math

import numpy as np
import pytest

import oracle
import synthetic
from golden_io import hex_table, tiny_layer

pytestmark = pytest.mark.filterwarnings("ignore::RuntimeWarning")


def bits(x):
    return synthetic.f32_to_bf16_bits(np.asarray(x, np.float32))


# ----------------------------------------------------------------- packing

def test_pack12_golden_vectors():
    table = hex_table("pack12_vectors.txt")
    idx = np.array([[r[0], r[1]] for r in table]).reshape(-1)
    packed = np.array([[r[2], r[3], r[4]] for r in table], np.uint8).reshape(-1)
    assert np.array_equal(oracle.unpack12(packed, idx.size), idx)
    assert np.array_equal(oracle.pack12(idx), packed)


def test_pack12_roundtrip_random():
    rng = np.random.default_rng(5)
    idx = rng.integers(0, 4096, size=1000)
    assert np.array_equal(oracle.unpack12(oracle.pack12(idx), idx.size), idx)
    raw = rng.integers(0, 256, size=3 * 333, dtype=np.uint8)
    assert np.array_equal(oracle.pack12(oracle.unpack12(raw, 666)), raw)


def test_pack12_rejects_bad_input():
    with pytest.raises(ValueError):
        oracle.pack12(np.array([1, 2, 3]))
    with pytest.raises(ValueError):
        oracle.pack12(np.array([4096, 0]))


# ----------------------------------------------------------------- bf16

def test_bf16_rounding_golden():
    for f32, b16 in hex_table("bf16_rne_vectors.txt"):
        a = np.array([f32], np.uint32).view(np.float32)
        got = oracle.round_to_bf16(a).view(np.uint32)[0]
        assert got == (b16 << 16), (hex(f32), hex(got))


def test_bf16_rounding_matches_torch():
    import torch
    rng = np.random.default_rng(11)
    u = rng.integers(0, 2**32, size=200000, dtype=np.uint64).astype(np.uint32)
    # force many exact ties and near-ties
    u[:50000] = (u[:50000] & 0xFFFF0000) | 0x8000
    u[50000:60000] = (u[50000:60000] & 0xFFFF0000) | 0x7FFF
    a = u.view(np.float32)
    finite = np.isfinite(a)
    mine = oracle.round_to_bf16(a[finite])
    ref = torch.from_numpy(a[finite].copy()).to(torch.bfloat16).to(torch.float32).numpy()
    assert np.array_equal(mine.view(np.uint32), ref.view(np.uint32))


def test_bf16_widening_is_exact():
    b = np.arange(0, 65536, dtype=np.uint32).astype(np.uint16)
    w = oracle.bf16_bits_to_f64(b)
    import torch
    ref = torch.from_numpy(b.view(np.int16).copy()).view(torch.bfloat16).to(torch.float64).numpy()
    same = (w == ref) | (np.isnan(w) & np.isnan(ref))
    assert same.all()


# ----------------------------------------------------------------- golden layers

@pytest.mark.parametrize("name", ["tiny_scalar.txt", "tiny_vq2d.txt"])
def test_tiny_layer_golden(name):
    layer, x, W, y, s = tiny_layer(name)
    W_hat, y_o, s_o = oracle.forward_layer(layer, bits(x))
    assert np.array_equal(W_hat, W.astype(np.float32))
    assert np.array_equal(y_o, y)
    assert np.array_equal(s_o, s)
    y_r, s_r = oracle.forward_rows(layer, bits(x), np.arange(layer["N"])[::-1])
    assert np.array_equal(y_r, y[:, ::-1]) and np.array_equal(s_r, s[:, ::-1])


# ----------------------------------------------------------------- brute force

def _brute_decode(layer):
    """Element-by-element decode with Python integers and loops."""
    N, K, cb, idx = layer["N"], layer["K"], layer["codebook"], layer["indices"]
    W = [[0.0] * K for _ in range(N)]
    for n in range(N):
        for k in range(K):
            if layer["mode"] == 0:
                W[n][k] = float(cb[int(idx[n * K + k])])
            else:
                g = n * (K // 2) + k // 2          # pair number, row-major
                b0, b1, b2 = (int(idx[3 * (g // 2) + t]) for t in range(3))
                if g % 2 == 0:
                    e = b0 + 256 * (b1 % 16)
                else:
                    e = b1 // 16 + 16 * b2
                W[n][k] = float(cb[2 * e + (k % 2)])
    for p, v in zip(layer["sidecar_pos"], layer["sidecar_val"]):
        W[int(p) // K][int(p) % K] = float(v)
    return W


def _brute_forward(x_f, W):
    M, N = len(x_f), len(W)
    y = [[math.fsum(a * b for a, b in zip(x_f[m], W[n])) for n in range(N)] for m in range(M)]
    s = [[math.fsum(abs(a * b) for a, b in zip(x_f[m], W[n])) for n in range(N)] for m in range(M)]
    return np.array(y), np.array(s)


@pytest.mark.parametrize("mode", [0, 1])
@pytest.mark.parametrize("N,K", [(4, 4), (8, 12), (12, 8), (16, 16), (5, 20)])
@pytest.mark.parametrize("M", [1, 3])
def test_bruteforce_tiny(mode, N, K, M):
    seed = 100 * N + K + 7 * M + mode
    layer = synthetic.make_layer(mode, N, K, seed, sidecar_count=max(1, N * K // 9))
    x = synthetic.activations(M, K, seed)
    W_hat, y, s = oracle.forward_layer(layer, x)
    Wb = _brute_decode(layer)
    assert np.array_equal(W_hat, np.array(Wb, np.float32))
    xf = oracle.bf16_bits_to_f64(x).tolist()
    yb, sb = _brute_forward(xf, Wb)
    assert np.all(np.abs(y - yb) <= 1e-13 * sb + 1e-300)
    assert np.all(np.abs(s - sb) <= 1e-13 * sb + 1e-300)


def test_dyadic_exact_integer_bruteforce():
    """Codebook j/256 - 1/2, dyadic sidecar, integer x in [-4, 4]: every
    product and partial sum is a multiple of 1/256 and far below 2^53, so y is
    exact; compare with integer arithmetic on 256*W."""
    N, K, M = 37, 300, 3
    rng = np.random.default_rng(3)
    cb = (np.arange(256) / 256.0 - 0.5).astype(np.float32)
    idx = rng.integers(0, 256, size=N * K, dtype=np.uint8)
    pos = rng.choice(N * K, size=60, replace=False).astype(np.int64)
    val = (rng.integers(-128, 129, size=60) / 256.0).astype(np.float32)
    layer = dict(mode=0, N=N, K=K, codebook=cb, indices=idx, sidecar_pos=pos, sidecar_val=val)
    xi = rng.integers(-4, 5, size=(M, K))
    W_hat, y, _ = oracle.forward_layer(layer, bits(xi))
    Wi = idx.astype(np.int64).reshape(N, K) - 128
    Wi.reshape(-1)[pos] = np.rint(val * 256).astype(np.int64)
    exact = np.array([[sum(int(a) * int(b) for a, b in zip(xi[m], Wi[n])) for n in range(N)]
                      for m in range(M)])
    assert np.array_equal(y * 256, exact.astype(np.float64))
    assert np.array_equal(W_hat * 256, Wi.astype(np.float32))


# ----------------------------------------------------------------- invariants

@pytest.mark.parametrize("mode", [0, 1])
def test_constant_codebook(mode):
    N, K, M = 50, 64, 2
    c = np.float32(0.0625)
    layer = synthetic.make_layer(mode, N, K, 9, sidecar_count=20)
    layer["codebook"] = np.full_like(layer["codebook"], c)
    x = synthetic.activations(M, K, 9)
    W_hat, y, s = oracle.forward_layer(layer, x)
    xf = oracle.bf16_bits_to_f64(x)
    expect = np.repeat((float(c) * xf.sum(1))[:, None], N, 1)
    K_ = K
    for p, v in zip(layer["sidecar_pos"], layer["sidecar_val"]):
        n, k = int(p) // K_, int(p) % K_
        expect[:, n] += (float(v) - float(c)) * xf[:, k]
    assert np.all(np.abs(y - expect) <= 1e-13 * s)
    untouched = np.setdiff1d(np.arange(N), layer["sidecar_pos"] // K)
    assert untouched.size > 0
    assert np.all(np.abs(y[:, untouched] - float(c) * xf.sum(1)[:, None]) <= 1e-13 * s[:, untouched])


@pytest.mark.parametrize("mode", [0, 1])
def test_one_hot_selects_column(mode):
    N, K = 40, 48
    layer = synthetic.make_layer(mode, N, K, 4, sidecar_count=30)
    W_hat = oracle.decode(layer["mode"], layer["codebook"], layer["indices"],
                          layer["sidecar_pos"], layer["sidecar_val"], N, K)
    for kstar in (0, 1, 17, K - 1):
        x = np.zeros((1, K), np.float32)
        x[0, kstar] = 1.0
        y = oracle.forward(bits(x), W_hat)
        assert np.array_equal(y[0], W_hat[:, kstar].astype(np.float64))


def test_cartesian_product_2d_equals_scalar():
    """cb2[i] = (cb[i & 63], cb[i >> 6]): 2D decode with pair index i must equal
    the scalar decode with indices (i & 63, i >> 6) for the same pair."""
    N, K = 24, 40
    rng = np.random.default_rng(8)
    cb = np.zeros(256, np.float32)
    cb[:64] = rng.normal(0, 0.02, 64).astype(np.float32)
    i = np.arange(4096)
    cb2 = np.stack([cb[i & 63], cb[i >> 6]], 1).reshape(-1)
    j = rng.integers(0, 4096, size=N * K // 2)
    sidx = np.empty(N * K, np.uint8)
    sidx[0::2] = j & 63
    sidx[1::2] = j >> 6
    pos = rng.choice(N * K, size=25, replace=False).astype(np.int64)
    val = rng.normal(0, 0.2, 25).astype(np.float32)
    W2 = oracle.decode(1, cb2, oracle.pack12(j), pos, val, N, K)
    W1 = oracle.decode(0, cb, sidx, pos, val, N, K)
    assert np.array_equal(W1, W2)


def test_sidecar_replaces_exactly():
    N, K = 30, 32
    layer = synthetic.scalar_layer(N, K, 2, sidecar_count=0)
    base = oracle.decode(0, layer["codebook"], layer["indices"], [], [], N, K)
    pos = np.array([0, N * K - 1, 5, 6, 7, K], np.int64)       # first, last, a run, next row
    val = np.array([1.5, -2.5, 0.1, 0.2, 0.3, 7.0], np.float32)
    W = oracle.decode(0, layer["codebook"], layer["indices"], pos, val, N, K)
    assert np.array_equal(W.reshape(-1)[pos], val)
    mask = np.ones(N * K, bool)
    mask[pos] = False
    assert np.array_equal(W.reshape(-1)[mask], base.reshape(-1)[mask])


def test_decode_rejects_bad_sidecar():
    layer = synthetic.scalar_layer(4, 4, 0, sidecar_count=0)
    args = (0, layer["codebook"], layer["indices"])
    with pytest.raises(ValueError):
        oracle.decode(*args, [16], [1.0], 4, 4)
    with pytest.raises(ValueError):
        oracle.decode(*args, [3, 3], [1.0, 2.0], 4, 4)
    with pytest.raises(ValueError):
        oracle.decode(1, np.zeros(8192, np.float32), np.zeros(6, np.uint8), [], [], 2, 6)


def test_forward_rows_matches_full():
    layer = synthetic.vq2d_layer(64, 96, 1, sidecar_count=50)
    x = synthetic.activations(3, 96, 1)
    _, y, s = oracle.forward_layer(layer, x)
    rows = np.array([63, 0, 17, 18, 40])
    yr, sr = oracle.forward_rows(layer, x, rows)
    assert np.array_equal(yr, y[:, rows]) and np.array_equal(sr, s[:, rows])


# ----------------------------------------------------------------- planted mistakes

def _pins_pass():
    try:
        test_pack12_golden_vectors()
        for name in ("tiny_scalar.txt", "tiny_vq2d.txt"):
            test_tiny_layer_golden(name)
        test_cartesian_product_2d_equals_scalar()
        test_one_hot_selects_column(0)
        test_one_hot_selects_column(1)
        test_constant_codebook(0)
        test_dyadic_exact_integer_bruteforce()
        for mode in (0, 1):
            test_bruteforce_tiny(mode, 8, 12, 3)
    except AssertionError:
        return False
    return True


def _unpack_swapped(packed, count):
    i = oracle.hxq_oracle.__dict__["_orig_unpack12"](packed, count)
    out = i.copy()
    out[0::2], out[1::2] = i[1::2], i[0::2]
    return out


def _unpack_big_endian(packed, count):
    b = np.asarray(packed, np.uint8)[: 3 * ((count + 1) // 2)].reshape(-1, 3).astype(np.int64)
    w = (b[:, 0] << 16) | (b[:, 1] << 8) | b[:, 2]
    out = np.empty(2 * w.size, np.int64)
    out[0::2], out[1::2] = w >> 12, w & 0xFFF
    return out[:count]


def _forward_transposed_x(x_bits, W_hat):
    X = oracle.bf16_bits_to_f64(np.atleast_2d(x_bits))
    return X[:, ::-1] @ np.asarray(W_hat, np.float64).T


@pytest.mark.parametrize("mutant", ["swap_pair", "big_endian", "delta_sidecar",
                                    "no_sidecar", "colmajor_sidecar", "swap_2d_components",
                                    "reversed_k"])
def test_planted_mistakes_are_caught(monkeypatch, mutant):
    mod = oracle.hxq_oracle
    assert _pins_pass()
    orig_decode = mod.decode
    monkeypatch.setitem(mod.__dict__, "_orig_unpack12", mod.unpack12)
    if mutant == "swap_pair":
        monkeypatch.setattr(mod, "unpack12", _unpack_swapped)
        monkeypatch.setattr(oracle, "unpack12", _unpack_swapped)
    elif mutant == "big_endian":
        monkeypatch.setattr(mod, "unpack12", _unpack_big_endian)
        monkeypatch.setattr(oracle, "unpack12", _unpack_big_endian)
    elif mutant in ("delta_sidecar", "no_sidecar", "colmajor_sidecar", "swap_2d_components"):
        def bad_decode(mode, cb, idx, pos, val, N, K):
            pos = np.asarray(pos, np.int64)
            val = np.asarray(val, np.float32)
            if mutant == "swap_2d_components" and mode == 1:
                cb = np.asarray(cb, np.float32).reshape(-1, 2)[:, ::-1].reshape(-1)
            W = orig_decode(mode, cb, idx, [], [], N, K)
            if mutant == "delta_sidecar":
                W.reshape(-1)[pos] += val
            elif mutant == "colmajor_sidecar":
                n, k = pos % N, pos // N
                ok = k < K
                W[n[ok], k[ok]] = val[ok]
            elif mutant == "swap_2d_components":
                W.reshape(-1)[pos] = val
            return W
        monkeypatch.setattr(mod, "decode", bad_decode)
        monkeypatch.setattr(oracle, "decode", bad_decode)
    elif mutant == "reversed_k":
        monkeypatch.setattr(mod, "forward", _forward_transposed_x)
        monkeypatch.setattr(oracle, "forward", _forward_transposed_x)
    assert not _pins_pass(), f"planted mistake {mutant} was not caught"
