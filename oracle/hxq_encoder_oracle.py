"""CPU oracle for the HXQ encoder side -- TEST INFRASTRUCTURE.

Only the tests use this module; the CUDA library never imports, links or
calls it, and the two share no code.

The HXQ whitepaper (method section) compresses each weight tensor on its
own, in this order:

1. "Per-tensor k-means": k-means on the weight values (k = 256 entries of
   one weight for scalar VQ, k = 4096 entries of an adjacent pair for 2D VQ)
   gives the codebook; no calibration data is used.
2. "Index assignment": each weight, or pair, gets the index of its nearest
   codebook entry.
3. "Sidecar outlier correction": weights whose reconstruction error exceeds
   a threshold are stored apart, exactly.
4. "12-bit index packing" (2D): two 12-bit indices per 3 bytes, the layout
   the decoder reads (oracle.pack12).

k-means is Lloyd's algorithm: assign every point to its nearest centroid,
move every centroid to the mean of its points, repeat.

Readings where the pages are silent (each is listed in the design notes):
* The initial centroids are an input (the pages name no initialisation; a
  random draw is the caller's, passed in), and the number of Lloyd rounds is
  fixed by the caller: no convergence test, so both sides take the same
  steps.
* Distances are decided in fp32, the precision of the weights and of the
  kernels: for one dimension d = |p - c| (one rounded subtraction); for
  pairs d = dx*dx + dy*dy, each product and the sum rounded to fp32 in that
  order, with no fused multiply-add. Equal distances go to the lowest index.
* A centroid moves to the mean of its points: the exact mean of the points'
  fp32 coordinates (their exact sum over their count, a rational number),
  rounded once to fp32, nearest even; a centroid with no points stays where
  it is. The sums are formed exactly, in integers.
* The sidecar threshold is on |w - w_hat| per weight, in fp32, and strict
  (an error equal to the threshold is not stored). An entry stores the
  weight itself, the replacement form the decoder takes (the whitepaper's
  "(row, col, delta)" wording read as a value that restores w exactly),
  at flat position n*K + k, in ascending order. On a 2D pair each of the
  two weights is tested and stored on its own.

Pins (tests/test_encoder_oracle.py): pure-Python brute force on tiny sets,
the midpoint rule for sorted 1D centroids, scikit-learn's Lloyd k-means
from the same start, the non-increasing objective, weights drawn exactly
from a codebook, planted outliers at dyadic values, and planted mistakes.
"""
from __future__ import annotations

import numpy as np

from .hxq_oracle import MODE_SCALAR8, MODE_VQ2D12, SCALAR_ENTRIES, VQ2D_ENTRIES, pack12

_CHUNK_CELLS = 1 << 22  # points x centroids per block of the distance table


def _as_points(a) -> np.ndarray:
    p = np.asarray(a, dtype=np.float32)
    return p.reshape(-1, 1) if p.ndim == 1 else p


def distances_f32(points, centroids) -> np.ndarray:
    """fp32 distance table [n][k] as the readings define it."""
    p = _as_points(points)
    c = _as_points(centroids)
    if p.shape[1] != c.shape[1] or p.shape[1] not in (1, 2):
        raise ValueError("points and centroids need the same dimension, 1 or 2")
    if p.shape[1] == 1:
        return np.abs(p[:, 0][:, None] - c[:, 0][None, :])  # float32 throughout
    dx = p[:, 0][:, None] - c[:, 0][None, :]
    dy = p[:, 1][:, None] - c[:, 1][None, :]
    return dx * dx + dy * dy  # numpy rounds each float32 operation; nothing is fused


def assign(points, centroids) -> np.ndarray:
    """Index assignment: the nearest centroid of each point (int64), fp32
    distances, lowest index on ties (argmin returns the first minimum)."""
    p = _as_points(points)
    c = _as_points(centroids)
    out = np.empty(p.shape[0], dtype=np.int64)
    step = max(1, _CHUNK_CELLS // max(1, c.shape[0]))
    for i in range(0, p.shape[0], step):
        out[i:i + step] = np.argmin(distances_f32(p[i:i + step], c), axis=1)
    return out


def round_rational_f32(num: int, den: int) -> np.float32:
    """The fp32 value nearest to the rational num / den (den > 0), ties to
    the even significand (IEEE 754 round to nearest even), subnormals
    included; exact integer arithmetic throughout."""
    num, den = int(num), int(den)
    if den <= 0:
        raise ValueError("den must be positive")
    if num == 0:
        return np.float32(0.0)
    a = abs(num)
    # 2^E <= a / den < 2^(E + 1)
    E = a.bit_length() - den.bit_length()
    if (a << max(0, -E)) < (den << max(0, E)):
        E -= 1
    lsb = max(E - 23, -149)  # weight of the significand's last bit
    if lsb >= 0:
        d = den << lsb
        q, r = divmod(a, d)
    else:
        d = den
        q, r = divmod(a << -lsb, den)
    if 2 * r > d or (2 * r == d and q & 1):
        q += 1
    v = float(q) * 2.0 ** lsb  # exact: q <= 2^24 and 2^lsb >= 2^-149
    return np.float32(-v if num < 0 else v)


def f32_integer_parts(v):
    """(m, e) with v = m * 2^e exactly, m a signed int64 (|m| < 2^24) and e
    the exponent of the last significand bit (-149 for subnormals)."""
    bits = np.ascontiguousarray(v, dtype=np.float32).view(np.uint32).astype(np.int64)
    ef = (bits >> 23) & 0xFF
    frac = bits & 0x7FFFFF
    m = np.where(ef == 0, frac, frac | 0x800000)
    m = np.where(bits >> 31 != 0, -m, m)
    e = np.where(ef == 0, -149, ef - 150)
    return m, e


def exact_sums(values, labels, k):
    """Exact sum of the fp32 values of each label 0..k-1, as Python integers
    in units of 2^-149 (every fp32 value is an integer multiple of 2^-149).
    The signed mantissas are split into 12-bit halves and added per (label,
    exponent) bin with float64 weights: a bin of at most 2^31 values sums
    to under 2^43 in magnitude, so float64 adds those integers exactly; each
    bin's sum is then shifted into place as a Python integer."""
    m, e = f32_integer_parts(values)
    lab = np.asarray(labels, dtype=np.int64)
    if lab.size >= 1 << 31:
        raise ValueError("too many points for exact float64 bins")
    key = lab * 256 + (e + 149)
    sgn = np.sign(m)
    a = np.abs(m)
    lo = np.bincount(key, weights=(sgn * (a & 0xFFF)).astype(np.float64), minlength=k * 256)
    hi = np.bincount(key, weights=(sgn * (a >> 12)).astype(np.float64), minlength=k * 256)
    out = [0] * k
    for b in np.flatnonzero((lo != 0) | (hi != 0)).tolist():
        out[b >> 8] += ((int(hi[b]) << 12) + int(lo[b])) << (b & 255)
    return out


def kmeans_update(points, labels, centroids) -> np.ndarray:
    """Each centroid moves to the mean of its points: their exact sum over
    their count, rounded once to fp32 (nearest even); one without points
    keeps its position."""
    p = _as_points(points)
    c = _as_points(centroids)
    k, dim = c.shape
    labels = np.asarray(labels, dtype=np.int64)
    count = np.bincount(labels, minlength=k)
    new = c.copy()
    for d in range(dim):
        sums = exact_sums(p[:, d], labels, k)
        for j in np.flatnonzero(count > 0).tolist():
            new[j, d] = round_rational_f32(sums[j], int(count[j]) << 149)
    return new


def kmeans(points, init, iters: int) -> tuple[np.ndarray, np.ndarray]:
    """Lloyd's k-means from `init` for `iters` rounds; returns the centroids
    (fp32, shaped like init) and the assignment to them."""
    c = _as_points(init).copy()
    p = _as_points(points)
    for _ in range(int(iters)):
        c = kmeans_update(p, assign(p, c), c)
    labels = assign(p, c)
    return c.reshape(np.shape(init)), labels


def inertia(points, centroids, labels) -> float:
    """Sum of squared distances to the assigned centroids, in float64."""
    p = _as_points(points).astype(np.float64)
    c = _as_points(centroids).astype(np.float64)
    return float(np.sum((p - c[np.asarray(labels, dtype=np.int64)]) ** 2))


def sidecar_select(W, W_hat, threshold: float) -> tuple[np.ndarray, np.ndarray]:
    """Sidecar outlier correction: flat positions (ascending, int64) where
    |w - w_hat| > threshold in fp32, and the weights there (the values that
    replace the decoded ones)."""
    w = np.asarray(W, dtype=np.float32).reshape(-1)
    wh = np.asarray(W_hat, dtype=np.float32).reshape(-1)
    err = np.abs(w - wh)
    pos = np.nonzero(err > np.float32(threshold))[0].astype(np.int64)
    return pos, w[pos].copy()


def encode(W, mode: int, codebook, threshold: float):
    """Steps 2-4 for a trained codebook: W fp32 [N][K] -> (index bytes in the
    decoder's layout, sidecar positions, sidecar values)."""
    W = np.asarray(W, dtype=np.float32)
    N, K = W.shape
    cb = np.asarray(codebook, dtype=np.float32).reshape(-1)
    if mode == MODE_SCALAR8:
        if cb.size != SCALAR_ENTRIES:
            raise ValueError("scalar mode needs 256 codebook entries")
        lab = assign(W.reshape(-1), cb)
        indices = lab.astype(np.uint8)
        W_hat = cb[lab].reshape(N, K)
    elif mode == MODE_VQ2D12:
        if K % 4 or cb.size != 2 * VQ2D_ENTRIES:
            raise ValueError("2D mode needs K % 4 == 0 and 4096 pairs")
        pairs = cb.reshape(VQ2D_ENTRIES, 2)
        lab = assign(W.reshape(-1, 2), pairs)
        indices = pack12(lab)
        W_hat = pairs[lab].reshape(N, K)
    else:
        raise ValueError(f"unknown mode {mode}")
    pos, val = sidecar_select(W, W_hat, threshold)
    return indices, pos, val
