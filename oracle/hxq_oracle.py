"""CPU oracle for the HXQ HelixLinear forward y = x . W^T -- TEST INFRASTRUCTURE.

Only the tests, the smoke check and the benchmark's CPU-baseline leg use this
module. The product path (the CUDA library and its Python binding) never
imports, links or calls it, and it shares no code with them.

What it computes, written out as the plain definition in float64:

1. Decode the weight matrix W_hat [N out][K in] from its compressed form:
   * scalar mode: W_hat[n, k] = codebook[indices[n*K + k]], a 256-entry fp32
     codebook addressed by one uint8 per weight (Zamba2-1.2B-HXQ model card,
     "What is HelixCode?": codebook + uint8 index matrix, forward computes
     codebook[indices] against x);
   * 2D mode: adjacent weights (k, k+1), k even, of one row form a pair that
     is one entry of a 4096-entry codebook of fp32 pairs; the 12-bit pair
     indices are stored two per 3 bytes (HXQ whitepaper, method section: the
     "Per-tensor k-means" step with k=4096 for 2D VQ, the "12-bit index
     packing" step, and the 2D VQ paragraph: pairs of adjacent weights, 12
     bits per pair, 6 bits per weight).
2. Apply the sidecar: each (flat position p = n*K + k, fp32 value v) replaces
   W_hat[n, k] by v (HXQ whitepaper, method section, "Sidecar outlier
   correction" step; the replacement reading is the one adopted, see below).
3. y[m, n] = sum_k x[m, k] * W_hat[n, k] in float64, x given as bf16 bit
   patterns and widened exactly.
4. The per-output tolerance scale s[m, n] = sum_k |x[m, k]| * |W_hat[n, k]|.

Readings where the pages are silent (each is listed in the design notes):
* W is [out][in] row-major, as for any nn.Linear weight, and y = x . W^T.
* 12-bit packing: the two indices of a 3-byte group form one 24-bit
  little-endian word b0 | b1<<8 | b2<<16; the first index of the group is
  its low 12 bits, the second its high 12 bits. Groups run over one flat
  stream of pairs in row-major order (pair g = n*K/2 + k/2). With K % 4 == 0
  every row is a whole number of groups.
* 2D codebook layout: fp32 [4096][2]; component 0 goes to the even column.
* The sidecar replaces the decoded value (the whitepaper's text speaks of
  (row, col, delta) triplets; the (flat position, value) replacement form is
  the contract this library implements). A sidecar entry on a 2D weight
  replaces that single scalar.
* The bf16 weight variant rounds W_hat to bf16 with round-to-nearest-even,
  ties to even, written from the IEEE-754 definition.

Pins (tests/test_oracle.py): hand-derived golden vectors for the packing and
for two tiny layers (tests/golden/), exact integer brute force, pure-Python
loops on tiny shapes, the constant-codebook, one-hot and Cartesian-product
invariants, and torch's bf16 conversion for the rounding.
"""
from __future__ import annotations

import numpy as np

MODE_SCALAR8 = 0
MODE_VQ2D12 = 1
SCALAR_ENTRIES = 256
VQ2D_ENTRIES = 4096


def bf16_bits_to_f64(bits: np.ndarray) -> np.ndarray:
    """Widen bf16 bit patterns exactly: a bf16 is the top half of an fp32."""
    b = np.asarray(bits, dtype=np.uint16).astype(np.uint32) << np.uint32(16)
    return b.view(np.float32).astype(np.float64)


def unpack12(packed: np.ndarray, count: int) -> np.ndarray:
    """3-byte groups -> 12-bit indices (little-endian 24-bit word, first index
    in the low 12 bits). Returns `count` indices as int64."""
    packed = np.asarray(packed, dtype=np.uint8)
    groups = (count + 1) // 2
    b = packed[: 3 * groups].reshape(groups, 3).astype(np.int64)
    word = b[:, 0] | (b[:, 1] << 8) | (b[:, 2] << 16)
    out = np.empty(2 * groups, dtype=np.int64)
    out[0::2] = word & 0xFFF
    out[1::2] = word >> 12
    return out[:count]


def pack12(idx: np.ndarray) -> np.ndarray:
    """Encoder side of the same packing: 12-bit indices (even count) -> bytes.
    Used by tests to build 2D layers with chosen indices."""
    idx = np.asarray(idx, dtype=np.int64)
    if idx.size % 2 or (idx.size and (idx.min() < 0 or idx.max() > 0xFFF)):
        raise ValueError("pack12 needs an even number of indices in 0..4095")
    word = idx[0::2] | (idx[1::2] << 12)
    out = np.empty((word.size, 3), dtype=np.uint8)
    out[:, 0] = word & 0xFF
    out[:, 1] = (word >> 8) & 0xFF
    out[:, 2] = (word >> 16) & 0xFF
    return out.reshape(-1)


def decode(mode: int, codebook, indices, sidecar_pos, sidecar_val, N: int, K: int) -> np.ndarray:
    """Decoded weights W_hat as fp32 [N][K], sidecar applied (steps 1-2)."""
    codebook = np.asarray(codebook, dtype=np.float32)
    indices = np.asarray(indices, dtype=np.uint8)
    if mode == MODE_SCALAR8:
        if codebook.size != SCALAR_ENTRIES or indices.size != N * K:
            raise ValueError("scalar mode: 256 codebook entries and N*K indices")
        W = codebook[indices.astype(np.int64).reshape(N, K)]
    elif mode == MODE_VQ2D12:
        if K % 4 or codebook.size != 2 * VQ2D_ENTRIES or indices.size != 3 * N * K // 4:
            raise ValueError("2D mode: K % 4 == 0, 4096x2 codebook, 3*N*K/4 bytes")
        pairs = codebook.reshape(VQ2D_ENTRIES, 2)
        j = unpack12(indices, N * K // 2).reshape(N, K // 2)
        W = np.empty((N, K), dtype=np.float32)
        W[:, 0::2] = pairs[j, 0]
        W[:, 1::2] = pairs[j, 1]
    else:
        raise ValueError(f"unknown mode {mode}")
    pos = np.asarray(sidecar_pos, dtype=np.int64).reshape(-1)
    val = np.asarray(sidecar_val, dtype=np.float32).reshape(-1)
    if pos.size != val.size:
        raise ValueError("sidecar positions and values differ in length")
    if pos.size:
        if pos.min() < 0 or pos.max() >= N * K:
            raise ValueError("sidecar position out of range")
        if np.unique(pos).size != pos.size:
            raise ValueError("duplicate sidecar position")
        W.reshape(-1)[pos] = val
    return W


def forward(x_bits, W_hat) -> np.ndarray:
    """y[m, n] = sum_k x[m, k] * W_hat[n, k] in float64 (step 3)."""
    X = bf16_bits_to_f64(np.atleast_2d(x_bits))
    return X @ np.asarray(W_hat, dtype=np.float32).astype(np.float64).T


def abs_scale(x_bits, W_hat) -> np.ndarray:
    """s[m, n] = sum_k |x[m, k]| * |W_hat[n, k]| in float64 (step 4)."""
    X = np.abs(bf16_bits_to_f64(np.atleast_2d(x_bits)))
    return X @ np.abs(np.asarray(W_hat, dtype=np.float32).astype(np.float64)).T


def round_to_bf16(a) -> np.ndarray:
    """fp32 -> nearest bf16 value (ties to even), returned as fp32.

    From the IEEE-754 definition on the bit pattern: keep the top 16 bits and
    add one unit in their last place when the dropped 16 bits exceed half a
    unit, or equal half a unit and the kept part is odd. NaNs stay NaN (quiet
    bit set); infinities and overflow to infinity follow from the same
    carry into the exponent field.
    """
    u = np.ascontiguousarray(a, dtype=np.float32).view(np.uint32).astype(np.uint64)
    low = u & 0xFFFF
    keep = u >> 16
    half = np.uint64(0x8000)
    round_up = (low > half) | ((low == half) & ((keep & 1) == 1))
    r = (keep + round_up.astype(np.uint64)) << 16
    is_nan = ((u & 0x7F800000) == 0x7F800000) & ((u & 0x007FFFFF) != 0)
    r = np.where(is_nan, (keep | 0x0040) << 16, r)
    return r.astype(np.uint32).view(np.float32)


def forward_layer(layer: dict, x_bits) -> tuple[np.ndarray, np.ndarray, np.ndarray]:
    """Convenience: decode a layer dict and return (W_hat, y, s)."""
    W = decode(layer["mode"], layer["codebook"], layer["indices"], layer["sidecar_pos"],
               layer["sidecar_val"], layer["N"], layer["K"])
    return W, forward(x_bits, W), abs_scale(x_bits, W)


def forward_rows(layer: dict, x_bits, rows: np.ndarray) -> tuple[np.ndarray, np.ndarray]:
    """y and s restricted to output rows `rows`, decoding only those rows.

    Same definition as decode() + forward(); used where the full matrix is too
    large to decode on the CPU in the time a test allows.
    """
    N, K, mode = layer["N"], layer["K"], layer["mode"]
    rows = np.asarray(rows, dtype=np.int64)
    cb = np.asarray(layer["codebook"], dtype=np.float32)
    idx = np.asarray(layer["indices"], dtype=np.uint8)
    if mode == MODE_SCALAR8:
        W = cb[idx.reshape(N, K)[rows].astype(np.int64)]
    else:
        rb = 3 * K // 4
        sel = idx.reshape(N, rb)[rows].reshape(-1)
        j = unpack12(sel, rows.size * K // 2).reshape(rows.size, K // 2)
        pairs = cb.reshape(VQ2D_ENTRIES, 2)
        W = np.empty((rows.size, K), dtype=np.float32)
        W[:, 0::2] = pairs[j, 0]
        W[:, 1::2] = pairs[j, 1]
    pos = np.asarray(layer["sidecar_pos"], dtype=np.int64)
    val = np.asarray(layer["sidecar_val"], dtype=np.float32)
    prow = pos // K
    hit = np.isin(prow, rows)
    order = np.argsort(rows, kind="stable")
    i = order[np.searchsorted(rows[order], prow[hit])]
    W[i, pos[hit] % K] = val[hit]
    return forward(x_bits, W), abs_scale(x_bits, W)
