"""ctypes wrapper of the plain C++ oracle (oracle/hxq_oracle_ref.cpp) --
TEST INFRASTRUCTURE, used only by the tests to check it against the numpy
oracle. build() compiles it with the host C++ compiler next to its source;
the CUDA library never loads it."""
from __future__ import annotations

import ctypes
import os
import shutil
import subprocess

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "hxq_oracle_ref.cpp")
LIB = os.path.join(HERE, "libhxq_oracle_ref.so")
_lib = None


def build() -> str:
    """Compile the oracle (no fused multiply-add contraction, so every
    product and sum is rounded as written)."""
    cxx = os.environ.get("CXX") or shutil.which("g++") or shutil.which("c++")
    if not cxx:
        raise RuntimeError("no host C++ compiler")
    tmp = LIB + ".tmp"
    subprocess.run([cxx, "-O2", "-std=c++17", "-ffp-contract=off", "-fPIC", "-shared", "-pthread", SRC, "-o", tmp],
                   check=True)
    os.replace(tmp, LIB)
    return LIB


def _load():
    global _lib
    if _lib is None:
        if not os.path.exists(LIB) or os.path.getmtime(LIB) < os.path.getmtime(SRC):
            build()
        lib = ctypes.CDLL(LIB)
        vp, i, i64 = ctypes.c_void_p, ctypes.c_int, ctypes.c_int64
        lib.oracle_decode.argtypes = [i, vp, vp, vp, vp, i64, i, i, vp]
        lib.oracle_decode.restype = i
        lib.oracle_forward.argtypes = [vp, vp, i, i, i, vp, vp]
        lib.oracle_forward.restype = None
        lib.oracle_assign.argtypes = [vp, i64, i, vp, i, vp]
        lib.oracle_assign.restype = None
        lib.oracle_assign_threads.argtypes = [vp, i64, i, vp, i, vp, i]
        lib.oracle_assign_threads.restype = None
        lib.oracle_kmeans_update.argtypes = [vp, i64, i, vp, i, vp]
        lib.oracle_kmeans_update.restype = None
        lib.oracle_sidecar_select.argtypes = [vp, vp, i64, ctypes.c_float, vp, vp, i64]
        lib.oracle_sidecar_select.restype = i64
        _declare_rows(lib)
        _lib = lib
    return _lib


def _declare_rows(lib):
    vp, i, i64 = ctypes.c_void_p, ctypes.c_int, ctypes.c_int64
    lib.oracle_forward_rows.argtypes = [i, vp, vp, vp, vp, i64, i, i, vp, i, i, i, i, vp]
    lib.oracle_forward_rows.restype = i


def load_timing_build(out_dir):
    """The same oracle compiled for timing on this host (-O3 -march=native,
    still without fused multiply-add) into out_dir; returns the loaded
    library. Used by bench.py's CPU baseline leg only."""
    cxx = os.environ.get("CXX") or shutil.which("g++") or shutil.which("c++")
    if not cxx:
        raise RuntimeError("no host C++ compiler")
    os.makedirs(out_dir, exist_ok=True)
    path = os.path.join(out_dir, "libhxq_oracle_timing.so")
    subprocess.run([cxx, "-O3", "-march=native", "-std=c++17", "-ffp-contract=off", "-fPIC", "-shared", "-pthread",
                    SRC, "-o", path], check=True)
    lib = ctypes.CDLL(path)
    _declare_rows(lib)
    return lib


def _p(a):
    return None if a is None else a.ctypes.data


def decode(mode, codebook, indices, sidecar_pos, sidecar_val, N, K) -> np.ndarray:
    cb = np.ascontiguousarray(codebook, dtype=np.float32)
    idx = np.ascontiguousarray(indices, dtype=np.uint8)
    pos = np.ascontiguousarray(sidecar_pos, dtype=np.int64).reshape(-1)
    val = np.ascontiguousarray(sidecar_val, dtype=np.float32).reshape(-1)
    W = np.empty((N, K), dtype=np.float32)
    rc = _load().oracle_decode(int(mode), _p(cb), _p(idx), _p(pos), _p(val), int(pos.size), int(N), int(K), _p(W))
    if rc != 0:
        raise ValueError("invalid layer")
    return W


def forward(x_bits, W) -> tuple[np.ndarray, np.ndarray]:
    x = np.ascontiguousarray(np.atleast_2d(x_bits), dtype=np.uint16)
    W = np.ascontiguousarray(W, dtype=np.float32)
    M, K = x.shape
    N = W.shape[0]
    y = np.empty((M, N), np.float64)
    s = np.empty((M, N), np.float64)
    _load().oracle_forward(_p(x), _p(W), int(M), int(N), int(K), _p(y), _p(s))
    return y, s


def _pts(a):
    p = np.ascontiguousarray(a, dtype=np.float32)
    return p.reshape(-1, 1) if p.ndim == 1 else p


def assign(points, centroids, threads=1) -> np.ndarray:
    p, c = _pts(points), _pts(centroids)
    lab = np.empty(p.shape[0], np.int32)
    if threads > 1:
        _load().oracle_assign_threads(_p(p), int(p.shape[0]), int(p.shape[1]), _p(c), int(c.shape[0]), _p(lab),
                                      int(threads))
    else:
        _load().oracle_assign(_p(p), int(p.shape[0]), int(p.shape[1]), _p(c), int(c.shape[0]), _p(lab))
    return lab.astype(np.int64)


def kmeans_update(points, labels, centroids) -> np.ndarray:
    p, c = _pts(points), _pts(centroids).copy()
    lab = np.ascontiguousarray(labels, dtype=np.int32)
    _load().oracle_kmeans_update(_p(p), int(p.shape[0]), int(p.shape[1]), _p(lab), int(c.shape[0]), _p(c))
    return c


def kmeans(points, init, iters):
    c = _pts(init).copy()
    for _ in range(int(iters)):
        c = kmeans_update(points, assign(points, c), c)
    return c.reshape(np.shape(init)), assign(points, c)


def sidecar_select(W, W_hat, threshold):
    w = np.ascontiguousarray(W, dtype=np.float32).reshape(-1)
    wh = np.ascontiguousarray(W_hat, dtype=np.float32).reshape(-1)
    pos = np.empty(w.size, np.int64)
    val = np.empty(w.size, np.float32)
    n = _load().oracle_sidecar_select(_p(w), _p(wh), int(w.size), float(threshold), _p(pos), _p(val), int(w.size))
    return pos[:n].copy(), val[:n].copy()


def forward_rows(layer, x_bits, r0, r1, threads=1, lib=None):
    """y[:, r0:r1] of the layer's forward (decode with the sidecar, then the
    float64 dot products), computed by oracle_forward_rows on `threads`
    host threads."""
    L = lib or _load()
    x = np.ascontiguousarray(np.atleast_2d(x_bits), dtype=np.uint16)
    cb = np.ascontiguousarray(layer["codebook"], dtype=np.float32)
    idx = np.ascontiguousarray(layer["indices"], dtype=np.uint8)
    pos = np.ascontiguousarray(layer["sidecar_pos"], dtype=np.int64).reshape(-1)
    val = np.ascontiguousarray(layer["sidecar_val"], dtype=np.float32).reshape(-1)
    M = x.shape[0]
    y = np.empty((M, r1 - r0), np.float64)
    rc = L.oracle_forward_rows(int(layer["mode"]), _p(cb), _p(idx), _p(pos), _p(val), int(pos.size), int(layer["N"]),
                               int(layer["K"]), _p(x), int(M), int(r0), int(r1), int(threads), _p(y))
    if rc != 0:
        raise ValueError("invalid layer or rows")
    return y
