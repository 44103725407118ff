"""Seeded synthetic HelixLinear layers and activations.

This module only draws random inputs. It holds none of the codec's arithmetic:
no decoding, no unpacking, no packing, no matrix products. Both the CPU oracle
(through the tests) and the CUDA path consume exactly what it returns.

The layer shapes and value distributions stand in for the compressed
checkpoints the pages describe, which are not available here:

* scalar mode: a 256-entry fp32 codebook plus one uint8 index per weight
  (Zamba2-1.2B-HXQ model card, "What is HelixCode?");
* 2D mode: a 4096-entry codebook of fp32 pairs, one 12-bit index per pair of
  adjacent weights, two indices per 3 bytes (HXQ whitepaper, method section,
  "2D VQ" paragraph and the "12-bit index packing" pipeline step);
* sparse sidecar of outlier values (HXQ whitepaper, method section,
  "Sidecar outlier correction" step).

Uniformly random 12-bit indices packed two per 3 bytes are exactly uniformly
random bytes, so the 2D generator draws the packed stream directly and never
packs anything itself.
"""
from __future__ import annotations

import numpy as np

MODE_SCALAR8 = 0
MODE_VQ2D12 = 1


def _rng(*key: int) -> np.random.Generator:
    return np.random.default_rng(np.random.SeedSequence([int(k) & 0xFFFFFFFF for k in key]))


def _sidecar(rng, N, K, count, sigma):
    count = int(min(count, N * K))
    pos = rng.choice(N * K, size=count, replace=False).astype(np.int64)
    val = rng.normal(0.0, sigma, size=count).astype(np.float32)
    return pos, val


def _sidecar_count(N, K, density, count):
    if count is not None:
        return int(count)
    return int(round(density * N * K))


def scalar_layer(N, K, seed=0, *, cb_sigma=0.02, index_dist="gauss",
                 sidecar_density=0.001, sidecar_count=None, sidecar_sigma=0.15):
    """Scalar-mode layer: codebook f32[256] (sorted N(0, cb_sigma) draws),
    indices u8[N*K] row-major ([out][in]), sidecar (flat n*K+k, f32 value).

    index_dist "uniform" draws indices uniformly over 0..255; "gauss" draws a
    discretised Gaussian clamp(rint(127.5 + 42.5 z), 0, 255), so that +-3
    sigma spans the codebook.
    """
    rng = _rng(seed, 1, N, K)
    codebook = np.sort(rng.normal(0.0, cb_sigma, size=256)).astype(np.float32)
    if index_dist == "uniform":
        indices = rng.integers(0, 256, size=N * K, dtype=np.uint8)
    elif index_dist == "gauss":
        z = rng.standard_normal(size=N * K, dtype=np.float32)
        indices = np.clip(np.rint(127.5 + 42.5 * z), 0, 255).astype(np.uint8)
    else:
        raise ValueError(index_dist)
    pos, val = _sidecar(rng, N, K, _sidecar_count(N, K, sidecar_density, sidecar_count),
                        sidecar_sigma)
    return dict(mode=MODE_SCALAR8, N=N, K=K, codebook=codebook, indices=indices,
                sidecar_pos=pos, sidecar_val=val)


def vq2d_layer(N, K, seed=0, *, cb_sigma=0.02, sidecar_density=0.0005,
               sidecar_count=None, sidecar_sigma=0.15):
    """2D-mode layer: codebook f32[4096*2] (pair-interleaved, each component
    N(0, cb_sigma)), packed index stream u8[3*N*K/4] (uniform bytes, i.e.
    uniform 12-bit indices), sidecar as in scalar mode. K must be a multiple
    of 4 so that every row is a whole number of 3-byte groups."""
    if K % 4:
        raise ValueError("2D mode needs K % 4 == 0")
    rng = _rng(seed, 2, N, K)
    codebook = rng.normal(0.0, cb_sigma, size=4096 * 2).astype(np.float32)
    indices = rng.integers(0, 256, size=3 * N * K // 4, dtype=np.uint8)
    pos, val = _sidecar(rng, N, K, _sidecar_count(N, K, sidecar_density, sidecar_count),
                        sidecar_sigma)
    return dict(mode=MODE_VQ2D12, N=N, K=K, codebook=codebook, indices=indices,
                sidecar_pos=pos, sidecar_val=val)


def f32_to_bf16_bits(a: np.ndarray) -> np.ndarray:
    """Round fp32 to bf16 (round-to-nearest-even) with torch's conversion and
    return the raw uint16 bit patterns."""
    import torch
    t = torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).to(torch.bfloat16)
    return t.view(torch.int16).numpy().view(np.uint16).copy()


def activations(M, K, seed=0, sigma=1.0) -> np.ndarray:
    """x as bf16 bit patterns u16[M][K], drawn N(0, sigma) in fp32 then rounded."""
    rng = _rng(seed, 3, M, K)
    return f32_to_bf16_bits(rng.normal(0.0, sigma, size=(M, K)).astype(np.float32))


# The five workloads, restated: (name, mode, N, K, Ms, layer kwargs).
# Shapes: Mamba2-1.3B in/out projections (hidden 2048, Mamba2-1.3B-HXQ model
# card), the Qwen2.5-3B layer set with 2 KV heads (Qwen2.5-3B-Instruct-HXQ
# model card), a 2D-VQ 11008x4096 layer, and Zamba2-7B-like MLP widths.
CONFIGS = {
    "tiny": [
        ("tiny", MODE_SCALAR8, 256, 256, (1, 4),
         dict(index_dist="uniform", sidecar_count=64, sidecar_sigma=0.2)),
    ],
    "mamba2": [
        ("in_proj", MODE_SCALAR8, 8512, 2048, (1,), dict()),
        ("out_proj", MODE_SCALAR8, 2048, 4096, (1,), dict()),
    ],
    "qwen25_3b": [
        ("q", MODE_SCALAR8, 2048, 2048, (1, 8, 32), dict()),
        ("k", MODE_SCALAR8, 256, 2048, (1, 8, 32), dict()),
        ("v", MODE_SCALAR8, 256, 2048, (1, 8, 32), dict()),
        ("o", MODE_SCALAR8, 2048, 2048, (1, 8, 32), dict()),
        ("gate", MODE_SCALAR8, 11008, 2048, (1, 8, 32), dict()),
        ("up", MODE_SCALAR8, 11008, 2048, (1, 8, 32), dict()),
        ("down", MODE_SCALAR8, 2048, 11008, (1, 8, 32), dict()),
    ],
    "vq2d": [
        ("vq2d", MODE_VQ2D12, 11008, 4096, (1, 4, 16), dict()),
    ],
    "prefill": [
        ("mlp_up", MODE_SCALAR8, 14336, 3584, (512, 2048), dict(cb_sigma=0.015)),
        ("mlp_down", MODE_SCALAR8, 3584, 14336, (512, 2048), dict(cb_sigma=0.015)),
    ],
}


def make_layer(mode, N, K, seed=0, **kw):
    if mode == MODE_SCALAR8:
        return scalar_layer(N, K, seed, **kw)
    return vq2d_layer(N, K, seed, **kw)


def config_layers(config: str, seed: int = 0):
    """Yield (name, layer dict, Ms) for one named workload."""
    for li, (name, mode, N, K, Ms, kw) in enumerate(CONFIGS[config]):
        yield name, make_layer(mode, N, K, seed * 1000 + li, **kw), Ms
