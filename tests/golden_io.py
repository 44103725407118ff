"""Reader for the hand-worked fixtures under tests/golden/."""
import os

import numpy as np

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def _lines(name):
    with open(os.path.join(GOLDEN, name)) as f:
        for raw in f:
            line = raw.split("#", 1)[0].strip()
            if line:
                yield line


def hex_table(name):
    return [[int(t, 16) for t in line.split()] for line in _lines(name)]


def tiny_layer(name):
    kv = {}
    for line in _lines(name):
        key, val = line.split(":", 1)
        kv[key.strip()] = val.split()
    mode, N, K = int(kv["mode"][0]), int(kv["N"][0]), int(kv["K"][0])
    if mode == 0:
        cb = np.zeros(256, np.float32)
        vals = [float(v) for v in kv["codebook"]]
        cb[: len(vals)] = vals
        idx = np.array([int(v) for v in kv["indices"]], np.uint8)
    else:
        cb = np.zeros(4096 * 2, np.float32)
        for ent in kv["codebook"]:
            i, c = ent.split(":")
            c0, c1 = (float(t) for t in c.split(","))
            cb[2 * int(i, 16)] = c0
            cb[2 * int(i, 16) + 1] = c1
        idx = np.array([int(v, 16) for v in kv["indices_hex"]], np.uint8)
    f = lambda k: np.array([float(v) for v in kv[k]])
    layer = dict(mode=mode, N=N, K=K, codebook=cb, indices=idx,
                 sidecar_pos=np.array([int(v) for v in kv["sidecar_pos"]], np.int64),
                 sidecar_val=f("sidecar_val").astype(np.float32))
    M = f("x").size // K
    return layer, f("x").reshape(M, K), f("W").reshape(N, K), f("y").reshape(M, N), f("s").reshape(M, N)
