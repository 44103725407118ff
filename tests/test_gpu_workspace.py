"""Device memory of a handle and the tensor-core workspace per (device,
stream): a handle holds its compressed layer plus a small GEMV workspace, so
that a whole model's layers fit next to each other; tensor-core forwards of
different handles on one stream, and on two streams at once, stay exact
against the oracle."""
import numpy as np
import pytest

import oracle
import synthetic

pytestmark = pytest.mark.gpu

TAU_TC = 8e-3  # bf16 weights above 32 tokens, times sum |x||w|


def _footprint_bound(layer, num_sms):
    """Bytes a handle may hold: indices padded to whole 64-weight stages,
    12 B per sidecar entry, row and stage patch offsets, codebook, status,
    GEMV workspace (2 x 8 x 128 floats per SM) and the stream-K counters,
    each allocation rounded up to 2 MiB."""
    N, K = layer["N"], layer["K"]
    Kp = (K + 63) // 64 * 64
    n_tiles = (N + 127) // 128
    sizes = [N * Kp if layer["mode"] == 0 else 3 * N * Kp // 4, 4 * layer["sidecar_pos"].size,
             4 * layer["sidecar_pos"].size, 4 * layer["sidecar_pos"].size, 4 * (N + 1), 4 * (Kp // 64 + 1) * N,
             1024 if layer["mode"] == 0 else 32768, 4, 4 * num_sms * 2 * 8 * 128, 4 * n_tiles * 64 * 4]
    mib2 = 2 << 20
    return sum((s + mib2 - 1) // mib2 * mib2 for s in sizes)


def test_many_handles_fit(hxq):
    """256 Qwen2.5-3B q-shaped handles (2048 x 2048, 0.1 % sidecar): each
    holds its compressed layer and a small workspace, not a tensor-core
    workspace of its own."""
    import torch
    layer = synthetic.make_layer(0, 2048, 2048, 5, sidecar_count=2048 * 2048 // 1000)
    num_sms = torch.cuda.get_device_properties(0).multi_processor_count
    torch.cuda.synchronize()
    free0, _ = torch.cuda.mem_get_info()
    lins = [hxq.HelixLinear.from_layer(layer) for _ in range(256)]
    torch.cuda.synchronize()
    free1, _ = torch.cuda.mem_get_info()
    per_handle = (free0 - free1) / 256
    assert per_handle <= _footprint_bound(layer, num_sms), per_handle
    for lin in lins:
        lin.close()


def _check(y, x, W, what):
    y_ref, s = oracle.forward(x, W), oracle.abs_scale(x, W)
    err = np.abs(y.cpu().numpy().astype(np.float64) - y_ref)
    assert np.all(err <= TAU_TC * s), f"{what}: max err/s {np.max(err / s):.3e}"


@pytest.mark.parametrize("M", [64, 600])
def test_two_handles_one_stream_and_two_streams(hxq, M):
    """Tensor-core forwards of two handles back to back on one stream (the
    stream's workspace serves both in turn), then on two streams at once
    (each stream has its own workspace)."""
    import torch
    layers = [synthetic.make_layer(0, 1000 + 200 * i, 1024, 60 + i, sidecar_count=2000) for i in range(2)]
    Ws = [oracle.decode(0, l["codebook"], l["indices"], l["sidecar_pos"], l["sidecar_val"], l["N"], 1024)
          for l in layers]
    lins = [hxq.HelixLinear.from_layer(l) for l in layers]
    xs = [synthetic.activations(M, 1024, 70 + i) for i in range(2)]
    xd = [torch.from_numpy(x.view(np.int16)).cuda() for x in xs]
    s1 = torch.cuda.Stream()
    ys = [torch.full((M, l["N"]), float("nan"), device="cuda") for l in layers]
    for i in range(2):
        lins[i].forward(xd[i], ys[i], stream=s1)
    s1.synchronize()
    for i in range(2):
        _check(ys[i], xs[i], Ws[i], f"one stream, layer {i}")
    s2 = torch.cuda.Stream()
    ys = [torch.full((M, l["N"]), float("nan"), device="cuda") for l in layers]
    for _ in range(3):
        lins[0].forward(xd[0], ys[0], stream=s1)
        lins[1].forward(xd[1], ys[1], stream=s2)
    torch.cuda.synchronize()
    for i in range(2):
        lins[i].check()
        _check(ys[i], xs[i], Ws[i], f"two streams, layer {i}")
    for lin in lins:
        lin.close()
