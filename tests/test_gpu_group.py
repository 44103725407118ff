"""Grouped forward (hxq_group_*): layers that read the same activations, one
launch for M <= 4, against the CPU oracle layer by layer.

Each layer of a group has its own codebook, sidecar and output; the tests
build every layer from its own seed so that a kernel picking up the wrong
layer's codebook, sidecar or row count fails. The shapes reach both ways the
grouped GEMV cuts its grid: one cluster of CTAs per 128-row tile when the
tiles of all layers fill most of the GPU that way, stream-K shares in
proportion to each layer's weights otherwise (small groups, and groups with
more tiles than SMs).
"""
import numpy as np
import pytest

import oracle
import synthetic

pytestmark = pytest.mark.gpu

TAU_GEMV = 1e-5
TAU_PREFILL = 8e-3


def xdev(x_bits):
    import torch
    return torch.from_numpy(np.ascontiguousarray(x_bits).view(np.int16)).cuda()


def assert_within(y, y_ref, s, tau, what=""):
    err = np.abs(y.astype(np.float64) - y_ref)
    bad = err > tau * s
    if bad.any():
        i = np.unravel_index(np.argmax(err / np.maximum(tau * s, 1e-300)), err.shape)
        raise AssertionError(f"{what}: {int(bad.sum())}/{bad.size} outputs over {tau}*s; worst at {i}: "
                             f"err {err[i]:.3e} s {s[i]:.3e} y {y[i]!r} ref {y_ref[i]!r}")


def make_group_layers(mode, Ns, K, seed):
    return [synthetic.make_layer(mode, N, K, seed + 17 * i, sidecar_count=max(1, N * K // 700))
            for i, N in enumerate(Ns)]


GROUPS = [
    # (mode, output features of each layer, K)
    (0, (2048, 256, 256), 2048),         # q, k, v with 2 KV heads: 20 tiles
    (0, (2048, 256, 256, 2048), 2048),   # four layers: 36 tiles
    (0, (8512,), 2048),                  # one layer through the grouped kernel
    (0, (8192, 2048), 1024),             # 80 tiles: more than fit as clusters
    (0, (300, 200, 136), 200),           # ragged tiles, K not a multiple of 64: 7 tiles
    (1, (1100, 520, 256), 1024),         # 2D codebooks: 16 tiles
    (1, (200, 136), 136),                # 2D, small and ragged
]


@pytest.mark.parametrize("mode,Ns,K", GROUPS)
@pytest.mark.parametrize("M", [1, 2, 3, 4])
def test_group_matches_oracle(hxq, mode, Ns, K, M):
    import torch
    layers = make_group_layers(mode, Ns, K, 70)
    lins = [hxq.HelixLinear.from_layer(l) for l in layers]
    grp = hxq.HelixGroup(lins)
    x = synthetic.activations(M, K, 71 + M)
    xd = xdev(x)
    ys = grp.forward(xd)
    torch.cuda.synchronize()
    for lin in lins:
        lin.check()
    first = [y.cpu().numpy() for y in ys]
    for i, layer in enumerate(layers):
        _, y_ref, s = oracle.forward_layer(layer, x)
        assert first[i].shape == (M, Ns[i])
        assert_within(first[i], y_ref, s, TAU_GEMV, f"layer {i} of {Ns} K={K} mode {mode} M={M}")
    # bitwise repeatable: a second call into the same buffers
    grp.forward(xd, ys=ys)
    torch.cuda.synchronize()
    for i in range(len(layers)):
        assert np.array_equal(ys[i].cpu().numpy(), first[i]), f"layer {i}: second call differs"
    grp.close()
    for lin in lins:
        lin.close()


@pytest.mark.parametrize("M", [16, 64])
def test_group_above_four_tokens_runs_each_layer(hxq, M):
    """Above 4 tokens every layer runs its own tensor-core kernel in turn."""
    import torch
    mode, Ns, K = 0, (640, 256, 130), 512
    layers = make_group_layers(mode, Ns, K, 80)
    lins = [hxq.HelixLinear.from_layer(l) for l in layers]
    grp = hxq.HelixGroup(lins)
    x = synthetic.activations(M, K, 81)
    ys = grp.forward(xdev(x))
    torch.cuda.synchronize()
    for i, layer in enumerate(layers):
        lins[i].check()
        _, y_ref, s = oracle.forward_layer(layer, x)
        assert_within(ys[i].cpu().numpy(), y_ref, s, TAU_GEMV if M <= 32 else TAU_PREFILL, f"layer {i} M={M}")
    grp.close()


@pytest.mark.parametrize("M", [1, 4, 16])
def test_group_bias_and_bf16(hxq, M):
    """Bias and bf16 output per layer, as hxq_linear_forward_out: the bf16
    values are the round-to-nearest-even of the same call's fp32 values."""
    import torch
    mode, Ns, K = 0, (2048, 256, 300), 1024
    layers = make_group_layers(mode, Ns, K, 90)
    lins = [hxq.HelixLinear.from_layer(l) for l in layers]
    grp = hxq.HelixGroup(lins)
    x = synthetic.activations(M, K, 91)
    xd = xdev(x)
    rng = np.random.default_rng(92)
    biases = [rng.normal(0.0, 0.5, N).astype(np.float32) for N in Ns]
    # the middle layer without bias
    bias_d = [torch.from_numpy(b).cuda() for b in biases]
    bias_d[1] = None
    y32 = grp.forward(xd, biases=bias_d, out_dtype=hxq.HXQ_OUT_F32)
    y16 = grp.forward(xd, biases=bias_d, out_dtype=hxq.HXQ_OUT_BF16)
    torch.cuda.synchronize()
    for i, layer in enumerate(layers):
        lins[i].check()
        W = oracle.decode(mode, layer["codebook"], layer["indices"], layer["sidecar_pos"], layer["sidecar_val"],
                          Ns[i], K)
        b = biases[i] if i != 1 else np.zeros(Ns[i], np.float32)
        a = y32[i].cpu().numpy()
        assert_within(a, oracle.forward(x, W) + b.astype(np.float64)[None, :],
                      oracle.abs_scale(x, W) + np.abs(b)[None, :], TAU_GEMV, f"layer {i} fp32+bias M={M}")
        want = (oracle.round_to_bf16(a).view(np.uint32) >> 16).astype(np.uint16)
        got = y16[i].view(torch.int16).cpu().numpy().view(np.uint16)
        assert np.array_equal(got, want), f"layer {i}: bf16 output is not the RNE of the fp32 output"
    grp.close()


def test_group_create_rejects(hxq):
    import ctypes
    a = synthetic.scalar_layer(256, 64, 1, sidecar_count=4)
    b = synthetic.scalar_layer(128, 64, 2, sidecar_count=4)
    c = synthetic.scalar_layer(128, 128, 3, sidecar_count=4)        # other K
    d = synthetic.vq2d_layer(128, 64, 4, sidecar_count=4)           # other mode
    la, lb, lc, ld = (hxq.HelixLinear.from_layer(l) for l in (a, b, c, d))

    def create(handles, n=None):
        g = ctypes.c_void_p()
        arr = (ctypes.c_void_p * max(1, len(handles)))(*handles)
        rc = hxq.lib.hxq_group_create(arr, len(handles) if n is None else n, ctypes.byref(g))
        if rc == hxq.HXQ_OK:
            hxq.lib.hxq_group_destroy(g)
        return rc

    assert create([la.handle, lb.handle]) == hxq.HXQ_OK
    assert create([la.handle, lc.handle]) == hxq.HXQ_EINVAL      # mixed K
    assert create([la.handle, ld.handle]) == hxq.HXQ_EINVAL      # mixed modes
    assert create([la.handle, la.handle]) == hxq.HXQ_EINVAL      # repeated handle
    assert create([la.handle, None]) == hxq.HXQ_EINVAL           # NULL handle
    assert create([la.handle], n=0) == hxq.HXQ_EINVAL
    assert create([la.handle, lb.handle, la.handle, lb.handle, la.handle]) == hxq.HXQ_EINVAL  # 5 > max


def test_group_forward_rejects(hxq):
    import torch
    a = synthetic.scalar_layer(256, 64, 1, sidecar_count=4)
    b = synthetic.scalar_layer(128, 64, 2, sidecar_count=4)
    lins = [hxq.HelixLinear.from_layer(l) for l in (a, b)]
    grp = hxq.HelixGroup(lins)
    x = xdev(synthetic.activations(1, 64, 5))
    ys = [torch.empty((1, 256), dtype=torch.float32, device="cuda"),
          torch.empty((1, 128), dtype=torch.float32, device="cuda")]
    f = hxq.lib.hxq_group_forward
    arr = hxq._ptr_array
    assert f(grp.handle, x.data_ptr(), None, arr(ys), 2, 1, None) == hxq.HXQ_EINVAL           # out dtype
    assert f(grp.handle, x.data_ptr(), None, None, 0, 1, None) == hxq.HXQ_EINVAL              # no outputs
    assert f(grp.handle, x.data_ptr(), None, arr([ys[0], None]), 0, 1, None) == hxq.HXQ_EINVAL
    assert f(grp.handle, x.data_ptr() + 2, None, arr(ys), 0, 1, None) == hxq.HXQ_EINVAL       # misaligned x
    assert f(grp.handle, x.data_ptr(), None, arr(ys), 0, 0, None) == hxq.HXQ_EINVAL           # M = 0
    assert f(None, x.data_ptr(), None, arr(ys), 0, 1, None) == hxq.HXQ_EINVAL
    assert f(grp.handle, x.data_ptr(), None, arr(ys), 0, 1, None) == hxq.HXQ_OK
    torch.cuda.synchronize()
    grp.close()
