"""CUDA path vs the CPU oracle, element by element, through the C ABI.

Bars: hxq_decode bit-exact; M <= 32 (fp32 codebook weights)
|y - y_ref| <= 1e-5 * s; M > 32 (bf16 tensor-core prefill) <= 8e-3 * s,
where s = sum_k |x||w| per output, y_ref in float64.
"""
import numpy as np
import pytest

import oracle
import synthetic

pytestmark = pytest.mark.gpu

TAU_GEMV = 1e-5
TAU_PREFILL = 8e-3
GEMV, TC, AUTO = 1, 2, 0


def xdev(x_bits):
    import torch
    return torch.from_numpy(np.ascontiguousarray(x_bits).view(np.int16)).cuda()


def run(hxq, lin, x_bits, kernel=AUTO, split=0):
    import torch
    y = lin.forward(xdev(x_bits), kernel=kernel, split_k=split)
    torch.cuda.synchronize()
    lin.check()
    return y.cpu().numpy()


def assert_within(y, y_ref, s, tau, what=""):
    err = np.abs(y.astype(np.float64) - y_ref)
    bad = err > tau * s
    if bad.any():
        i = np.unravel_index(np.argmax(err / np.maximum(tau * s, 1e-300)), err.shape)
        raise AssertionError(f"{what}: {int(bad.sum())}/{bad.size} outputs over {tau}*s; worst at {i}: "
                             f"err {err[i]:.3e} s {s[i]:.3e} y {y[i]!r} ref {y_ref[i]!r}")


def tau_for(M, kernel):
    return TAU_GEMV if M <= 32 else TAU_PREFILL


# ----------------------------------------------------------------- decode

@pytest.mark.parametrize("mode,N,K,ns", [
    (0, 256, 256, 64), (0, 300, 200, 77), (0, 129, 8, 5), (0, 8512, 2048, 17433),
    (1, 200, 136, 50), (1, 128, 64, 0), (1, 257, 4096, 526), (1, 11008, 4096, 22544),
])
def test_decode_bit_exact(hxq, mode, N, K, ns):
    layer = synthetic.make_layer(mode, N, K, 1, sidecar_count=ns)
    lin = hxq.HelixLinear.from_layer(layer)
    W = lin.decode().cpu().numpy()
    W_ref = oracle.decode(mode, layer["codebook"], layer["indices"], layer["sidecar_pos"],
                          layer["sidecar_val"], N, K)
    assert np.array_equal(W.view(np.uint32), W_ref.view(np.uint32))


def test_decode_sidecar_edges(hxq):
    N, K = 130, 72
    layer = synthetic.scalar_layer(N, K, 3, sidecar_count=0)
    pos = np.array([0, N * K - 1, K - 1, K, 5, 6, 7, 8, 9, 10, 11, 12, 13, 14, 15, 16, 20 * K + 63,
                    20 * K + 64, 129 * K], np.int64)
    layer["sidecar_pos"] = pos
    layer["sidecar_val"] = np.linspace(-1, 1, pos.size).astype(np.float32)
    lin = hxq.HelixLinear.from_layer(layer)
    W = lin.decode().cpu().numpy()
    W_ref = oracle.decode(0, layer["codebook"], layer["indices"], pos, layer["sidecar_val"], N, K)
    assert np.array_equal(W, W_ref)


# ----------------------------------------------------------------- forward, small shapes

SHAPES = [(0, 256, 256), (0, 300, 200), (0, 130, 72), (1, 200, 136), (1, 384, 256), (0, 1000, 1088)]


@pytest.mark.parametrize("mode,N,K", SHAPES)
@pytest.mark.parametrize("M", [1, 2, 3, 4, 5, 8, 16, 31, 32, 33, 64, 100, 255, 256, 257])
def test_forward_matches_oracle(hxq, mode, N, K, M):
    layer = synthetic.make_layer(mode, N, K, 7, sidecar_count=max(1, N * K // 500))
    x = synthetic.activations(M, K, 7)
    _, y_ref, s = oracle.forward_layer(layer, x)
    lin = hxq.HelixLinear.from_layer(layer)
    kernels = [AUTO, TC] + ([GEMV] if M <= 8 else [])
    for kernel in kernels:
        for split in (0, 1, 3):
            y = run(hxq, lin, x, kernel, split)
            assert_within(y, y_ref, s, tau_for(M, kernel), f"mode {mode} {N}x{K} M={M} k={kernel} S={split}")


# Any nn.Linear width: scalar K with no alignment, 2D K a multiple of 4 but
# not of 8. Rows of x are then not 16-byte aligned (element-wise staging in
# the GEMV, a re-strided copy ahead of the tensor-core kernel).
RAGGED = [(0, 37, 1), (0, 130, 7), (0, 129, 13), (0, 300, 1001), (1, 131, 4), (1, 200, 12), (1, 257, 1004)]


@pytest.mark.parametrize("mode,N,K", RAGGED)
def test_ragged_k_decode_bit_exact(hxq, mode, N, K):
    layer = synthetic.make_layer(mode, N, K, 13, sidecar_count=max(1, N * K // 300))
    W = hxq.HelixLinear.from_layer(layer).decode().cpu().numpy()
    W_ref = oracle.decode(mode, layer["codebook"], layer["indices"], layer["sidecar_pos"],
                          layer["sidecar_val"], N, K)
    assert np.array_equal(W.view(np.uint32), W_ref.view(np.uint32))


@pytest.mark.parametrize("mode,N,K", RAGGED)
def test_ragged_k_forward_matches_oracle(hxq, mode, N, K):
    layer = synthetic.make_layer(mode, N, K, 13, sidecar_count=max(1, N * K // 300))
    lin = hxq.HelixLinear.from_layer(layer)
    # M rising then falling: the tensor-core path's re-strided copy grows,
    # then is reused by smaller forwards
    for M in (1, 3, 4, 5, 8, 16, 32, 33, 300, 6):
        x = synthetic.activations(M, K, 13 + M)
        _, y_ref, s = oracle.forward_layer(layer, x)
        kernels = [AUTO, TC] + ([GEMV] if M <= 8 else [])
        for kernel in kernels:
            for split in (0, 3):
                y = run(hxq, lin, x, kernel, split)
                assert_within(y, y_ref, s, tau_for(M, kernel), f"mode {mode} {N}x{K} M={M} k={kernel} S={split}")


@pytest.mark.parametrize("pinned", [True, False])
@pytest.mark.parametrize("mode,N,K,M", [(0, 300, 200, 1), (0, 129, 13, 3), (1, 200, 136, 8), (0, 256, 512, 40),
                                        (0, 8512, 2048, 1)])
def test_forward_host_buffers(hxq, mode, N, K, M, pinned):
    """hxq_linear_forward_host: x in, y out on one stream, with no
    synchronisation between calls until the end; every call's y against
    the oracle, and a bad call (misaligned x_dev) rejected before any copy.
    Pinned buffers are read and written by the kernels, pageable ones go
    through copies."""
    import torch
    layer = synthetic.make_layer(mode, N, K, 21, sidecar_count=max(1, N * K // 400))
    lin = hxq.HelixLinear.from_layer(layer)
    st = torch.cuda.Stream()
    xs = [synthetic.activations(M, K, 21 + i) for i in range(3)]
    pin = (lambda t: t.pin_memory()) if pinned else (lambda t: t)
    xh = [pin(torch.from_numpy(x.view(np.int16))) for x in xs]
    yh = [pin(torch.full((M, N), float("nan"), dtype=torch.float32)) for _ in xs]
    xd = torch.empty((M, K), dtype=torch.int16, device="cuda")
    yd = torch.empty((M, N), dtype=torch.float32, device="cuda")
    for i in range(3):
        lin.forward_host(xh[i], yh[i], xd, yd, stream=st, sync=False)
    st.synchronize()
    lin.check()
    for i in range(3):
        _, y_ref, s = oracle.forward_layer(layer, xs[i])
        assert_within(yh[i].numpy(), y_ref, s, tau_for(M, AUTO), f"host buffers call {i}")
    if pinned:
        # x_host not 16-byte aligned: the fetch kernel copies element by element
        xh_off = torch.empty(M * K + 1, dtype=torch.int16).pin_memory()
        xh_off[1:].copy_(xh[0].view(-1))
        yh2 = torch.full((M, N), float("nan"), dtype=torch.float32).pin_memory()
        lin.forward_host(xh_off[1:].view(M, K), yh2, xd, yd, stream=st)
        _, y_ref, s = oracle.forward_layer(layer, xs[0])
        assert_within(yh2.numpy(), y_ref, s, tau_for(M, AUTO), "unaligned host x")
    xbad = torch.empty(M * K + 8, dtype=torch.int16, device="cuda")[1:]
    assert hxq.lib.hxq_linear_forward_host(lin.handle, hxq._ptr(xh[0]), hxq._ptr(xbad), hxq._ptr(yd),
                                           hxq._ptr(yh[0]), M, hxq._stream(st)) == hxq.HXQ_EINVAL


@pytest.mark.parametrize("M", [33, 256, 300])
@pytest.mark.parametrize("mode", [0, 1])
def test_prefill_equals_bf16_weight_oracle(hxq, mode, M):
    """Diagnostic for the bf16 tensor-core path: against the oracle run on
    bf16-rounded weights only fp32 accumulation error remains."""
    N, K = 384, 512
    layer = synthetic.make_layer(mode, N, K, 11, sidecar_count=200)
    x = synthetic.activations(M, K, 11)
    W = oracle.decode(mode, layer["codebook"], layer["indices"], layer["sidecar_pos"],
                      layer["sidecar_val"], N, K)
    Wb = oracle.round_to_bf16(W)
    y_ref = oracle.forward(x, Wb)
    s = oracle.abs_scale(x, Wb)
    y = run(hxq, hxq.HelixLinear.from_layer(layer), x, TC, 1)
    assert_within(y, y_ref, s, 1e-5, "bf16-weight diagnostic")


@pytest.mark.parametrize("mode", [0, 1])
@pytest.mark.parametrize("kernel,M", [(GEMV, 1), (GEMV, 4), (TC, 8), (TC, 32), (TC, 256)])
def test_dyadic_exact(hxq, mode, kernel, M):
    """Dyadic codebook / sidecar and integer x: every product and partial sum
    is exact in fp32, so the GPU must reproduce the oracle exactly."""
    N, K = 256, 512
    rng = np.random.default_rng(2)
    layer = synthetic.make_layer(mode, N, K, 2, sidecar_count=300)
    cb_size = layer["codebook"].size
    layer["codebook"] = (rng.integers(-128, 128, cb_size) / 256.0).astype(np.float32)
    layer["sidecar_val"] = (rng.integers(-128, 129, layer["sidecar_val"].size) / 256.0).astype(np.float32)
    xi = rng.integers(-4, 5, size=(M, K)).astype(np.float32)
    x = synthetic.f32_to_bf16_bits(xi)
    _, y_ref, _ = oracle.forward_layer(layer, x)
    y = run(hxq, hxq.HelixLinear.from_layer(layer), x, kernel, 3)
    assert np.array_equal(y.astype(np.float64), y_ref)


@pytest.mark.parametrize("mode", [0, 1])
def test_one_hot_selects_column(hxq, mode):
    N, K = 300, 256
    layer = synthetic.make_layer(mode, N, K, 5, sidecar_count=400)
    W = oracle.decode(mode, layer["codebook"], layer["indices"], layer["sidecar_pos"],
                      layer["sidecar_val"], N, K)
    lin = hxq.HelixLinear.from_layer(layer)
    for kstar in (0, 63, 64, 255):
        x = np.zeros((1, K), np.float32)
        x[0, kstar] = 1.0
        xb = synthetic.f32_to_bf16_bits(x)
        yg = run(hxq, lin, xb, GEMV, 1)[0]
        # the GEMV applies a sidecar entry as c + (v - c) in fp32: exact
        # except for at most one rounding of each of the two operations
        patched = np.zeros(N, bool)
        pos = layer["sidecar_pos"]
        patched[pos[pos % K == kstar] // K] = True
        assert np.array_equal(yg[~patched], W[~patched, kstar])
        cmax = np.abs(layer["codebook"]).max()
        assert np.all(np.abs(yg[patched] - W[patched, kstar]) <= 2.0 ** -23 * (np.abs(W[patched, kstar]) + cmax))
        x2 = np.zeros((40, K), np.float32)
        x2[:, kstar] = 1.0
        y = run(hxq, lin, synthetic.f32_to_bf16_bits(x2), TC, 1)
        assert np.array_equal(y[0], oracle.round_to_bf16(W[:, kstar]))     # bf16 weights, M > 32
        y8 = run(hxq, lin, synthetic.f32_to_bf16_bits(x2[:8]), TC, 1)       # hi+mid split, M <= 32
        assert np.all(np.abs(y8[0] - W[:, kstar]) <= 2.0 ** -17 * np.abs(W[:, kstar]))


def test_constant_codebook(hxq):
    N, K, M = 260, 320, 6
    layer = synthetic.scalar_layer(N, K, 6, sidecar_count=30)
    layer["codebook"][:] = np.float32(0.03125)
    x = synthetic.activations(M, K, 6)
    _, y_ref, s = oracle.forward_layer(layer, x)
    lin = hxq.HelixLinear.from_layer(layer)
    for kernel in (GEMV, TC):
        assert_within(run(hxq, lin, x, kernel, 2), y_ref, s, TAU_GEMV, f"constant cb k={kernel}")


@pytest.mark.parametrize("kernel,M", [(GEMV, 1), (GEMV, 3), (TC, 16), (TC, 512)])
def test_bitwise_repeatable(hxq, kernel, M):
    layer = synthetic.scalar_layer(2048, 2048, 4)
    x = synthetic.activations(M, 2048, 4)
    lin = hxq.HelixLinear.from_layer(layer)
    a = run(hxq, lin, x, kernel, 0)
    b = run(hxq, lin, x, kernel, 0)
    assert np.array_equal(a.view(np.uint32), b.view(np.uint32))


def test_no_sidecar_and_dense_sidecar(hxq):
    for ns in (0, 2000):
        layer = synthetic.scalar_layer(256, 128, 9, sidecar_count=ns)
        x = synthetic.activations(4, 128, 9)
        _, y_ref, s = oracle.forward_layer(layer, x)
        lin = hxq.HelixLinear.from_layer(layer)
        for kernel in (GEMV, TC):
            assert_within(run(hxq, lin, x, kernel, 1), y_ref, s, TAU_GEMV, f"ns={ns} k={kernel}")


# ----------------------------------------------------------------- error paths with a device

def test_create_rejects_bad_sidecar(hxq):
    N, K = 64, 64
    cb = np.zeros(256, np.float32)
    idx = np.zeros(N * K, np.uint8)
    for pos in ([N * K], [-1], [3, 3]):
        p = np.array(pos, np.int64)
        v = np.ones(p.size, np.float32)
        with pytest.raises(hxq.HXQError) as e:
            hxq.HelixLinear(cb, idx, 0, p, v, N, K)
        assert e.value.code == hxq.HXQ_EINVAL


def test_forward_rejects_bad_arguments(hxq):
    import torch
    layer = synthetic.scalar_layer(128, 64, 0)
    lin = hxq.HelixLinear.from_layer(layer)
    x = torch.zeros((40, 64), dtype=torch.int16, device="cuda")
    y = torch.zeros((40, 128), dtype=torch.float32, device="cuda")
    for kernel, split, M in ((3, 0, 1), (GEMV, 0, 9), (AUTO, 65, 1), (AUTO, -1, 1), (AUTO, 0, 0)):
        rc = hxq.lib.hxq_linear_forward_ex(lin.handle, x.data_ptr(), y.data_ptr(), M, kernel, split, None)
        assert rc == hxq.HXQ_EINVAL
    rc = hxq.lib.hxq_linear_forward(lin.handle, x.data_ptr() + 2, y.data_ptr(), 1, None)
    assert rc == hxq.HXQ_EINVAL   # x not 16-byte aligned
    assert hxq.hxq_linear_info(lin.handle) == (0, 128, 64, layer["sidecar_pos"].size)


# ----------------------------------------------------------------- full-size workloads

FULL = [(cfg, name, M) for cfg in ("tiny", "mamba2", "qwen25_3b", "vq2d")
        for name, _, _, _, Ms, _ in synthetic.CONFIGS[cfg] for M in Ms]


@pytest.mark.parametrize("cfg,name,M", FULL)
def test_full_size_decode_configs(hxq, cfg, name, M):
    """Full sizes, auto kernel choice and split (the configuration the
    benchmark times), every output compared with the full oracle."""
    layer = dict((n, l) for n, l, _ in synthetic.config_layers(cfg))[name]
    x = synthetic.activations(M, layer["K"], 0)
    _, y_ref, s = oracle.forward_layer(layer, x)
    y = run(hxq, hxq.HelixLinear.from_layer(layer), x)
    assert_within(y, y_ref, s, TAU_GEMV, f"{cfg}/{name} M={M}")


@pytest.mark.parametrize("name", ["mlp_up", "mlp_down"])
@pytest.mark.parametrize("M", [512, 2048])
def test_full_size_prefill_sampled_rows(hxq, name, M):
    """Full prefill sizes; the oracle recomputes 384 sampled output features
    (all M tokens each) from their own decode."""
    layer = dict((n, l) for n, l, _ in synthetic.config_layers("prefill"))[name]
    x = synthetic.activations(M, layer["K"], 0)
    y = run(hxq, hxq.HelixLinear.from_layer(layer), x)
    rng = np.random.default_rng(M)
    rows = np.unique(np.concatenate([rng.choice(layer["N"], 380, replace=False),
                                     [0, 127, 128, layer["N"] - 1]]))
    y_ref, s = oracle.forward_rows(layer, x, rows)
    assert_within(y[:, rows], y_ref, s, TAU_PREFILL, f"prefill {name} M={M}")


def _abs_layer(layer):
    """The layer with |codebook| and |sidecar values|: its decode is |W|
    elementwise (decode only selects values), so its forward on |x| is
    s = sum_k |x||w|."""
    a = dict(layer)
    a["codebook"] = np.abs(layer["codebook"])
    a["sidecar_val"] = np.abs(layer["sidecar_val"])
    return a


CPP_FULL = ([(cfg, name, M) for cfg in ("mamba2", "qwen25_3b", "vq2d")
             for name, _, _, _, Ms, _ in synthetic.CONFIGS[cfg] for M in Ms]
            + [("prefill", name, M) for name in ("mlp_up", "mlp_down") for M in (512, 2048)])


@pytest.mark.parametrize("cfg,name,M", CPP_FULL)
def test_full_size_against_plain_cpp_oracle(hxq, cfg, name, M):
    """The benchmark's layers at full size, checked by the plain C++ loop
    oracle (decode with the sidecar, float64 dot products, no library
    routine): every output feature for M <= 32, four 128-row blocks
    (first, last, two inside) for the prefill sizes."""
    import os
    from oracle import hxq_oracle_cpp as cpp
    layer = dict((n, l) for n, l, _ in synthetic.config_layers(cfg))[name]
    N = layer["N"]
    x = synthetic.activations(M, layer["K"], 0)
    y = run(hxq, hxq.HelixLinear.from_layer(layer), x)
    blocks = [(0, N)] if M <= 32 else [(0, 128), (N // 3, N // 3 + 128), (N // 2 + 64, N // 2 + 192),
                                       (N - 128, N)]
    threads = os.cpu_count() or 1
    for r0, r1 in blocks:
        y_ref = cpp.forward_rows(layer, x, r0, r1, threads)
        s = cpp.forward_rows(_abs_layer(layer), x & 0x7FFF, r0, r1, threads)
        assert_within(y[:, r0:r1], y_ref, s, tau_for(M, AUTO), f"{cfg}/{name} M={M} rows {r0}:{r1}")


def _cluster_shapes(num_sms):
    """Layer heights whose tile counts select each cluster size (2, 4, 8, and
    the non-portable 12 and 16 where the device allows them): tiles x size
    between 85 % and 100 % of the SMs, last tile partial."""
    out = []
    for cs in (2, 4, 8, 12, 16):
        tiles = num_sms // cs
        if 100 * tiles * cs >= 85 * num_sms:
            out.append((cs, tiles * 128 - 37))
    return out


@pytest.mark.parametrize("mode", [0, 1])
def test_gemv_cluster_split_shapes(hxq, mode):
    """Decode GEMV shapes that run as cluster splits of each tile's K (the
    ranks' sums meet in distributed shared memory), with sidecar entries and
    a partial last tile, against the oracle."""
    import torch
    num_sms = torch.cuda.get_device_properties(0).multi_processor_count
    K = 1024
    for cs, N in _cluster_shapes(num_sms):
        layer = synthetic.make_layer(mode, N, K, 40 + cs, sidecar_count=N * K // 500)
        lin = hxq.HelixLinear.from_layer(layer)
        W = oracle.decode(mode, layer["codebook"], layer["indices"], layer["sidecar_pos"], layer["sidecar_val"], N, K)
        for M in (1, 2, 4):
            x = synthetic.activations(M, K, 50 + M)
            y = run(hxq, lin, x, AUTO)
            assert_within(y, oracle.forward(x, W), oracle.abs_scale(x, W), TAU_GEMV, f"cluster {cs} N={N} M={M}")
        lin.close()


@pytest.mark.parametrize("mode,N,K", [(0, 300, 200), (1, 200, 136), (0, 8512, 2048)])
@pytest.mark.parametrize("M", [1, 4, 16, 64])
def test_forward_out_bias_and_bf16(hxq, mode, N, K, M):
    """hxq_linear_forward_out: y = x.W^T + bias as fp32 (within the kernel's
    tolerance of the exact value) and as bf16, which must be the
    round-to-nearest-even of the same kernel's fp32 result, bit for bit."""
    import torch
    layer = synthetic.make_layer(mode, N, K, 60, sidecar_count=max(1, N * K // 1000))
    lin = hxq.HelixLinear.from_layer(layer)
    W = oracle.decode(mode, layer["codebook"], layer["indices"], layer["sidecar_pos"], layer["sidecar_val"], N, K)
    x = synthetic.activations(M, K, 61)
    bias = np.random.default_rng(62).normal(0.0, 0.5, N).astype(np.float32)
    bias_d = torch.from_numpy(bias).cuda()
    xd = xdev(x)
    y32 = lin.forward_out(xd, bias_d, hxq.HXQ_OUT_F32)
    y16 = lin.forward_out(xd, bias_d, hxq.HXQ_OUT_BF16)
    ynb = lin.forward_out(xd, None, hxq.HXQ_OUT_F32)
    torch.cuda.synchronize()
    lin.check()
    y32 = y32.cpu().numpy()
    ynb = ynb.cpu().numpy()
    y16_bits = y16.view(torch.int16).cpu().numpy().view(np.uint16)
    ref = oracle.forward(x, W) + bias.astype(np.float64)[None, :]
    s = oracle.abs_scale(x, W)
    tau = tau_for(M, AUTO)
    assert_within(y32, ref, s + np.abs(bias)[None, :], tau, f"fp32+bias M={M}")
    # no bias: the plain forward
    assert_within(ynb, oracle.forward(x, W), s, tau, f"no bias M={M}")
    # bf16: exactly the rounding of this kernel's fp32 value
    want = (oracle.round_to_bf16(y32).view(np.uint32) >> 16).astype(np.uint16)
    assert np.array_equal(y16_bits, want), "bf16 output is not the RNE of the fp32 output"
    lin.close()


def test_forward_out_rejects_bad_dtype(hxq):
    import torch
    layer = synthetic.scalar_layer(256, 64, 3, sidecar_count=0)
    lin = hxq.HelixLinear.from_layer(layer)
    x = xdev(synthetic.activations(1, 64, 3))
    y = torch.empty((1, 256), dtype=torch.float32, device="cuda")
    assert hxq.lib.hxq_linear_forward_out(lin.handle, x.data_ptr(), None, y.data_ptr(), 2, 1, None) == hxq.HXQ_EINVAL
    assert hxq.lib.hxq_linear_forward_out(lin.handle, x.data_ptr(), None, None, 0, 1, None) == hxq.HXQ_EINVAL
