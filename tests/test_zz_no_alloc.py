"""hxq_linear_forward_noalloc: the GEMV for callers that cannot allocate.

Such callers (allocation-free loops after start-up, or code running handles
it did not create) get the same result as hxq_linear_forward from an entry
point whose scratch is a fixed array inside the library. These tests call it
through the C ABI and compare it with the existing entry point, twice in a
row (the array keeps the previous call's contents), and check its size
limits. The file sorts last so that a run stopping at the first failure has
already run everything else; it also passes on its own in a fresh process.
"""
import numpy as np
import pytest

import oracle
import synthetic

pytestmark = pytest.mark.gpu

TAU = 1e-5  # the fp32-codebook GEMV tolerance, times sum |x||w|


def _xdev(x_bits):
    import torch
    return torch.from_numpy(np.ascontiguousarray(x_bits).view(np.int16)).cuda()


# The last four shapes have more tiles than half the SMs, so no cluster size
# fits (2 x tiles > SMs) and they run the stream-K decomposition whose
# counters and partial sums live in the fixed array; the others take the
# cluster split (small layers at any fill). Two shapes have rows of x that
# are not 16-byte aligned.
@pytest.mark.parametrize("mode,N,K,M", [(0, 8512, 2048, 1), (0, 2048, 4096, 4), (1, 1100, 4096, 2),
                                        (0, 300, 200, 3), (0, 640, 8192, 4), (1, 260, 1004, 1),
                                        (0, 11008, 512, 1), (0, 9600, 1024, 4), (1, 10240, 512, 2),
                                        (0, 9600, 1001, 3)])
def test_noalloc_matches_forward_twice(hxq, mode, N, K, M):
    import torch
    num_sms = torch.cuda.get_device_properties(0).multi_processor_count
    if N >= 9600:  # stream-K for certain (see above)
        assert (N + 127) // 128 * 2 > num_sms
    layer = synthetic.make_layer(mode, N, K, 21, sidecar_count=max(1, N * K // 1000))
    x = synthetic.activations(M, K, 21)
    lin = hxq.HelixLinear.from_layer(layer)
    xd = _xdev(x)
    y_ref_dev = torch.empty((M, N), dtype=torch.float32, device="cuda")
    rc = hxq.lib.hxq_linear_forward(lin.handle, xd.data_ptr(), y_ref_dev.data_ptr(), M, None)
    assert rc == hxq.HXQ_OK
    torch.cuda.synchronize()
    y_existing = y_ref_dev.cpu().numpy()
    _, y_oracle, s = oracle.forward_layer(layer, x)
    for call in range(2):
        y = torch.full((M, N), float("nan"), dtype=torch.float32, device="cuda")
        rc = hxq.lib.hxq_linear_forward_noalloc(lin.handle, xd.data_ptr(), y.data_ptr(), M, None)
        assert rc == hxq.HXQ_OK, hxq.hxq_strerror(rc)
        torch.cuda.synchronize()
        lin.check()
        got = y.cpu().numpy()
        err = np.abs(got.astype(np.float64) - y_existing)
        assert np.all(err <= TAU * s), f"call {call}: max err/s {np.max(err / s):.3e}"
        assert np.all(np.abs(got.astype(np.float64) - y_oracle) <= TAU * s)


def test_noalloc_limits(hxq):
    import torch
    layer = synthetic.scalar_layer(256, 64, 3, sidecar_count=10)
    lin = hxq.HelixLinear.from_layer(layer)
    x = _xdev(synthetic.activations(5, 64, 3))
    y = torch.empty((5, 256), dtype=torch.float32, device="cuda")
    # more than 4 tokens, no tokens, NULL handle, misaligned x
    assert hxq.lib.hxq_linear_forward_noalloc(lin.handle, x.data_ptr(), y.data_ptr(), 5, None) == hxq.HXQ_EINVAL
    assert hxq.lib.hxq_linear_forward_noalloc(lin.handle, x.data_ptr(), y.data_ptr(), 0, None) == hxq.HXQ_EINVAL
    assert hxq.lib.hxq_linear_forward_noalloc(None, x.data_ptr(), y.data_ptr(), 1, None) == hxq.HXQ_EINVAL
    assert hxq.lib.hxq_linear_forward_noalloc(lin.handle, x.data_ptr() + 2, y.data_ptr(), 1,
                                              None) == hxq.HXQ_EINVAL
    # more output features than the fixed counter space (4096 tiles of 128)
    N_big, K_small = 4096 * 128 + 1, 8
    big = synthetic.scalar_layer(N_big, K_small, 4, sidecar_count=0)
    lin_big = hxq.HelixLinear.from_layer(big)
    xb = _xdev(synthetic.activations(1, K_small, 4))
    yb = torch.empty((1, N_big), dtype=torch.float32, device="cuda")
    assert hxq.lib.hxq_linear_forward_noalloc(lin_big.handle, xb.data_ptr(), yb.data_ptr(), 1,
                                              None) == hxq.HXQ_EINVAL
    # the regular entry point still serves that layer
    assert hxq.lib.hxq_linear_forward(lin_big.handle, xb.data_ptr(), yb.data_ptr(), 1, None) == hxq.HXQ_OK
    torch.cuda.synchronize()
    lin_big.check()
