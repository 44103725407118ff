"""Failure detection on the GPU without a fault: the tensor-core kernel's
pipeline waits are bounded; a test hook withholds one item's activations so
that the MMA thread's wait runs out (1 ms). The CTAs then drain what they
issued, free their tensor memory and return; hxq_linear_check reports
HXQ_ETIMEOUT once, and the next ordinary forward on the same handle is
exact -- the status word and the split-tile counters were reset and no
tensor memory was left allocated."""
import numpy as np
import pytest

import oracle
import synthetic

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("mode,M", [(0, 64), (0, 16), (1, 300)])
def test_withheld_activations_time_out_then_recover(hxq, mode, M):
    import torch
    N, K = 1024, 2048
    layer = synthetic.make_layer(mode, N, K, 80 + M, sidecar_count=2000)
    lin = hxq.HelixLinear.from_layer(layer)
    x = synthetic.activations(M, K, 81)
    xd = torch.from_numpy(x.view(np.int16)).cuda()
    y = torch.empty((M, N), dtype=torch.float32, device="cuda")
    rc = hxq.lib.hxq_test_forward_withheld(lin.handle, xd.data_ptr(), y.data_ptr(), M, 1, 1000, None)
    assert rc == hxq.HXQ_OK, hxq.hxq_strerror(rc)
    torch.cuda.synchronize()
    assert hxq.lib.hxq_linear_check(lin.handle) == hxq.HXQ_ETIMEOUT
    assert hxq.lib.hxq_linear_check(lin.handle) == hxq.HXQ_OK  # reported once, then cleared
    W = oracle.decode(mode, layer["codebook"], layer["indices"], layer["sidecar_pos"], layer["sidecar_val"], N, K)
    tau = 1e-5 if M <= 32 else 8e-3
    for _ in range(2):
        got = lin.forward(xd).cpu().numpy().astype(np.float64)
        torch.cuda.synchronize()
        lin.check()
        err = np.abs(got - oracle.forward(x, W))
        assert np.all(err <= tau * oracle.abs_scale(x, W))
    lin.close()


def test_withheld_hook_rejects_bad_arguments(hxq):
    import torch
    layer = synthetic.make_layer(0, 256, 256, 82, sidecar_count=10)
    lin = hxq.HelixLinear.from_layer(layer)
    x = torch.zeros((64, 256), dtype=torch.int16, device="cuda")
    y = torch.empty((64, 256), dtype=torch.float32, device="cuda")
    f = hxq.lib.hxq_test_forward_withheld
    assert f(lin.handle, x.data_ptr(), y.data_ptr(), 4, 1, 1000, None) == hxq.HXQ_EINVAL  # GEMV range
    assert f(lin.handle, x.data_ptr(), y.data_ptr(), 64, -1, 1000, None) == hxq.HXQ_EINVAL
    assert f(lin.handle, x.data_ptr(), y.data_ptr(), 64, 1, 0, None) == hxq.HXQ_EINVAL
    assert f(lin.handle, x.data_ptr(), y.data_ptr(), 64, 1, 3000000, None) == hxq.HXQ_EINVAL
    lin.close()
