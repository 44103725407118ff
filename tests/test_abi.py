"""The C ABI without a GPU: the library loads, exports every entry point that
include/hxq.h declares, and rejects bad arguments before touching CUDA."""
import ctypes
import os
import re

import numpy as np
import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def declared_functions():
    src = open(os.path.join(ROOT, "include", "hxq.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(hxq_[a-z0-9_]+)\s*\(", src)))


def test_header_declares_the_boundary():
    names = declared_functions()
    for required in ("hxq_linear_create", "hxq_linear_forward", "hxq_decode", "hxq_linear_destroy",
                     "hxq_strerror"):
        assert required in names


def test_library_exports_every_declared_symbol():
    import vq_compressed_linear_b200 as m
    for name in declared_functions():
        assert hasattr(m.lib, name), name          # ctypes resolves the symbol or raises
        assert name in m.EXPORTED
        assert callable(getattr(m, name))


def test_no_cpu_fallback_in_binding():
    """The binding only marshals: it must not import the oracle or numpy math."""
    src = open(os.path.join(ROOT, "vq_compressed_linear_b200", "__init__.py")).read()
    assert "oracle" not in src.replace("no Python or CPU fallback", "")
    assert "import numpy" not in src


def test_strerror():
    import vq_compressed_linear_b200 as m
    for code in (0, -1, -2, -3, -4, -5):
        assert m.hxq_strerror(code)
    assert m.hxq_strerror(-99) == "unknown status"


def _create(m, cb, idx, mode, pos, val, ns, N, K, out=True):
    h = ctypes.c_void_p()
    return m.lib.hxq_linear_create(m._ptr(cb), m._ptr(idx), mode, m._ptr(pos), m._ptr(val), ns, N, K,
                                   ctypes.byref(h) if out else None)


@pytest.mark.parametrize("case", ["null_out", "null_cb", "null_idx", "bad_mode", "N0", "K0", "Kneg",
                                  "vq2d_K_not_mult4", "neg_sidecar", "too_many_sidecar", "null_sidecar"])
def test_create_rejects_bad_arguments(case):
    import vq_compressed_linear_b200 as m
    N, K = 16, 32
    cb = np.zeros(256, np.float32)
    idx = np.zeros(N * K, np.uint8)
    pos = np.array([1], np.int64)
    val = np.array([1.0], np.float32)
    args = dict(cb=cb, idx=idx, mode=0, pos=pos, val=val, ns=1, N=N, K=K, out=True)
    if case == "null_out": args["out"] = False
    if case == "null_cb": args["cb"] = None
    if case == "null_idx": args["idx"] = None
    if case == "bad_mode": args["mode"] = 2
    if case == "N0": args["N"] = 0
    if case == "K0": args["K"] = 0
    if case == "Kneg": args["K"] = -8
    if case == "vq2d_K_not_mult4":
        args.update(mode=1, K=34, cb=np.zeros(8192, np.float32))
    if case == "neg_sidecar": args["ns"] = -1
    if case == "too_many_sidecar": args["ns"] = N * K + 1
    if case == "null_sidecar": args["pos"] = None
    assert _create(m, **args) == m.HXQ_EINVAL


def test_forward_and_decode_reject_null_handle():
    import vq_compressed_linear_b200 as m
    x = np.zeros(64, np.uint16)
    y = np.zeros(64, np.float32)
    assert m.lib.hxq_linear_forward(None, m._ptr(x), m._ptr(y), 1, None) == m.HXQ_EINVAL
    assert m.lib.hxq_linear_forward_ex(None, m._ptr(x), m._ptr(y), 1, 0, 0, None) == m.HXQ_EINVAL
    assert m.lib.hxq_linear_forward_out(None, m._ptr(x), None, m._ptr(y), m.HXQ_OUT_F32, 1, None) == m.HXQ_EINVAL
    assert m.lib.hxq_linear_forward_noalloc(None, m._ptr(x), m._ptr(y), 1, None) == m.HXQ_EINVAL
    assert m.lib.hxq_linear_forward_host(None, m._ptr(x), m._ptr(x), m._ptr(y), m._ptr(y), 1, None) == m.HXQ_EINVAL
    assert m.lib.hxq_decode(None, m._ptr(y), None) == m.HXQ_EINVAL
    assert m.lib.hxq_linear_check(None) == m.HXQ_EINVAL
    assert m.lib.hxq_linear_info(None, None, None, None, None) == m.HXQ_EINVAL
    m.lib.hxq_linear_destroy(None)  # ignored


def test_group_entry_points_reject_null_arguments():
    import ctypes
    import vq_compressed_linear_b200 as m
    g = ctypes.c_void_p()
    none2 = (ctypes.c_void_p * 2)(None, None)
    assert m.lib.hxq_group_create(None, 1, ctypes.byref(g)) == m.HXQ_EINVAL
    assert m.lib.hxq_group_create(none2, 2, None) == m.HXQ_EINVAL
    assert m.lib.hxq_group_create(none2, 2, ctypes.byref(g)) == m.HXQ_EINVAL   # NULL handles
    assert g.value is None                                                      # *out cleared
    for n in (0, -1, m.HXQ_MAX_GROUP + 1):
        assert m.lib.hxq_group_create(none2, n, ctypes.byref(g)) == m.HXQ_EINVAL
    x = np.zeros(64, np.uint16)
    assert m.lib.hxq_group_forward(None, m._ptr(x), None, none2, m.HXQ_OUT_F32, 1, None) == m.HXQ_EINVAL
    m.lib.hxq_group_destroy(None)  # ignored


def test_encoder_entry_points_reject_null_arguments():
    import vq_compressed_linear_b200 as m
    p = np.zeros(64, np.float32)
    lab = np.zeros(64, np.uint16)
    assert m.lib.hxq_assign(None, 64, 1, m._ptr(p), 8, m._ptr(lab), None) == m.HXQ_EINVAL
    assert m.lib.hxq_assign(m._ptr(p), 64, 1, None, 8, m._ptr(lab), None) == m.HXQ_EINVAL
    assert m.lib.hxq_assign(m._ptr(p), 64, 1, m._ptr(p), 8, None, None) == m.HXQ_EINVAL
    assert m.lib.hxq_kmeans(None, 64, 1, 8, 1, m._ptr(p), None, None) == m.HXQ_EINVAL
    assert m.lib.hxq_kmeans(m._ptr(p), 64, 1, 8, 1, None, None, None) == m.HXQ_EINVAL
    assert m.lib.hxq_kmeans(m._ptr(p), 64, 1, 0, 1, m._ptr(p), None, None) == m.HXQ_EINVAL
    cnt = np.zeros(1, np.int64)
    assert m.lib.hxq_encode(None, 0, 8, 8, m._ptr(p), 0.1, m._ptr(lab), None, None, 0, m._ptr(cnt),
                            None) == m.HXQ_EINVAL
    assert m.lib.hxq_encode(m._ptr(p), 0, 8, 8, m._ptr(p), 0.1, m._ptr(lab), None, None, 0, None,
                            None) == m.HXQ_EINVAL


def test_create_without_device_reports_unsupported():
    import torch
    if torch.cuda.is_available():
        pytest.skip("a CUDA device is present")
    import vq_compressed_linear_b200 as m
    N, K = 16, 32
    rc = _create(m, np.zeros(256, np.float32), np.zeros(N * K, np.uint8), 0, None, None, 0, N, K)
    assert rc == m.HXQ_EUNSUPPORTED


def test_build_flags_target_sm100a():
    import __graft_entry__
    assert __graft_entry__._builder().ARCH == ["-gencode", "arch=compute_100a,code=sm_100a"]


def test_create_argument_rules_fuzzed():
    """hxq_linear_create's documented argument rules, over random shapes,
    modes, sidecar counts and NULL pointers: every violation returns
    HXQ_EINVAL before any CUDA call; arguments that pass reach the device
    check (HXQ_EUNSUPPORTED here, without a GPU)."""
    import torch
    if torch.cuda.is_available():
        pytest.skip("a CUDA device is present")
    from hypothesis import given, settings, strategies as st
    import vq_compressed_linear_b200 as m

    cb = np.zeros(8192, np.float32)
    idx = np.zeros(64, np.uint8)
    pos = np.zeros(4, np.int64)
    val = np.zeros(4, np.float32)

    @settings(max_examples=400, deadline=None, derandomize=True)
    @given(mode=st.integers(-1, 3), N=st.integers(-2, 1 << 20), K=st.integers(-16, 1 << 16),
           ns=st.one_of(st.integers(-3, 8), st.sampled_from([(1 << 31) - 1, 1 << 31, 1 << 40])),
           null_cb=st.booleans(), null_idx=st.booleans(), null_side=st.booleans(), null_out=st.booleans())
    def check(mode, N, K, ns, null_cb, null_idx, null_side, null_out):
        invalid = (null_cb or null_idx or null_out or mode not in (0, 1) or N < 1 or K < 1
                   or (mode == 1 and K % 4) or ns < 0 or ns > N * K or (ns > 0 and null_side) or ns >= (1 << 31))
        h = ctypes.c_void_p()
        rc = m.lib.hxq_linear_create(None if null_cb else m._ptr(cb), None if null_idx else m._ptr(idx), mode,
                                     None if null_side else m._ptr(pos), None if null_side else m._ptr(val),
                                     ns, N, K, None if null_out else ctypes.byref(h))
        assert rc == (m.HXQ_EINVAL if invalid else m.HXQ_EUNSUPPORTED), (mode, N, K, ns)
        assert h.value is None

    check()


def test_encoder_argument_rules_fuzzed():
    """hxq_assign / hxq_kmeans / hxq_encode: every documented argument error
    returns HXQ_EINVAL before any CUDA call; arguments that pass go on to
    the launch, which fails here without a GPU (HXQ_ECUDA), except a
    k-means call with nothing to do (no rounds, no labels): HXQ_OK."""
    import torch
    if torch.cuda.is_available():
        pytest.skip("a CUDA device is present")
    from hypothesis import given, settings, strategies as st
    import vq_compressed_linear_b200 as m

    buf = np.zeros(64, np.float32)
    lab = np.zeros(64, np.uint16)
    cnt = np.zeros(1, np.int64)
    P = lambda null: None if null else m._ptr(buf)
    big = st.sampled_from([(1 << 31) - 1, 1 << 31, 1 << 40])

    @settings(max_examples=300, deadline=None, derandomize=True)
    @given(n=st.one_of(st.integers(-2, 100), big), dim=st.integers(0, 3), k=st.integers(-1, 4100),
           iters=st.integers(-2, 3), nulls=st.lists(st.booleans(), min_size=3, max_size=3))
    def check_assign_kmeans(n, dim, k, iters, nulls):
        shape_bad = n < 1 or n >= (1 << 31) or dim not in (1, 2) or k < 1 or k > 4096
        rc = m.lib.hxq_assign(P(nulls[0]), n, dim, P(nulls[1]), k, None if nulls[2] else m._ptr(lab), None)
        assert rc == (m.HXQ_EINVAL if shape_bad or any(nulls) else m.HXQ_ECUDA), ("assign", n, dim, k, nulls)
        rc = m.lib.hxq_kmeans(P(nulls[0]), n, dim, k, iters, P(nulls[1]), None if nulls[2] else m._ptr(lab), None)
        if shape_bad or nulls[0] or nulls[1] or iters < 0:
            want = m.HXQ_EINVAL
        else:
            want = m.HXQ_OK if iters == 0 and nulls[2] else m.HXQ_ECUDA
        assert rc == want, ("kmeans", n, dim, k, iters, nulls)

    @settings(max_examples=300, deadline=None, derandomize=True)
    @given(mode=st.integers(-1, 2), N=st.integers(-1, 1 << 20), K=st.integers(-8, 1 << 14),
           t=st.sampled_from([0.0, 0.5, -1e-9, float("nan"), float("inf")]), cap=st.integers(-2, 5),
           nulls=st.lists(st.booleans(), min_size=5, max_size=5))
    def check_encode(mode, N, K, t, cap, nulls):
        bad = (nulls[0] or nulls[1] or nulls[2] or nulls[3] or mode not in (0, 1) or N < 1 or K < 1
               or (mode == 1 and K % 4) or N * K >= (1 << 31) or not (t >= 0) or cap < 0 or (cap > 0 and nulls[4]))
        side = None if nulls[4] else m._ptr(buf)
        rc = m.lib.hxq_encode(P(nulls[0]), mode, N, K, P(nulls[1]), t, P(nulls[2]), side, side, cap,
                              None if nulls[3] else m._ptr(cnt), None)
        assert rc == (m.HXQ_EINVAL if bad else m.HXQ_ECUDA), (mode, N, K, t, cap, nulls)

    check_assign_kmeans()
    check_encode()
