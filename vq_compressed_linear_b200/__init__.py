"""Python binding of libhxq, the B200 (sm_100a) HelixLinear forward.

The C ABI (include/hxq.h) is the product: this module only marshals
arguments. Every step of the forward runs in the library's CUDA kernels;
there is no Python or CPU fallback, and importing fails loudly when the
library has not been built (python vq_compressed_linear_b200/build.py).

PyTorch is used for device memory and streams only: tensors are passed by
data pointer, the current torch stream is passed as the cudaStream_t.
"""
from __future__ import annotations

import ctypes
import os

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libhxq.so")

if not os.path.exists(LIB_PATH):
    raise ImportError(
        f"libhxq.so is missing at {LIB_PATH}: build it with "
        "`python vq_compressed_linear_b200/build.py` (nvcc, sm_100a)")

lib = ctypes.CDLL(LIB_PATH)

HXQ_MODE_SCALAR8 = 0
HXQ_MODE_VQ2D12 = 1
HXQ_OK = 0
HXQ_EINVAL = -1
HXQ_ENOMEM = -2
HXQ_ECUDA = -3
HXQ_EUNSUPPORTED = -4
HXQ_ETIMEOUT = -5
HXQ_KERNEL_AUTO = 0
HXQ_KERNEL_GEMV = 1
HXQ_KERNEL_TC = 2
HXQ_OUT_F32 = 0
HXQ_OUT_BF16 = 1
HXQ_MAX_GROUP = 4

_vp, _i, _i64 = ctypes.c_void_p, ctypes.c_int, ctypes.c_int64
lib.hxq_linear_create.argtypes = [_vp, _vp, _i, _vp, _vp, _i64, _i, _i, ctypes.POINTER(_vp)]
lib.hxq_linear_create.restype = _i
lib.hxq_linear_forward.argtypes = [_vp, _vp, _vp, _i, _vp]
lib.hxq_linear_forward.restype = _i
lib.hxq_linear_forward_ex.argtypes = [_vp, _vp, _vp, _i, _i, _i, _vp]
lib.hxq_linear_forward_ex.restype = _i
lib.hxq_linear_forward_out.argtypes = [_vp, _vp, _vp, _vp, _i, _i, _vp]
lib.hxq_linear_forward_out.restype = _i
lib.hxq_linear_forward_host.argtypes = [_vp, _vp, _vp, _vp, _vp, _i, _vp]
lib.hxq_linear_forward_host.restype = _i
lib.hxq_linear_forward_noalloc.argtypes = [_vp, _vp, _vp, _i, _vp]
lib.hxq_linear_forward_noalloc.restype = _i
lib.hxq_decode.argtypes = [_vp, _vp, _vp]
lib.hxq_decode.restype = _i
lib.hxq_linear_check.argtypes = [_vp]
lib.hxq_linear_check.restype = _i
lib.hxq_test_forward_withheld.argtypes = [_vp, _vp, _vp, _i, _i, ctypes.c_uint, _vp]
lib.hxq_test_forward_withheld.restype = _i
lib.hxq_linear_info.argtypes = [_vp, ctypes.POINTER(_i), ctypes.POINTER(_i), ctypes.POINTER(_i),
                                ctypes.POINTER(_i64)]
lib.hxq_linear_info.restype = _i
lib.hxq_group_create.argtypes = [ctypes.POINTER(_vp), _i, ctypes.POINTER(_vp)]
lib.hxq_group_create.restype = _i
lib.hxq_group_forward.argtypes = [_vp, _vp, ctypes.POINTER(_vp), ctypes.POINTER(_vp), _i, _i, _vp]
lib.hxq_group_forward.restype = _i
lib.hxq_group_destroy.argtypes = [_vp]
lib.hxq_group_destroy.restype = None
lib.hxq_assign.argtypes = [_vp, _i64, _i, _vp, _i, _vp, _vp]
lib.hxq_assign.restype = _i
lib.hxq_kmeans.argtypes = [_vp, _i64, _i, _i, _i, _vp, _vp, _vp]
lib.hxq_kmeans.restype = _i
lib.hxq_encode.argtypes = [_vp, _i, _i, _i, _vp, ctypes.c_float, _vp, _vp, _vp, _i64, _vp, _vp]
lib.hxq_encode.restype = _i
lib.hxq_linear_destroy.argtypes = [_vp]
lib.hxq_linear_destroy.restype = None
lib.hxq_strerror.argtypes = [_i]
lib.hxq_strerror.restype = ctypes.c_char_p

EXPORTED = ("hxq_linear_create", "hxq_linear_forward", "hxq_linear_forward_ex", "hxq_linear_forward_out",
            "hxq_linear_forward_host", "hxq_linear_forward_noalloc", "hxq_group_create", "hxq_group_forward", "hxq_group_destroy", "hxq_assign", "hxq_kmeans", "hxq_encode", "hxq_decode",
            "hxq_linear_check", "hxq_test_forward_withheld", "hxq_linear_info", "hxq_linear_destroy",
            "hxq_strerror")


class HXQError(RuntimeError):
    def __init__(self, code: int, what: str):
        self.code = code
        super().__init__(f"{what}: {hxq_strerror(code)} ({code})")


def _check(code: int, what: str) -> None:
    if code != HXQ_OK:
        raise HXQError(code, what)


def _ptr(t) -> int | None:
    """Data pointer of a tensor / ndarray, or None."""
    if t is None:
        return None
    if hasattr(t, "data_ptr"):
        return t.data_ptr()
    return t.ctypes.data


def _stream(stream) -> int | None:
    if stream is not None:
        return int(getattr(stream, "cuda_stream", stream))
    import torch
    return torch.cuda.current_stream().cuda_stream


# ---- same names as the C ABI -------------------------------------------------

def hxq_strerror(code: int) -> str:
    return lib.hxq_strerror(int(code)).decode()


def hxq_linear_create(codebook, indices, mode, sidecar_pos, sidecar_val, n_sidecar, N, K) -> int:
    """Returns the handle (an integer); raises HXQError on failure."""
    h = _vp()
    _check(lib.hxq_linear_create(_ptr(codebook), _ptr(indices), int(mode), _ptr(sidecar_pos),
                                 _ptr(sidecar_val), int(n_sidecar), int(N), int(K), ctypes.byref(h)),
           "hxq_linear_create")
    return h.value


def hxq_linear_forward(h, x, y, M, stream=None) -> None:
    _check(lib.hxq_linear_forward(h, _ptr(x), _ptr(y), int(M), _stream(stream)), "hxq_linear_forward")


def hxq_linear_forward_ex(h, x, y, M, kernel, split_k, stream=None) -> None:
    _check(lib.hxq_linear_forward_ex(h, _ptr(x), _ptr(y), int(M), int(kernel), int(split_k),
                                     _stream(stream)), "hxq_linear_forward_ex")


def hxq_linear_forward_out(h, x, bias, y, out_dtype, M, stream=None) -> None:
    _check(lib.hxq_linear_forward_out(h, _ptr(x), _ptr(bias), _ptr(y), int(out_dtype), int(M), _stream(stream)),
           "hxq_linear_forward_out")


def hxq_linear_forward_host(h, x_host, x_dev, y_dev, y_host, M, stream=None) -> None:
    _check(lib.hxq_linear_forward_host(h, _ptr(x_host), _ptr(x_dev), _ptr(y_dev), _ptr(y_host), int(M),
                                       _stream(stream)), "hxq_linear_forward_host")


def hxq_linear_forward_noalloc(h, x, y, M, stream=None) -> None:
    _check(lib.hxq_linear_forward_noalloc(h, _ptr(x), _ptr(y), int(M), _stream(stream)),
           "hxq_linear_forward_noalloc")


def _ptr_array(ts):
    """A C array of data pointers (None entries stay NULL), or NULL for None."""
    if ts is None:
        return None
    return (_vp * len(ts))(*[_ptr(t) for t in ts])


def hxq_group_create(handles) -> int:
    """Returns the group (an integer); raises HXQError on failure."""
    g = _vp()
    arr = (_vp * len(handles))(*handles)
    _check(lib.hxq_group_create(arr, len(handles), ctypes.byref(g)), "hxq_group_create")
    return g.value


def hxq_group_forward(g, x, biases, ys, out_dtype, M, stream=None) -> None:
    _check(lib.hxq_group_forward(g, _ptr(x), _ptr_array(biases), _ptr_array(ys), int(out_dtype), int(M),
                                 _stream(stream)), "hxq_group_forward")


def hxq_group_destroy(g) -> None:
    lib.hxq_group_destroy(g)


def hxq_assign(points, n, dim, centroids, k, labels, stream=None) -> None:
    _check(lib.hxq_assign(_ptr(points), int(n), int(dim), _ptr(centroids), int(k), _ptr(labels), _stream(stream)),
           "hxq_assign")


def hxq_kmeans(points, n, dim, k, iters, centroids, labels, stream=None) -> None:
    _check(lib.hxq_kmeans(_ptr(points), int(n), int(dim), int(k), int(iters), _ptr(centroids), _ptr(labels),
                          _stream(stream)), "hxq_kmeans")


def hxq_encode(W, mode, N, K, codebook, threshold, indices, sidecar_pos, sidecar_val, max_sidecar, n_sidecar,
               stream=None) -> None:
    _check(lib.hxq_encode(_ptr(W), int(mode), int(N), int(K), _ptr(codebook), float(threshold), _ptr(indices),
                          _ptr(sidecar_pos), _ptr(sidecar_val), int(max_sidecar), _ptr(n_sidecar),
                          _stream(stream)), "hxq_encode")


def hxq_decode(h, W_out, stream=None) -> None:
    _check(lib.hxq_decode(h, _ptr(W_out), _stream(stream)), "hxq_decode")


def hxq_linear_check(h) -> None:
    _check(lib.hxq_linear_check(h), "hxq_linear_check")


def hxq_test_forward_withheld(h, x, y, M, withhold_item, wait_limit_us, stream=None) -> None:
    """Test hook: the tensor-core forward with one item's activations withheld
    and every pipeline wait bounded at wait_limit_us (the next
    hxq_linear_check reports HXQ_ETIMEOUT)."""
    _check(lib.hxq_test_forward_withheld(h, _ptr(x), _ptr(y), int(M), int(withhold_item), int(wait_limit_us),
                                         _stream(stream)), "hxq_test_forward_withheld")


def hxq_linear_info(h) -> tuple[int, int, int, int]:
    m, n, k, s = _i(), _i(), _i(), _i64()
    _check(lib.hxq_linear_info(h, ctypes.byref(m), ctypes.byref(n), ctypes.byref(k), ctypes.byref(s)),
           "hxq_linear_info")
    return m.value, n.value, k.value, s.value


def hxq_linear_destroy(h) -> None:
    lib.hxq_linear_destroy(h)


# ---- convenience wrapper -----------------------------------------------------

class HelixLinear:
    """A compressed nn.Linear-shaped layer owned by libhxq.

    Arguments are tensors or arrays in the C ABI's layouts (host or device);
    the handle copies them. forward() takes x as a CUDA bf16 (or raw uint16 /
    int16 bit pattern) tensor [M, K] and returns float32 y [M, N].
    """

    def __init__(self, codebook, indices, mode, sidecar_pos, sidecar_val, N, K):
        n_sidecar = 0 if sidecar_pos is None else int(len(sidecar_pos))
        if n_sidecar == 0:
            sidecar_pos = sidecar_val = None
        self.mode, self.N, self.K = int(mode), int(N), int(K)
        self.handle = hxq_linear_create(codebook, indices, mode, sidecar_pos, sidecar_val,
                                        n_sidecar, N, K)

    @classmethod
    def from_layer(cls, layer: dict) -> "HelixLinear":
        return cls(layer["codebook"], layer["indices"], layer["mode"], layer["sidecar_pos"],
                   layer["sidecar_val"], layer["N"], layer["K"])

    def forward(self, x, y=None, kernel=HXQ_KERNEL_AUTO, split_k=0, stream=None):
        import torch
        M = int(x.shape[0])
        if y is None:
            y = torch.empty((M, self.N), dtype=torch.float32, device=x.device)
        hxq_linear_forward_ex(self.handle, x, y, M, kernel, split_k, stream)
        return y

    __call__ = forward

    def forward_out(self, x, bias=None, out_dtype=HXQ_OUT_F32, y=None, stream=None):
        """y = x . W^T (+ bias) as float32, or as bfloat16 (rounded to nearest
        even) with out_dtype=HXQ_OUT_BF16."""
        import torch
        M = int(x.shape[0])
        if y is None:
            dt = torch.bfloat16 if out_dtype == HXQ_OUT_BF16 else torch.float32
            y = torch.empty((M, self.N), dtype=dt, device=x.device)
        hxq_linear_forward_out(self.handle, x, bias, y, out_dtype, M, stream)
        return y

    def forward_host(self, x_host, y_host, x_dev, y_dev, stream=None, sync=True):
        """End-to-end call on host buffers (hxq_linear_forward_host): copy x
        (pinned) in, run, copy y (pinned) out, all on `stream`. The caller
        owns the four buffers. With sync=False the call returns after
        enqueuing; synchronise the stream before reading y_host."""
        import torch
        s = stream or torch.cuda.current_stream()
        hxq_linear_forward_host(self.handle, x_host, x_dev, y_dev, y_host, int(x_dev.shape[0]), s)
        if sync:
            s.synchronize()
        return y_host

    def decode(self, stream=None):
        import torch
        W = torch.empty((self.N, self.K), dtype=torch.float32, device="cuda")
        hxq_decode(self.handle, W, stream)
        return W

    def check(self) -> None:
        hxq_linear_check(self.handle)

    def close(self) -> None:
        if getattr(self, "handle", None):
            hxq_linear_destroy(self.handle)
            self.handle = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass


class HelixGroup:
    """HelixLinear layers that read the same activations (one mode, one K),
    run by one launch for M <= 4 tokens. Borrows the layers: keep them alive
    while the group is used."""

    def __init__(self, layers):
        self.layers = list(layers)
        self.handle = hxq_group_create([l.handle for l in self.layers])

    def forward(self, x, biases=None, out_dtype=HXQ_OUT_F32, ys=None, stream=None):
        """[y_i = x . W_i^T (+ bias_i)] for every layer, float32 or bfloat16."""
        import torch
        M = int(x.shape[0])
        if ys is None:
            dt = torch.bfloat16 if out_dtype == HXQ_OUT_BF16 else torch.float32
            ys = [torch.empty((M, l.N), dtype=dt, device=x.device) for l in self.layers]
        hxq_group_forward(self.handle, x, biases, ys, out_dtype, M, stream)
        return ys

    __call__ = forward

    def close(self) -> None:
        if getattr(self, "handle", None):
            hxq_group_destroy(self.handle)
            self.handle = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass


# ---- encoder convenience ------------------------------------------------------

def kmeans(points, init, iters, stream=None):
    """Lloyd k-means on the GPU: points float32 CUDA [n] or [n, 2], init
    [k] or [k, 2]. Returns (centroids like init, labels int16 bits of the
    uint16 indices as an int32 tensor)."""
    import torch
    dim = 1 if points.dim() == 1 else int(points.shape[1])
    n, k = int(points.shape[0]), int(init.shape[0])
    cent = init.detach().to(device=points.device, dtype=torch.float32).contiguous().clone()
    lab = torch.empty(n, dtype=torch.int16, device=points.device)
    hxq_kmeans(points.contiguous(), n, dim, k, iters, cent, lab, stream)
    return cent, lab.to(torch.int32) & 0xFFFF


def encode(W, mode, codebook, threshold, max_sidecar=None, stream=None):
    """Indices and sidecar of W (float32 CUDA [N, K]) for a trained codebook,
    in the layout HelixLinear takes. Returns (indices uint8, sidecar_pos
    int64, sidecar_val float32), all CUDA tensors."""
    import torch
    N, K = int(W.shape[0]), int(W.shape[1])
    W = W.contiguous()
    cb = codebook.to(device=W.device, dtype=torch.float32).contiguous()
    nbytes = N * K if mode == HXQ_MODE_SCALAR8 else 3 * N * K // 4
    idx = torch.empty(nbytes, dtype=torch.uint8, device=W.device)
    count = torch.zeros(1, dtype=torch.int64, device=W.device)
    cap = max(1024, N * K // 100) if max_sidecar is None else int(max_sidecar)
    while True:
        pos = torch.empty(max(cap, 1), dtype=torch.int64, device=W.device)
        val = torch.empty(max(cap, 1), dtype=torch.float32, device=W.device)
        hxq_encode(W, mode, N, K, cb, threshold, idx, pos, val, cap, count, stream)
        n = int(count.item())
        if n <= cap or max_sidecar is not None:
            m = min(n, cap)
            return idx, pos[:m], val[:m]
        cap = n
