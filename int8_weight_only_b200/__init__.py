"""W8A16 linear layer for NVIDIA B200: Python binding over libw8a16.so.

This module only marshals arguments: every step of the computation runs in
the CUDA kernels behind the C ABI declared in ``include/w8a16.h``.  PyTorch
is used for device memory and the current stream.  There is no CPU path: if
the library cannot be loaded, every call raises.

    q, scales = quantize(W)              # W: [K, N] fp32/fp16 cuda tensor
    packed = prepack(q)                  # tiled layout for the linear kernels
    Y = linear(X, packed, scales, bias)  # X: [M, K] fp16 -> Y: [M, N] fp16

``W8A16Linear`` bundles the three for a weight that is reused.
"""
from __future__ import annotations

import ctypes
import os
import threading

__all__ = [
    "W8Error", "load_library", "library_path", "quantize", "quantize_batched", "quantize_asym", "quantize_clip", "quantize_outliers", "prepack", "unpack",
    "prepacked_bytes", "workspace_bytes", "linear", "linear_asym", "linear_outliers", "linear_decode_static", "W8A16Linear", "device_status",
    "test_bounded_wait", "STATUS",
]

_HERE = os.path.dirname(os.path.abspath(__file__))
_LIB_PATH = os.path.join(_HERE, "libw8a16.so")

STATUS = {
    0: "W8_OK", -1: "W8_ERR_NULL", -2: "W8_ERR_SHAPE", -3: "W8_ERR_ALIGN", -4: "W8_ERR_DTYPE",
    -5: "W8_ERR_WORKSPACE", -6: "W8_ERR_CUDA", -7: "W8_ERR_TIMEOUT", -8: "W8_ERR_ALIAS",
    -9: "W8_ERR_DEVICE", -10: "W8_ERR_LIMIT",
}
W8_F32, W8_F16 = 0, 1

_lock = threading.Lock()
_lib = None


class W8Error(RuntimeError):
    def __init__(self, status: int, what: str):
        self.status = status
        self.name = STATUS.get(status, str(status))
        msg = _lib.w8_error_string(status).decode() if _lib is not None else self.name
        super().__init__(f"{what}: {self.name} ({msg})")


def library_path() -> str:
    return _LIB_PATH


def load_library():
    """Load libw8a16.so (raises if it has not been built)."""
    global _lib
    with _lock:
        if _lib is not None:
            return _lib
        if not os.path.exists(_LIB_PATH):
            raise RuntimeError(
                f"{_LIB_PATH} is missing: build it with `python -m int8_weight_only_b200.build`")
        lib = ctypes.CDLL(_LIB_PATH)
        vp, i64, i32, sz = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int, ctypes.c_size_t
        lib.w8_quantize_per_channel.argtypes = [vp, i32, i64, i64, vp, vp, vp]
        lib.w8_quantize_per_channel_asym.argtypes = [vp, i32, i64, i64, vp, vp, vp, vp]
        lib.w8_quantize_per_channel_batched.argtypes = [i32, vp, i32, vp, vp, vp, vp, vp]
        lib.w8_quantize_per_channel_clip.argtypes = [vp, i32, i64, i64, i32, ctypes.c_double, vp, vp, vp]
        lib.w8_outlier_capacity.argtypes = [i64, ctypes.c_double]
        lib.w8_outlier_capacity.restype = sz
        lib.w8_quantize_per_channel_outliers.argtypes = [vp, i32, i64, i64, ctypes.c_double, vp, vp, vp, vp, vp,
                                                         vp]
        lib.w8a16_linear_outliers_workspace_bytes.argtypes = [i64, i64, i64]
        lib.w8a16_linear_outliers_workspace_bytes.restype = sz
        lib.w8a16_linear_outliers.argtypes = [vp, vp, vp, vp, vp, vp, i64, vp, vp, i64, i64, i64, vp, sz, vp]
        lib.w8a16_linear_asym.argtypes = [vp, vp, vp, vp, vp, vp, i64, i64, i64, vp, sz, vp]
        lib.w8_prepacked_bytes.argtypes = [i64, i64]
        lib.w8_prepacked_bytes.restype = sz
        lib.w8_prepack.argtypes = [vp, i64, i64, vp, vp]
        lib.w8_unpack.argtypes = [vp, i64, i64, vp, vp]
        lib.w8a16_workspace_bytes.argtypes = [i64, i64, i64]
        lib.w8a16_workspace_bytes.restype = sz
        lib.w8a16_linear.argtypes = [vp, vp, vp, vp, vp, i64, i64, i64, vp, sz, vp]
        lib.w8a16_linear_decode_static.argtypes = [vp, vp, vp, vp, vp, i64, i64, i64, vp]
        lib.w8_error_string.argtypes = [i32]
        lib.w8_error_string.restype = ctypes.c_char_p
        lib.w8_device_status.argtypes = [vp, ctypes.POINTER(ctypes.c_uint32)]
        lib.w8_test_bounded_wait.argtypes = [ctypes.c_uint64, vp]
        lib.w8_test_set_decode_helper_delay.argtypes = [ctypes.c_uint64]
        lib.w8_version.argtypes = []
        for f in ("w8_quantize_per_channel", "w8_prepack", "w8_unpack", "w8a16_linear",
                  "w8a16_linear_decode_static",
                  "w8_device_status", "w8_test_bounded_wait", "w8_test_set_decode_helper_delay",
                  "w8_version"):
            getattr(lib, f).restype = i32
        _lib = lib
        return lib


def _check(rc: int, what: str):
    if rc != 0:
        raise W8Error(rc, what)


def _torch():
    import torch
    return torch


def _stream(device):
    torch = _torch()
    return ctypes.c_void_p(torch.cuda.current_stream(device).cuda_stream)


def _ptr(t):
    return ctypes.c_void_p(t.data_ptr()) if t is not None else None


def _need_cuda(t, name):
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")


def prepacked_bytes(K: int, N: int) -> int:
    return int(load_library().w8_prepacked_bytes(K, N))


def quantize(W, q=None, scales=None):
    """Per-output-channel symmetric int8 quantization of W [K, N].

    Returns (q int8 [K, N], scales fp16 [N]) on W's device.
    """
    torch = _torch()
    lib = load_library()
    _need_cuda(W, "W")
    if W.dim() != 2:
        raise ValueError("W must be [K, N]")
    if W.dtype == torch.float32:
        dt = W8_F32
    elif W.dtype == torch.float16:
        dt = W8_F16
    else:
        raise ValueError("W must be float32 or float16")
    K, N = W.shape
    if q is None:
        q = torch.empty((K, N), dtype=torch.int8, device=W.device)
    if scales is None:
        scales = torch.empty((N,), dtype=torch.float16, device=W.device)
    with torch.cuda.device(W.device):
        _check(lib.w8_quantize_per_channel(_ptr(W), dt, K, N, _ptr(q), _ptr(scales), _stream(W.device)),
               "w8_quantize_per_channel")
    return q, scales


def quantize_batched(Ws, qs=None, scales=None):
    """Per-output-channel symmetric int8 quantization of several weights in
    as few launches as possible (up to 64 per launch).  Ws: list of [K, N]
    tensors of one dtype (float32 or float16) on one device.  Returns
    (list of q int8, list of scales fp16), bit for bit those of quantize."""
    torch = _torch()
    lib = load_library()
    Ws = list(Ws)
    if not Ws:
        return [], []
    dev = Ws[0].device
    dtype = Ws[0].dtype
    for W in Ws:
        _need_cuda(W, "W")
        if W.dim() != 2 or W.dtype != dtype or W.device != dev:
            raise ValueError("Ws must be 2-D tensors of one dtype on one device")
    if dtype == torch.float32:
        dt = W8_F32
    elif dtype == torch.float16:
        dt = W8_F16
    else:
        raise ValueError("W must be float32 or float16")
    if qs is None:
        qs = [torch.empty(tuple(W.shape), dtype=torch.int8, device=dev) for W in Ws]
    if scales is None:
        scales = [torch.empty((W.shape[1],), dtype=torch.float16, device=dev) for W in Ws]
    n = len(Ws)
    arr_p = ctypes.c_void_p * n
    arr_i = ctypes.c_int64 * n
    with torch.cuda.device(dev):
        _check(lib.w8_quantize_per_channel_batched(
            n, arr_p(*[W.data_ptr() for W in Ws]), dt, arr_i(*[W.shape[0] for W in Ws]),
            arr_i(*[W.shape[1] for W in Ws]), arr_p(*[q.data_ptr() for q in qs]),
            arr_p(*[s.data_ptr() for s in scales]), _stream(dev)), "w8_quantize_per_channel_batched")
    return qs, scales


def quantize_asym(W, q=None, scales=None, zeros=None):
    """Per-output-channel asymmetric (affine) int8 quantization of W [K, N].

    Returns (q int8 [K, N], scales fp16 [N], zeros int8 [N]) on W's device;
    a weight is dequantized as (q - zero) * scale.
    """
    torch = _torch()
    lib = load_library()
    _need_cuda(W, "W")
    if W.dim() != 2:
        raise ValueError("W must be [K, N]")
    if W.dtype == torch.float32:
        dt = W8_F32
    elif W.dtype == torch.float16:
        dt = W8_F16
    else:
        raise ValueError("W must be float32 or float16")
    K, N = W.shape
    if q is None:
        q = torch.empty((K, N), dtype=torch.int8, device=W.device)
    if scales is None:
        scales = torch.empty((N,), dtype=torch.float16, device=W.device)
    if zeros is None:
        zeros = torch.empty((N,), dtype=torch.int8, device=W.device)
    with torch.cuda.device(W.device):
        _check(lib.w8_quantize_per_channel_asym(_ptr(W), dt, K, N, _ptr(q), _ptr(scales), _ptr(zeros),
                                                _stream(W.device)), "w8_quantize_per_channel_asym")
    return q, scales, zeros


W8_CLIP_FIXED, W8_CLIP_PERCENTILE = 0, 1


def quantize_clip(W, mode, param, q=None, scales=None):
    """Symmetric int8 quantization of W [K, N] with a clipped bound.

    mode "fixed": bound = min(max|W|, param) per channel; mode "percentile":
    bound = the ceil(param K)-th smallest |W| per channel.  Returns
    (q int8 [K, N], scales fp16 [N]) in the format of ``quantize``.
    """
    torch = _torch()
    lib = load_library()
    _need_cuda(W, "W")
    modes = {"fixed": W8_CLIP_FIXED, "percentile": W8_CLIP_PERCENTILE}
    if mode not in modes:
        raise ValueError("mode must be 'fixed' or 'percentile'")
    if W.dim() != 2:
        raise ValueError("W must be [K, N]")
    if W.dtype == torch.float32:
        dt = W8_F32
    elif W.dtype == torch.float16:
        dt = W8_F16
    else:
        raise ValueError("W must be float32 or float16")
    K, N = W.shape
    if q is None:
        q = torch.empty((K, N), dtype=torch.int8, device=W.device)
    if scales is None:
        scales = torch.empty((N,), dtype=torch.float16, device=W.device)
    with torch.cuda.device(W.device):
        _check(lib.w8_quantize_per_channel_clip(_ptr(W), dt, K, N, modes[mode], float(param), _ptr(q),
                                                _ptr(scales), _stream(W.device)), "w8_quantize_per_channel_clip")
    return q, scales


def quantize_outliers(W, p):
    """Outlier split of W [K, N]: per channel the weights above the
    ceil(pK)-th smallest magnitude are kept as fp16 (code 0); the rest is
    quantized with that bound.  Returns (q int8 [K, N], scales fp16 [N],
    count int32 [N], rows int32 [N, cap], vals fp16 [N, cap])."""
    torch = _torch()
    lib = load_library()
    _need_cuda(W, "W")
    if W.dim() != 2:
        raise ValueError("W must be [K, N]")
    if W.dtype == torch.float32:
        dt = W8_F32
    elif W.dtype == torch.float16:
        dt = W8_F16
    else:
        raise ValueError("W must be float32 or float16")
    K, N = W.shape
    cap = int(lib.w8_outlier_capacity(K, float(p)))
    dev = W.device
    q = torch.empty((K, N), dtype=torch.int8, device=dev)
    scales = torch.empty((N,), dtype=torch.float16, device=dev)
    count = torch.empty((N,), dtype=torch.int32, device=dev)
    rows = torch.empty((N, cap), dtype=torch.int32, device=dev)
    vals = torch.empty((N, cap), dtype=torch.float16, device=dev)
    with torch.cuda.device(dev):
        _check(lib.w8_quantize_per_channel_outliers(_ptr(W), dt, K, N, float(p), _ptr(q), _ptr(scales),
                                                    _ptr(count), _ptr(rows) if cap else None,
                                                    _ptr(vals) if cap else None, _stream(dev)),
               "w8_quantize_per_channel_outliers")
    return q, scales, count, rows, vals


def linear_outliers(X, packed, scales, count, rows, vals, bias=None, out=None, workspace=None):
    """Y [M, N] fp16 = X . dequant(q) + X . outliers (+ bias), for the
    output of quantize_outliers (q prepacked)."""
    torch = _torch()
    lib = load_library()
    _need_cuda(X, "X")
    if X.dim() != 2 or X.dtype != torch.float16:
        raise ValueError("X must be [M, K] float16")
    M, K = X.shape
    N = scales.shape[0]
    cap = rows.shape[1]
    if out is None:
        out = torch.empty((M, N), dtype=torch.float16, device=X.device)
    with torch.cuda.device(X.device):
        need = int(lib.w8a16_linear_outliers_workspace_bytes(M, K, N))
        ws = workspace if workspace is not None else _workspace(X.device, need)
        ws_bytes = 0 if ws is None else ws.numel() * ws.element_size()
        _check(lib.w8a16_linear_outliers(_ptr(X), _ptr(packed), _ptr(scales), _ptr(count),
                                         _ptr(rows) if cap else None, _ptr(vals) if cap else None, cap, _ptr(bias),
                                         _ptr(out), M, K, N, _ptr(ws), ws_bytes, _stream(X.device)),
               "w8a16_linear_outliers")
    return out


def prepack(q, out=None):
    """Reorder q [K, N] int8 into the tiled layout (uint8, flat)."""
    torch = _torch()
    lib = load_library()
    _need_cuda(q, "q")
    K, N = q.shape
    if out is None:
        out = torch.empty((prepacked_bytes(K, N),), dtype=torch.uint8, device=q.device)
    with torch.cuda.device(q.device):
        _check(lib.w8_prepack(_ptr(q), K, N, _ptr(out), _stream(q.device)), "w8_prepack")
    return out


def unpack(packed, K: int, N: int, out=None):
    """Inverse of prepack: packed -> q [K, N] int8."""
    torch = _torch()
    lib = load_library()
    _need_cuda(packed, "packed")
    if out is None:
        out = torch.empty((K, N), dtype=torch.int8, device=packed.device)
    with torch.cuda.device(packed.device):
        _check(lib.w8_unpack(_ptr(packed), K, N, _ptr(out), _stream(packed.device)), "w8_unpack")
    return out


def workspace_bytes(M: int, K: int, N: int, device=None) -> int:
    torch = _torch()
    with torch.cuda.device(device if device is not None else torch.cuda.current_device()):
        return int(load_library().w8a16_workspace_bytes(M, K, N))


_ws_cache = {}


def _workspace(device, nbytes: int):
    """The default split-K scratch: one zero-filled buffer per (device,
    stream), grown on demand.  The kernels leave it zeroed after every
    completed call, so calls on one stream (which never overlap) reuse it;
    calls on two streams may overlap on the GPU and so get two buffers."""
    torch = _torch()
    if nbytes == 0:
        return None
    dev = torch.device(device)
    key = (dev.index, torch.cuda.current_stream(dev).cuda_stream)
    buf = _ws_cache.get(key)
    if buf is None or buf.numel() < nbytes:
        buf = torch.zeros((max(nbytes, 1 << 20),), dtype=torch.uint8, device=dev)
        _ws_cache[key] = buf
    return buf


def _reset_workspaces(device_index: int):
    """Zero every default workspace of a device.  A kernel whose bounded wait
    gave up may have left split-K counters set; the next call through that
    workspace would otherwise start from them."""
    for (dev, _), buf in _ws_cache.items():
        if dev == device_index:
            buf.zero_()


def linear(X, packed, scales, bias=None, out=None, workspace=None):
    """Y [M, N] fp16 = X [M, K] fp16 . dequant(packed, scales) (+ bias)."""
    torch = _torch()
    lib = load_library()
    _need_cuda(X, "X")
    if X.dim() != 2 or X.dtype != torch.float16:
        raise ValueError("X must be [M, K] float16")
    M, K = X.shape
    N = scales.shape[0]
    if out is None:
        out = torch.empty((M, N), dtype=torch.float16, device=X.device)
    with torch.cuda.device(X.device):
        need = int(lib.w8a16_workspace_bytes(M, K, N))
        ws = workspace if workspace is not None else _workspace(X.device, need)
        ws_bytes = 0 if ws is None else ws.numel() * ws.element_size()
        _check(lib.w8a16_linear(_ptr(X), _ptr(packed), _ptr(scales), _ptr(bias), _ptr(out),
                                M, K, N, _ptr(ws), ws_bytes, _stream(X.device)), "w8a16_linear")
    return out


def linear_asym(X, packed, scales, zeros, bias=None, out=None, workspace=None):
    """Y [M, N] fp16 = X [M, K] fp16 . ((q - zeros) o scales) (+ bias), for
    codes from quantize_asym."""
    torch = _torch()
    lib = load_library()
    _need_cuda(X, "X")
    if X.dim() != 2 or X.dtype != torch.float16:
        raise ValueError("X must be [M, K] float16")
    M, K = X.shape
    N = scales.shape[0]
    if zeros.dtype != torch.int8 or zeros.shape != (N,):
        raise ValueError("zeros must be [N] int8")
    if out is None:
        out = torch.empty((M, N), dtype=torch.float16, device=X.device)
    with torch.cuda.device(X.device):
        need = int(lib.w8a16_workspace_bytes(M, K, N))
        ws = workspace if workspace is not None else _workspace(X.device, need)
        ws_bytes = 0 if ws is None else ws.numel() * ws.element_size()
        _check(lib.w8a16_linear_asym(_ptr(X), _ptr(packed), _ptr(scales), _ptr(zeros), _ptr(bias), _ptr(out),
                                     M, K, N, _ptr(ws), ws_bytes, _stream(X.device)), "w8a16_linear_asym")
    return out


def linear_decode_static(X, packed, scales, bias=None, out=None):
    """Decode-path linear (M <= 16) that needs no workspace: its scratch is a
    fixed array of static device memory inside the library.  For callers
    that cannot allocate device memory (an operator inside a host framework
    whose signature has no workspace argument, or a loop whose memory is
    planned up front by another allocator).  Calls that may overlap on the
    GPU share that array and must be ordered by the caller."""
    torch = _torch()
    lib = load_library()
    _need_cuda(X, "X")
    if X.dim() != 2 or X.dtype != torch.float16:
        raise ValueError("X must be [M, K] float16")
    M, K = X.shape
    N = scales.shape[0]
    if out is None:
        out = torch.empty((M, N), dtype=torch.float16, device=X.device)
    with torch.cuda.device(X.device):
        _check(lib.w8a16_linear_decode_static(_ptr(X), _ptr(packed), _ptr(scales), _ptr(bias),
                                              _ptr(out), M, K, N, _stream(X.device)),
               "w8a16_linear_decode_static")
    return out


class W8A16Linear:
    """A linear layer whose weight W [K, N] is stored as int8 + fp16 scales."""

    def __init__(self, W, bias=None):
        q, self.scales = quantize(W)
        self.K, self.N = W.shape
        self.packed = prepack(q)
        self.bias = bias

    def __call__(self, X, out=None):
        return linear(X, self.packed, self.scales, self.bias, out=out)


def device_status(device=None) -> int:
    """Synchronize and read (then clear) the device status word.  A nonzero
    value means a bounded device wait gave up; the default workspaces of the
    device are then zeroed, so later calls without ``workspace=`` start from
    clean split-K counters (a caller-owned workspace must be zeroed by its
    owner, as include/w8a16.h states)."""
    torch = _torch()
    lib = load_library()
    dev = device if device is not None else torch.cuda.current_device()
    v = ctypes.c_uint32(0)
    with torch.cuda.device(dev):
        _check(lib.w8_device_status(_stream(dev), ctypes.byref(v)), "w8_device_status")
        if v.value != 0:
            # a wait ran out: the default workspaces may hold stale counters
            _reset_workspaces(torch.device("cuda", torch.cuda.current_device()).index)
            torch.cuda.synchronize()
    return int(v.value)


def test_bounded_wait(limit_ns: int, device=None):
    torch = _torch()
    lib = load_library()
    dev = device if device is not None else torch.cuda.current_device()
    with torch.cuda.device(dev):
        _check(lib.w8_test_bounded_wait(limit_ns, _stream(dev)), "w8_test_bounded_wait")


test_bounded_wait.__test__ = False   # not a pytest test


def test_set_decode_helper_delay(delay_ns: int, device=None):
    """Test hook: delay the decode kernel's count of each CTA's first part."""
    torch = _torch()
    lib = load_library()
    dev = device if device is not None else torch.cuda.current_device()
    with torch.cuda.device(dev):
        _check(lib.w8_test_set_decode_helper_delay(delay_ns), "w8_test_set_decode_helper_delay")


test_set_decode_helper_delay.__test__ = False   # not a pytest test
