"""CPU oracle for the W8A16 linear layer -- TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and the benchmark's CPU-baseline
leg (``bench.py`` ``cpu_baseline`` and ``--impl reference``) may import this
package.  The product library (``int8_weight_only_b200``) never imports it and
shares no code with it.

The arithmetic lives in ``w8a16_oracle.c`` (plain C, single-threaded, built
with ``-O2 -fno-fast-math -ffp-contract=off``); this module only builds it and
marshals numpy arrays.  Every function here pins to the pages as documented in
the C file: per-output-channel symmetric int8 quantization (TPU-MLIR ChatGLM2
W8A16 article, sections 2-3; LightSeq 2020 slides "clipping + symmetric") and
the dequantized GEMM Y = X . (q o s) (+ bias) of that article's section 4, the
latter evaluated in fp64.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "w8a16_oracle.c")
_BUILD = os.path.join(_HERE, "_build")
_SO = os.path.join(_BUILD, "liboracle_w8a16.so")
_CFLAGS = ["-O2", "-std=c11", "-fno-fast-math", "-ffp-contract=off", "-fPIC", "-shared"]

_lock = threading.Lock()
_default = None


def build(force: bool = False, src: str = _SRC, out: str = _SO) -> str:
    """Compile the oracle with gcc (idempotent).  Returns the .so path."""
    os.makedirs(os.path.dirname(out), exist_ok=True)
    if (not force and os.path.exists(out)
            and os.path.getmtime(out) >= os.path.getmtime(src)):
        return out
    tmp = out + f".tmp{os.getpid()}"
    subprocess.check_call(["gcc", *_CFLAGS, "-o", tmp, src, "-lm"])
    os.replace(tmp, out)
    return out


def _ptr(a: np.ndarray):
    return a.ctypes.data_as(ctypes.c_void_p)


class Oracle:
    """numpy front end over one compiled copy of ``w8a16_oracle.c``."""

    def __init__(self, so_path: str):
        lib = ctypes.CDLL(so_path)
        i64 = ctypes.c_int64
        vp = ctypes.c_void_p
        lib.oracle_f32_to_f16_array.argtypes = [vp, i64, vp]
        lib.oracle_f16_to_f32_array.argtypes = [vp, i64, vp]
        lib.oracle_quantize_f32.argtypes = [vp, i64, i64, vp, vp, vp]
        lib.oracle_quantize_f16.argtypes = [vp, i64, i64, vp, vp, vp]
        lib.oracle_linear.argtypes = [vp, vp, vp, vp, i64, i64, i64, vp, vp]
        lib.oracle_quantize_asym_f32.argtypes = [vp, i64, i64, vp, vp, vp, vp]
        lib.oracle_quantize_asym_f16.argtypes = [vp, i64, i64, vp, vp, vp, vp]
        lib.oracle_linear_asym.argtypes = [vp, vp, vp, vp, vp, i64, i64, i64, vp, vp]
        lib.oracle_quantize_clip.argtypes = [vp, ctypes.c_int, i64, i64, ctypes.c_int, ctypes.c_double,
                                             vp, vp, vp, vp]
        lib.oracle_quantize_clip.restype = None
        lib.oracle_quantize_outliers.argtypes = [vp, ctypes.c_int, i64, i64, ctypes.c_double, vp, vp, vp, vp,
                                                 vp, vp, vp]
        lib.oracle_quantize_outliers.restype = None
        lib.oracle_linear_outliers.argtypes = [vp, vp, vp, vp, vp, vp, i64, vp, i64, i64, i64, vp, vp]
        lib.oracle_linear_outliers.restype = None
        for f in ("oracle_f32_to_f16_array", "oracle_f16_to_f32_array",
                  "oracle_quantize_f32", "oracle_quantize_f16", "oracle_linear",
                  "oracle_quantize_asym_f32", "oracle_quantize_asym_f16", "oracle_linear_asym"):
            getattr(lib, f).restype = None
        self.lib = lib
        self.path = so_path

    def f32_to_f16_bits(self, x) -> np.ndarray:
        """binary32 -> binary16 bit patterns, round to nearest even."""
        x = np.ascontiguousarray(x, dtype=np.float32)
        out = np.empty(x.shape, dtype=np.uint16)
        self.lib.oracle_f32_to_f16_array(_ptr(x), x.size, _ptr(out))
        return out

    def f16_bits_to_f32(self, h) -> np.ndarray:
        h = np.ascontiguousarray(h, dtype=np.uint16)
        out = np.empty(h.shape, dtype=np.float32)
        self.lib.oracle_f16_to_f32_array(_ptr(h), h.size, _ptr(out))
        return out

    def quantize(self, W: np.ndarray):
        """Per-output-channel symmetric int8 quantization.

        W: [K, N] float32 or float16.  Returns (q int8 [K, N], scales float16 [N]).
        """
        if W.ndim != 2:
            raise ValueError("W must be 2-D [K, N]")
        K, N = W.shape
        q = np.empty((K, N), dtype=np.int8)
        s = np.empty(N, dtype=np.uint16)
        buf = np.empty(max(K, 1), dtype=np.float32)
        if W.dtype == np.float32:
            Wc = np.ascontiguousarray(W)
            self.lib.oracle_quantize_f32(_ptr(Wc), K, N, _ptr(q), _ptr(s), _ptr(buf))
        elif W.dtype == np.float16:
            Wc = np.ascontiguousarray(W).view(np.uint16)
            self.lib.oracle_quantize_f16(_ptr(Wc), K, N, _ptr(q), _ptr(s), _ptr(buf))
        else:
            raise TypeError("W must be float32 or float16")
        return q, s.view(np.float16)

    def linear(self, X: np.ndarray, q: np.ndarray, scales: np.ndarray, bias=None) -> np.ndarray:
        """Y[M, N] = X . dequant(q) (+ bias) in fp64 (not rounded to fp16).

        X: [M, K] float16; q: [K, N] int8; scales: [N] float16; bias: [N]
        float16 or None.
        """
        M, K = X.shape
        K2, N = q.shape
        if K2 != K or scales.shape != (N,):
            raise ValueError("shape mismatch")
        Xc = np.ascontiguousarray(X, dtype=np.float16).view(np.uint16)
        qc = np.ascontiguousarray(q, dtype=np.int8)
        sc = np.ascontiguousarray(scales, dtype=np.float16).view(np.uint16)
        bc = None if bias is None else np.ascontiguousarray(bias, dtype=np.float16).view(np.uint16)
        Y = np.empty((M, N), dtype=np.float64)
        acc = np.empty(max(N, 1), dtype=np.float64)
        self.lib.oracle_linear(_ptr(Xc), _ptr(qc), _ptr(sc),
                               None if bc is None else _ptr(bc), M, K, N, _ptr(Y), _ptr(acc))
        return Y


    def quantize_asym(self, W: np.ndarray):
        """Per-output-channel asymmetric (affine) int8 quantization.

        W: [K, N] float32 or float16.  Returns (q int8 [K, N], scales
        float16 [N], zeros int8 [N]); a weight is dequantized as
        (q - zero) * scale.
        """
        if W.ndim != 2:
            raise ValueError("W must be 2-D [K, N]")
        K, N = W.shape
        q = np.empty((K, N), dtype=np.int8)
        s = np.empty(N, dtype=np.uint16)
        z = np.empty(N, dtype=np.int8)
        buf = np.empty(max(K, 1), dtype=np.float32)
        if W.dtype == np.float32:
            Wc = np.ascontiguousarray(W)
            self.lib.oracle_quantize_asym_f32(_ptr(Wc), K, N, _ptr(q), _ptr(s), _ptr(z), _ptr(buf))
        elif W.dtype == np.float16:
            Wc = np.ascontiguousarray(W).view(np.uint16)
            self.lib.oracle_quantize_asym_f16(_ptr(Wc), K, N, _ptr(q), _ptr(s), _ptr(z), _ptr(buf))
        else:
            raise TypeError("W must be float32 or float16")
        return q, s.view(np.float16), z

    def quantize_clip(self, W: np.ndarray, mode: str, param: float):
        """Clipped symmetric int8 quantization (same code format as
        ``quantize``).  mode "fixed": bound = min(max|W|, param); mode
        "percentile": bound = the ceil(param K)-th smallest |W| per channel.
        Returns (q int8 [K, N], scales float16 [N])."""
        if W.ndim != 2:
            raise ValueError("W must be 2-D [K, N]")
        modes = {"fixed": 0, "percentile": 1}
        if mode not in modes:
            raise ValueError("mode must be 'fixed' or 'percentile'")
        K, N = W.shape
        q = np.empty((K, N), dtype=np.int8)
        s = np.empty(N, dtype=np.uint16)
        buf = np.empty(max(K, 1), dtype=np.float32)
        sbuf = np.empty(max(K, 1), dtype=np.float32)
        if W.dtype == np.float32:
            Wc, f16 = np.ascontiguousarray(W), 0
        elif W.dtype == np.float16:
            Wc, f16 = np.ascontiguousarray(W).view(np.uint16), 1
        else:
            raise TypeError("W must be float32 or float16")
        self.lib.oracle_quantize_clip(_ptr(Wc), f16, K, N, modes[mode], float(param), _ptr(q), _ptr(s),
                                      _ptr(buf), _ptr(sbuf))
        return q, s.view(np.float16)

    def quantize_outliers(self, W: np.ndarray, p: float):
        """Outlier split: per channel, weights with |w| above the
        ceil(pK)-th smallest magnitude are kept as fp16 (code 0), the rest
        quantized with that bound.  Returns (q, scales, count int32 [N],
        rows int32 [N, cap], vals float16 [N, cap]) with cap = K - r."""
        if W.ndim != 2:
            raise ValueError("W must be 2-D [K, N]")
        K, N = W.shape
        rr = np.ceil(np.float64(p) * np.float64(K))
        r = int(min(max(rr, 1.0), float(K)))
        cap = K - r
        q = np.empty((K, N), dtype=np.int8)
        s = np.empty(N, dtype=np.uint16)
        cnt = np.empty(N, dtype=np.int32)
        rows = np.empty((N, max(cap, 0)), dtype=np.int32)
        vals = np.empty((N, max(cap, 0)), dtype=np.uint16)
        buf = np.empty(max(K, 1), dtype=np.float32)
        sbuf = np.empty(max(K, 1), dtype=np.float32)
        if W.dtype == np.float32:
            Wc, f16 = np.ascontiguousarray(W), 0
        elif W.dtype == np.float16:
            Wc, f16 = np.ascontiguousarray(W).view(np.uint16), 1
        else:
            raise TypeError("W must be float32 or float16")
        self.lib.oracle_quantize_outliers(_ptr(Wc), f16, K, N, float(p), _ptr(q), _ptr(s), _ptr(cnt),
                                          _ptr(rows), _ptr(vals), _ptr(buf), _ptr(sbuf))
        return q, s.view(np.float16), cnt, rows, vals.view(np.float16)

    def linear_outliers(self, X, q, scales, count, rows, vals, bias=None) -> np.ndarray:
        """Y = X . dequant(q) + X . outliers (+ bias) in fp64 (not rounded)."""
        M, K = X.shape
        K2, N = q.shape
        cap = rows.shape[1]
        if K2 != K or scales.shape != (N,) or count.shape != (N,) or vals.shape != (N, cap):
            raise ValueError("shape mismatch")
        Xc = np.ascontiguousarray(X, dtype=np.float16).view(np.uint16)
        qc = np.ascontiguousarray(q, dtype=np.int8)
        sc = np.ascontiguousarray(scales, dtype=np.float16).view(np.uint16)
        cc = np.ascontiguousarray(count, dtype=np.int32)
        rc = np.ascontiguousarray(rows, dtype=np.int32)
        vc = np.ascontiguousarray(vals, dtype=np.float16).view(np.uint16)
        bc = None if bias is None else np.ascontiguousarray(bias, dtype=np.float16).view(np.uint16)
        Y = np.empty((M, N), dtype=np.float64)
        acc = np.empty(max(N, 1), dtype=np.float64)
        self.lib.oracle_linear_outliers(_ptr(Xc), _ptr(qc), _ptr(sc), _ptr(cc), _ptr(rc), _ptr(vc), cap,
                                        None if bc is None else _ptr(bc), M, K, N, _ptr(Y), _ptr(acc))
        return Y

    def linear_asym(self, X, q, scales, zeros, bias=None) -> np.ndarray:
        """Y = X . ((q - zeros) o scales) (+ bias) in fp64 (not rounded)."""
        M, K = X.shape
        K2, N = q.shape
        if K2 != K or scales.shape != (N,) or zeros.shape != (N,):
            raise ValueError("shape mismatch")
        Xc = np.ascontiguousarray(X, dtype=np.float16).view(np.uint16)
        qc = np.ascontiguousarray(q, dtype=np.int8)
        sc = np.ascontiguousarray(scales, dtype=np.float16).view(np.uint16)
        zc = np.ascontiguousarray(zeros, dtype=np.int8)
        bc = None if bias is None else np.ascontiguousarray(bias, dtype=np.float16).view(np.uint16)
        Y = np.empty((M, N), dtype=np.float64)
        acc = np.empty(max(N, 1), dtype=np.float64)
        self.lib.oracle_linear_asym(_ptr(Xc), _ptr(qc), _ptr(sc), _ptr(zc),
                                    None if bc is None else _ptr(bc), M, K, N, _ptr(Y), _ptr(acc))
        return Y


def default() -> Oracle:
    global _default
    with _lock:
        if _default is None:
            _default = Oracle(build())
        return _default


def f32_to_f16_bits(x):
    return default().f32_to_f16_bits(x)


def f16_bits_to_f32(h):
    return default().f16_bits_to_f32(h)


def quantize(W):
    return default().quantize(W)


def linear(X, q, scales, bias=None):
    return default().linear(X, q, scales, bias)


def quantize_asym(W):
    return default().quantize_asym(W)


def linear_asym(X, q, scales, zeros, bias=None):
    return default().linear_asym(X, q, scales, zeros, bias)


def quantize_clip(W, mode, param):
    return default().quantize_clip(W, mode, param)


def quantize_outliers(W, p):
    return default().quantize_outliers(W, p)


def linear_outliers(X, q, scales, count, rows, vals, bias=None):
    return default().linear_outliers(X, q, scales, count, rows, vals, bias)


def tolerance_ok(y_test: np.ndarray, y_ref: np.ndarray):
    """The acceptance bound for Y (fixed by the problem statement):
    |Y - Y_ref| <= 2^-9 |Y_ref| + 1e-3 rms(Y_ref), element-wise.
    Returns (ok, worst ratio err / bound)."""
    y_ref = np.asarray(y_ref, dtype=np.float64)
    y_test = np.asarray(y_test, dtype=np.float64)
    rms = float(np.sqrt(np.mean(y_ref * y_ref))) if y_ref.size else 0.0
    bound = 2.0 ** -9 * np.abs(y_ref) + 1e-3 * rms
    err = np.abs(y_test - y_ref)
    if y_ref.size == 0:
        return True, 0.0
    with np.errstate(divide="ignore", invalid="ignore"):
        ratio = np.where(bound > 0, err / bound, np.where(err > 0, np.inf, 0.0))
    worst = float(np.max(ratio))
    return bool(np.all(err <= bound)), worst
