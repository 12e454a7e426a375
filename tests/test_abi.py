"""C-ABI boundary checks that need no GPU: the library loads, exports every
function include/w8a16.h declares, computes sizes by the documented closed
forms, and rejects invalid arguments on the host before any CUDA call."""
import ctypes
import os
import re

import pytest

from tests import golden

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "w8a16.h")

# fake, 16-byte aligned addresses: validation must reject before touching them
A = ctypes.c_void_p(0x10000)
B = ctypes.c_void_p(0x20000000)
C = ctypes.c_void_p(0x40000000)
D = ctypes.c_void_p(0x60000000)
E = ctypes.c_void_p(0x70000000)


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(w8a?1?6?_\w+)\s*\(", text)))


def test_header_declares_the_boundary():
    names = declared_functions()
    for need in ("w8_quantize_per_channel", "w8_prepack", "w8a16_linear", "w8_prepacked_bytes",
                 "w8a16_workspace_bytes", "w8_error_string", "w8_unpack"):
        assert need in names


def test_every_declared_symbol_is_exported(w8lib):
    for name in declared_functions():
        assert hasattr(w8lib, name), name


def test_error_strings(w8lib):
    for code in range(0, -10, -1):
        s = w8lib.w8_error_string(code).decode()
        assert s and s != "unknown status"
    assert w8lib.w8_error_string(-99).decode() == "unknown status"
    assert w8lib.w8_version() == 100


def test_prepacked_bytes_closed_form(w8lib):
    f = w8lib.w8_prepacked_bytes
    assert f(64, 128) == 8192
    assert f(1, 8) == 8192
    assert f(65, 136) == 2 * 2 * 8192
    assert f(0, 128) == 0 and f(64, 0) == 0
    # the page's ChatGLM2 weight: int8 storage is exactly K*N bytes (107 MB)
    g = golden.load("chatglm2_h_to_4h_weight_bytes.txt")
    K, N = g["K"], g["N"]
    assert f(K, N) == K * N
    assert round(f(K, N) / 2 ** 20) == g["int8_mb"]
    assert round(2 * K * N / 2 ** 20) == g["f16_mb"]


def test_quantize_rejects_bad_arguments(w8lib):
    q = w8lib.w8_quantize_per_channel
    assert q(None, 0, 4, 8, B, C, None) == -1
    assert q(A, 0, 4, 8, None, C, None) == -1
    assert q(A, 7, 4, 8, B, C, None) == -4
    assert q(A, 0, 0, 8, B, C, None) == -2
    assert q(A, 0, 4, 12, B, C, None) == -2          # N % 8
    assert q(ctypes.c_void_p(0x10004), 0, 4, 8, B, C, None) == -3
    assert q(A, 0, 4, 8, ctypes.c_void_p(0x10000 + 16), C, None) == -8   # q inside W
    assert q(A, 0, 4, 0, B, C, None) == 0                                   # empty: no-op
    assert q(None, 0, 4, 0, None, None, None) == 0                          # empty tensors


def test_pack_rejects_bad_arguments(w8lib):
    for fn in (w8lib.w8_prepack, w8lib.w8_unpack):
        assert fn(None, 64, 128, B, None) == -1
        assert fn(A, 0, 128, B, None) == -2
        assert fn(A, 64, 100, B, None) == -2
        assert fn(A, 64, 128, ctypes.c_void_p(0x20000008), None) == -3
        assert fn(A, 64, 128, ctypes.c_void_p(0x10000 + 4096), None) == -8
    # ragged shape: q holds K*N = 8840 bytes, the packed copy 4 tiles; a
    # packed buffer that starts right after q does not overlap it
    K, N = 65, 136
    qa, pk = 0x10000, 0x10000 + ((K * N + 15) // 16) * 16
    assert w8lib.w8_prepacked_bytes(K, N) > K * N
    # valid arguments reach the CUDA runtime (-6 without a device) instead
    # of being refused as overlapping
    assert w8lib.w8_prepack(ctypes.c_void_p(qa), K, N, ctypes.c_void_p(pk), None) != -8
    assert w8lib.w8_unpack(ctypes.c_void_p(pk), K, N, ctypes.c_void_p(qa), None) != -8
    assert w8lib.w8_prepack(ctypes.c_void_p(qa), K, N, ctypes.c_void_p(pk - 16), None) == -8


def test_linear_rejects_bad_arguments(w8lib):
    L = w8lib.w8a16_linear
    assert L(None, B, C, None, D, 1, 64, 128, E, 1 << 20, None) == -1
    assert L(A, B, C, None, None, 1, 64, 128, E, 1 << 20, None) == -1
    assert L(A, B, C, None, D, -1, 64, 128, E, 1 << 20, None) == -2
    assert L(A, B, C, None, D, 1, 60, 128, E, 1 << 20, None) == -2     # K % 8
    assert L(A, B, C, None, D, 1, 64, 100, E, 1 << 20, None) == -2     # N % 8
    assert L(A, B, C, None, D, 1, 0, 128, E, 1 << 20, None) == -2
    assert L(A, B, C, ctypes.c_void_p(0x3), D, 1, 64, 128, E, 1 << 20, None) == -3
    assert L(A, B, C, None, ctypes.c_void_p(0x10000 + 64), 1, 64, 128, E, 1 << 20, None) == -8
    assert L(A, B, C, None, D, 0, 64, 128, E, 1 << 20, None) == 0        # M == 0: no-op
    assert L(None, B, C, None, None, 0, 64, 128, None, 0, None) == 0     # empty X, Y
    assert L(None, None, C, None, None, 0, 64, 128, None, 0, None) == -1


def test_valid_call_without_gpu_fails_loudly(w8lib):
    import torch
    if torch.cuda.is_available():
        pytest.skip("a GPU is present")
    # a well-formed call reaches the CUDA runtime, which has no device here:
    # the library reports an error instead of computing anything on the CPU
    assert w8lib.w8a16_linear(A, B, C, None, D, 1, 64, 128, E, 1 << 20, None) == -6
    assert w8lib.w8_quantize_per_channel(A, 0, 64, 128, B, C, None) == -6
    assert w8lib.w8a16_workspace_bytes(1, 64, 128) == 0


def test_decode_helper_delay_hook_range(w8lib):
    # checked on the host before any CUDA call
    w8lib.w8_test_set_decode_helper_delay.argtypes = [ctypes.c_uint64]
    assert w8lib.w8_test_set_decode_helper_delay(1_000_001) == -2
    assert w8lib.w8_test_set_decode_helper_delay(1 << 40) == -2
