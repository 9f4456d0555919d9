"""The C-ABI library on CPU: it loads, exports every symbol include/q4k.h declares,
and its host-side logic (sizes, status strings, argument validation, launch
plans) behaves. No call here reaches the GPU: every q4k_gemv / q4k_dequant_f32
call below has an argument the library refuses before any CUDA call."""
import ctypes
import os
import re

import pytest

import gguf_quant_dequant_q4k_b200 as q4k
from gguf_quant_dequant_q4k_b200 import capi

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "q4k.h")


def declared_functions():
    with open(HEADER) as f:
        text = f.read()
    return sorted(set(re.findall(r"Q4K_API\s+[^;(]*?\b(q4k_\w+)\s*\(", text)))


def test_header_declares_the_binding_exports():
    assert declared_functions() == sorted(capi.EXPORTS)


def test_library_exports_every_declared_symbol():
    lib = ctypes.CDLL(capi.LIB_PATH)
    for name in declared_functions():
        assert hasattr(lib, name), name


def test_weight_bytes_size_rule():
    for n, k in [(256, 1024), (8960, 1536), (1536, 8960), (11008, 4096), (128256, 4096),
                 (4096, 14336), (1, 256)]:
        assert q4k.q4k_weight_bytes(n, k) == n * (k // 256) * 144
    assert q4k.q4k_weight_bytes(128256, 4096) == 295_501_824
    for n, k in [(0, 256), (-1, 256), (4, 0), (4, 255), (4, 257), (4, -256)]:
        assert q4k.q4k_weight_bytes(n, k) == 0
    # the size of the largest int shape does not overflow 64 bits
    assert q4k.q4k_weight_bytes(2**31 - 1, 2**31 - 256) == (2**31 - 1) * ((2**31 - 256) // 256) * 144


def test_status_strings():
    for st in range(7):
        assert q4k.q4k_status_string(st)
    assert q4k.q4k_status_string(99) == "unknown status"
    assert q4k.q4k_last_cuda_error() == 0


A16 = 1 << 20  # a 16-byte-aligned fake address; never dereferenced


@pytest.mark.parametrize("args,expect", [
    ((0, A16, A16 + 4096, 1, 4, 256), q4k.Q4K_ERR_NULL),
    ((A16, 0, A16 + 4096, 1, 4, 256), q4k.Q4K_ERR_NULL),
    ((A16, A16 + 4096, 0, 1, 4, 256), q4k.Q4K_ERR_NULL),
    ((A16, A16 * 2, A16 * 3, 1, 4, 255), q4k.Q4K_ERR_SHAPE),
    ((A16, A16 * 2, A16 * 3, 1, 4, 0), q4k.Q4K_ERR_SHAPE),
    ((A16, A16 * 2, A16 * 3, 1, 0, 256), q4k.Q4K_ERR_SHAPE),
    ((A16, A16 * 2, A16 * 3, 1, -3, 256), q4k.Q4K_ERR_SHAPE),
    ((A16, A16 * 2, A16 * 3, 0, 4, 256), q4k.Q4K_ERR_UNSUPPORTED_M),
    ((A16, A16 * 2, A16 * 3, 9, 4, 256), q4k.Q4K_ERR_UNSUPPORTED_M),
    ((A16 + 8, A16 * 2, A16 * 3, 1, 4, 256), q4k.Q4K_ERR_ALIGN),
    ((A16, A16 * 2 + 4, A16 * 3, 1, 4, 256), q4k.Q4K_ERR_ALIGN),
    ((A16, A16 * 2, A16 * 3 + 2, 1, 4, 256), q4k.Q4K_ERR_ALIGN),
    ((A16, A16 * 2, A16 + 16, 1, 4, 256), q4k.Q4K_ERR_OVERLAP),      # y inside w
    ((A16, A16 * 2, A16 * 2 + 512, 1, 4, 256), q4k.Q4K_ERR_OVERLAP),  # y inside x
])
def test_gemv_validation_before_any_cuda_call(args, expect):
    assert q4k.q4k_gemv_status(*args, stream=0) == expect


@pytest.mark.parametrize("args,expect", [
    ((0, A16, 4, 256), q4k.Q4K_ERR_NULL),
    ((A16, 0, 4, 256), q4k.Q4K_ERR_NULL),
    ((A16, A16 * 2, 4, 100), q4k.Q4K_ERR_SHAPE),
    ((A16, A16 * 2, 0, 256), q4k.Q4K_ERR_SHAPE),
    ((A16 + 4, A16 * 2, 4, 256), q4k.Q4K_ERR_ALIGN),
    ((A16, A16 * 2 + 4, 4, 256), q4k.Q4K_ERR_ALIGN),
    ((A16, A16 + 64, 4, 256), q4k.Q4K_ERR_OVERLAP),
])
def test_dequant_validation_before_any_cuda_call(args, expect):
    assert q4k.q4k_dequant_f32_status(*args, stream=0) == expect


def test_gemv_raises_q4kerror():
    with pytest.raises(q4k.Q4KError) as e:
        q4k.q4k_gemv(A16, A16 * 2, A16 * 3, 1, 4, 100, stream=0)
    assert e.value.status == q4k.Q4K_ERR_SHAPE
