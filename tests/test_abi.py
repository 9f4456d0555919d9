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
    for st in range(8):
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
    ((A16, A16 * 2, A16 * 3, 65, 4, 256), q4k.Q4K_ERR_UNSUPPORTED_M),
    ((A16 + 8, A16 * 2, A16 * 3, 1, 4, 256), q4k.Q4K_ERR_ALIGN),
    ((A16, A16 * 2 + 4, A16 * 3, 1, 4, 256), q4k.Q4K_ERR_ALIGN),
    ((A16, A16 * 2, A16 * 3 + 2, 1, 4, 256), q4k.Q4K_ERR_ALIGN),
    ((A16, A16 * 2, A16 + 16, 1, 4, 256), q4k.Q4K_ERR_OVERLAP),      # y inside w
    ((A16, A16 * 2, A16 * 2 + 512, 1, 4, 256), q4k.Q4K_ERR_OVERLAP),  # y inside x
])
def test_gemv_validation_before_any_cuda_call(args, expect):
    assert q4k.q4k_gemv_status(*args, stream=0) == expect
    # q4k_gemv_ex with the x-ready flag validates the same way
    assert q4k.q4k_gemv_status(*args, stream=0, flags=q4k.Q4K_GEMV_X_READY) == expect


@pytest.mark.parametrize("flags", [0x2, 0x80000000, 0xFFFFFFFF])
def test_gemv_ex_rejects_unknown_flags(flags):
    """Bits other than Q4K_GEMV_X_READY are refused before any CUDA call."""
    assert q4k.q4k_gemv_status(A16, A16 * 2, A16 * 3, 1, 4, 256, stream=0, flags=flags) == q4k.Q4K_ERR_SHAPE


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


# Embedding validation: every call below is refused before any CUDA call.
GOLDEN_EMBED = os.path.join(ROOT, "tests", "golden", "embed_validation_cases.txt")


def embed_page_cases():
    cases = []
    with open(GOLDEN_EMBED) as f:
        for line in f:
            if line.startswith("#") or not line.strip():
                continue
            *nums, expect = line.split()
            cases.append(([int(v) for v in nums], expect))
    return cases


def test_embed_page_cases_refused_like_the_oracle():
    """The page's validation test: the failing cases are refused by the C ABI
    with the status the oracle's verdict maps to (token -> Q4K_ERR_RANGE, the
    other rules -> Q4K_ERR_SHAPE); the passing case passes validation (it is then
    refused for its NULL output, before any CUDA call)."""
    import oracle
    cases = embed_page_cases()
    assert len(cases) == 4
    for (table_bytes, rows, cols, hidden, token), expect in cases:
        verdict = oracle.embed_validate(table_bytes, rows, cols, hidden, token)
        st = capi.q4k_embed_lookup_f32_status(A16, rows, cols, hidden, token, 1.0, None,
                                              stream=0, table_bytes=table_bytes)
        if expect == "ok":
            assert verdict == oracle.EMBED_OK and st == q4k.Q4K_ERR_NULL
        else:
            want = q4k.Q4K_ERR_RANGE if verdict == oracle.EMBED_TOKEN else q4k.Q4K_ERR_SHAPE
            assert verdict != oracle.EMBED_OK and st == want, (table_bytes, rows, cols, token)


@pytest.mark.parametrize("table_bytes,rows,cols,hidden,token,expect", [
    (10 * 144, 10, 512, 256, 9, q4k.Q4K_ERR_SHAPE),      # cols != hidden
    (10 * 144, 10, 256, 256, 10, q4k.Q4K_ERR_RANGE),     # token == rows
    (0, 0, 256, 256, 0, q4k.Q4K_ERR_RANGE),              # empty table
    (10 * 144, 10, 300, 300, 0, q4k.Q4K_ERR_SHAPE),      # not whole blocks
    (0, 10, 0, 0, 0, q4k.Q4K_ERR_SHAPE),                 # zero width
    (10 * 144 + 1, 10, 256, 256, 0, q4k.Q4K_ERR_SHAPE),  # one byte too many
    (10 * 144 - 1, 10, 256, 256, 0, q4k.Q4K_ERR_SHAPE),  # one byte short
    (0, 1, 512, 256, 5, q4k.Q4K_ERR_SHAPE),              # shape before token
    (0, 1, 300, 300, 5, q4k.Q4K_ERR_RANGE),              # token before width
])
def test_embed_lookup_rules(table_bytes, rows, cols, hidden, token, expect):
    import oracle
    verdict = oracle.embed_validate(table_bytes, rows, cols, hidden, token)
    assert (verdict == oracle.EMBED_TOKEN) == (expect == q4k.Q4K_ERR_RANGE)
    assert verdict != oracle.EMBED_OK
    st = capi.q4k_embed_lookup_f32_status(A16, rows, cols, hidden, token, 1.0, A16 * 4,
                                          stream=0, table_bytes=table_bytes)
    assert st == expect


def test_embed_lookup_pointer_checks():
    ok = dict(rows=10, cols=256, hidden=256, token=3, embed_scale=1.0, stream=0,
              table_bytes=10 * 144)
    assert capi.q4k_embed_lookup_f32_status(0, out=A16 * 4, **ok) == q4k.Q4K_ERR_NULL
    assert capi.q4k_embed_lookup_f32_status(A16, out=0, **ok) == q4k.Q4K_ERR_NULL
    assert capi.q4k_embed_lookup_f32_status(A16 + 8, out=A16 * 4, **ok) == q4k.Q4K_ERR_ALIGN
    assert capi.q4k_embed_lookup_f32_status(A16, out=A16 * 4 + 4, **ok) == q4k.Q4K_ERR_ALIGN
    assert capi.q4k_embed_lookup_f32_status(A16, out=A16 + 16, **ok) == q4k.Q4K_ERR_OVERLAP


@pytest.mark.parametrize("kw,expect", [
    (dict(table=0), q4k.Q4K_ERR_NULL),
    (dict(tokens=0), q4k.Q4K_ERR_NULL),
    (dict(out=0), q4k.Q4K_ERR_NULL),
    (dict(rows=0, table_bytes=0), q4k.Q4K_ERR_SHAPE),
    (dict(hidden=300), q4k.Q4K_ERR_SHAPE),
    (dict(hidden=0), q4k.Q4K_ERR_SHAPE),
    (dict(n_tokens=-1), q4k.Q4K_ERR_SHAPE),
    (dict(table_bytes=10 * 144 - 144), q4k.Q4K_ERR_SHAPE),
    (dict(tokens=A16 * 2 + 2), q4k.Q4K_ERR_ALIGN),
    (dict(out=A16 * 4 + 8), q4k.Q4K_ERR_ALIGN),
    (dict(out=A16), q4k.Q4K_ERR_OVERLAP),
    (dict(tokens=A16 * 4 + 16), q4k.Q4K_ERR_OVERLAP),
    (dict(n_tokens=0), q4k.Q4K_OK),                        # nothing to do: no launch
])
def test_embed_gather_checks(kw, expect):
    args = dict(table=A16, rows=10, hidden=256, tokens=A16 * 2, n_tokens=4, embed_scale=1.0,
                out=A16 * 4, stream=0, table_bytes=10 * 144)
    args.update(kw)
    assert capi.q4k_embed_gather_f32_status(**args) == expect


def test_binding_refuses_wrong_element_types():
    """The library reads raw bytes; the binding refuses tensors of another
    element type before any call (CPU tensors here, never dereferenced)."""
    torch = pytest.importorskip("torch")
    half = torch.zeros(256, dtype=torch.float16)
    f32 = torch.zeros(256, dtype=torch.float32)
    with pytest.raises(TypeError):
        capi.q4k_gemv_status(A16, half, f32, 1, 1, 256, stream=0)
    with pytest.raises(TypeError):
        capi.q4k_gemv_status(A16, A16 * 2, half, 1, 1, 256, stream=0)
    with pytest.raises(TypeError):
        capi.q4k_dequant_f32_status(A16, half, 1, 256, stream=0)
    with pytest.raises(TypeError):
        capi.q4k_embed_gather_f32_status(A16, 10, 256, torch.zeros(4, dtype=torch.int64), 4,
                                         1.0, A16 * 4, stream=0, table_bytes=10 * 144)
    with pytest.raises(ValueError):
        capi.q4k_embed_lookup_f32_status(A16, 10, 256, 256, 0, 1.0, A16 * 4, stream=0)


def test_binding_refuses_host_tensors():
    """A CPU tensor would reach the kernel as a host pointer: refused before the
    call (never dereferenced here)."""
    torch = pytest.importorskip("torch")
    f32 = torch.zeros(256, dtype=torch.float32)
    w = torch.zeros(144, dtype=torch.uint8)
    with pytest.raises(ValueError):
        capi.q4k_gemv_status(A16, f32, A16 * 2, 1, 1, 256, stream=0)
    with pytest.raises(ValueError):
        capi.q4k_gemv_status(w, A16, A16 * 2, 1, 1, 256, stream=0)
    with pytest.raises(ValueError):
        capi.q4k_dequant_f32_status(A16, f32, 1, 256, stream=0)
    with pytest.raises(ValueError):
        capi.q4k_gemv_swiglu_status(A16, w, A16 * 2, A16 * 4, 1, 1, 256, stream=0)


@pytest.mark.parametrize("args,expect", [
    ((0, A16, A16 * 2, 4, 8, 64), q4k.Q4K_ERR_NULL),
    ((A16, 0, A16 * 2, 4, 8, 64), q4k.Q4K_ERR_NULL),
    ((A16, A16 * 2, 0, 4, 8, 64), q4k.Q4K_ERR_NULL),
    ((A16, A16 * 2, A16 * 3, 0, 8, 64), q4k.Q4K_ERR_SHAPE),
    ((A16, A16 * 2, A16 * 3, 4, 0, 64), q4k.Q4K_ERR_SHAPE),
    ((A16, A16 * 2, A16 * 3, 4, 8, 32), q4k.Q4K_ERR_SHAPE),
    ((A16, A16 * 2, A16 * 3, 4, 8, 0), q4k.Q4K_ERR_SHAPE),
    ((A16 + 8, A16 * 2, A16 * 3, 4, 8, 64), q4k.Q4K_ERR_ALIGN),
    ((A16, A16 * 2 + 8, A16 * 3, 4, 8, 64), q4k.Q4K_ERR_ALIGN),
    ((A16, A16 * 2, A16 * 3 + 2, 4, 8, 64), q4k.Q4K_ERR_ALIGN),
    ((A16, A16 * 2, A16 + 64, 4, 8, 64), q4k.Q4K_ERR_OVERLAP),        # y inside w16
    ((A16, A16 * 2, A16 * 2 + 64, 4, 8, 64), q4k.Q4K_ERR_OVERLAP),    # y inside x16
])
def test_gemm_f16_validation(args, expect):
    assert q4k.q4k_gemm_f16_status(*args, stream=0) == expect


def test_prefill_and_convert_validation():
    # scratch overlapping x, w16 or y; x misaligned; null x
    assert q4k.q4k_prefill_f16_status(A16, A16 * 2, A16 * 2 + 16, A16 * 4, 4, 8, 64,
                                      stream=0) == q4k.Q4K_ERR_OVERLAP
    assert q4k.q4k_prefill_f16_status(A16, A16 * 2, A16 + 16, A16 * 4, 4, 8, 64,
                                      stream=0) == q4k.Q4K_ERR_OVERLAP
    assert q4k.q4k_prefill_f16_status(A16, A16 * 2 + 4, A16 * 3, A16 * 4, 4, 8, 64,
                                      stream=0) == q4k.Q4K_ERR_ALIGN
    assert q4k.q4k_prefill_f16_status(A16, 0, A16 * 3, A16 * 4, 4, 8, 64,
                                      stream=0) == q4k.Q4K_ERR_NULL
    assert q4k.q4k_prefill_f16_status(A16, A16 * 2, A16 * 3, A16 * 4, 4, 8, 100,
                                      stream=0) == q4k.Q4K_ERR_SHAPE
    assert q4k.q4k_f32_to_f16_status(A16, A16 + 8, 16, stream=0) == q4k.Q4K_ERR_ALIGN
    assert q4k.q4k_f32_to_f16_status(A16, A16 + 16, 16, stream=0) == q4k.Q4K_ERR_OVERLAP
    assert q4k.q4k_f32_to_f16_status(0, A16, 16, stream=0) == q4k.Q4K_ERR_NULL
    assert q4k.q4k_dequant_f16_status(A16, A16 * 2, 4, 255, stream=0) == q4k.Q4K_ERR_SHAPE
    assert q4k.q4k_dequant_f16_status(A16, A16 + 16, 4, 256, stream=0) == q4k.Q4K_ERR_OVERLAP
    assert q4k.q4k_dequant_f16_status(A16, A16 * 2 + 8, 4, 256, stream=0) == q4k.Q4K_ERR_ALIGN
