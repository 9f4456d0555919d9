"""ctypes binding of libq4k_b200.so: the C ABI of include/q4k.h, same names.

Argument marshalling only: torch tensors (or raw integer device addresses) are
turned into pointers and the current torch CUDA stream into a cudaStream_t;
every step of the computation runs in the library's CUDA kernels. There is no
fallback: if the library is missing this module raises on import.
"""
from __future__ import annotations

import ctypes
import os

PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(PKG, "libq4k_b200.so")

Q4K_OK = 0
Q4K_ERR_NULL = 1
Q4K_ERR_SHAPE = 2
Q4K_ERR_ALIGN = 3
Q4K_ERR_UNSUPPORTED_M = 4
Q4K_ERR_CUDA = 5
Q4K_ERR_OVERLAP = 6
Q4K_ERR_RANGE = 7
Q4K_ERR_CAPACITY = 8
Q4K_FAULT_COPY_TIMEOUT = 1
Q4K_FAULT_TOKEN_RANGE = 2
Q4K_QK = 256
Q4K_BLOCK_BYTES = 144
Q4K_MAX_M = 64
Q4K_GEMV_X_READY = 0x1   # q4k_gemv_ex flag: x not written by the pending work on the stream
Q4K_GEMM_K_MULTIPLE = 64
Q4K_PREFILL_NOALLOC_MAX_ELEMS = 8388608
Q4K_KERNEL_WARP_ROWS = 1
Q4K_KERNEL_STREAM = 2
Q4K_KERNEL_TC = 3
Q4K_KERNEL_I8 = 4

# Every function include/q4k.h declares.
EXPORTS = ("q4k_gemv", "q4k_gemv_ex", "q4k_dequant_f32", "q4k_weight_bytes", "q4k_status_string",
           "q4k_last_cuda_error", "q4k_gemv_plan_for", "q4k_device_fault_flags",
           "q4k_embed_lookup_f32", "q4k_embed_gather_f32", "q4k_gemv_swiglu",
           "q4k_gemv_swiglu_plan_for", "q4k_selftest_wait_timeout", "q4k_dequant_f16",
           "q4k_f32_to_f16", "q4k_gemm_f16", "q4k_prefill_f16", "q4k_prefill_f16_noalloc")


class Q4KError(RuntimeError):
    def __init__(self, status: int, what: str):
        self.status = status
        msg = f"{what}: {q4k_status_string(status)} (status {status})"
        if status == Q4K_ERR_CUDA:
            msg += f", cudaError {q4k_last_cuda_error()}"
        super().__init__(msg)


class q4k_gemv_plan(ctypes.Structure):
    _fields_ = [("kernel", ctypes.c_int), ("grid", ctypes.c_int), ("block", ctypes.c_int),
                ("smem_bytes", ctypes.c_int), ("cluster", ctypes.c_int), ("teams", ctypes.c_int),
                ("depth", ctypes.c_int),
                ("launches", ctypes.c_int), ("units", ctypes.c_longlong),
                ("units_per_cta_max", ctypes.c_longlong), ("slices", ctypes.c_int)]

    def as_dict(self) -> dict:
        return {name: getattr(self, name) for name, _ in self._fields_}


if not os.path.exists(LIB_PATH):
    raise ImportError(f"{LIB_PATH} is not built; run `python gguf_quant_dequant_q4k_b200/build.py` "
                      "(or __graft_entry__.build()). There is no CPU fallback.")

_lib = ctypes.CDLL(LIB_PATH)
_vp = ctypes.c_void_p
_lib.q4k_gemv.argtypes = [_vp, _vp, _vp, ctypes.c_int, ctypes.c_int, ctypes.c_int, _vp]
_lib.q4k_gemv.restype = ctypes.c_int
_lib.q4k_gemv_ex.argtypes = [_vp, _vp, _vp, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_uint, _vp]
_lib.q4k_gemv_ex.restype = ctypes.c_int
_lib.q4k_dequant_f32.argtypes = [_vp, _vp, ctypes.c_int, ctypes.c_int, _vp]
_lib.q4k_dequant_f32.restype = ctypes.c_int
_lib.q4k_weight_bytes.argtypes = [ctypes.c_int, ctypes.c_int]
_lib.q4k_weight_bytes.restype = ctypes.c_size_t
_lib.q4k_status_string.argtypes = [ctypes.c_int]
_lib.q4k_status_string.restype = ctypes.c_char_p
_lib.q4k_last_cuda_error.argtypes = []
_lib.q4k_last_cuda_error.restype = ctypes.c_int
_lib.q4k_gemv_plan_for.argtypes = [ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                   ctypes.POINTER(q4k_gemv_plan)]
_lib.q4k_gemv_plan_for.restype = ctypes.c_int
_lib.q4k_device_fault_flags.argtypes = [ctypes.POINTER(ctypes.c_uint)]
_lib.q4k_device_fault_flags.restype = ctypes.c_int
_lib.q4k_gemv_swiglu.argtypes = [_vp, _vp, _vp, _vp, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                 _vp]
_lib.q4k_gemv_swiglu.restype = ctypes.c_int
_lib.q4k_gemv_swiglu_plan_for.argtypes = [ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                          ctypes.POINTER(q4k_gemv_plan)]
_lib.q4k_gemv_swiglu_plan_for.restype = ctypes.c_int
_lib.q4k_selftest_wait_timeout.argtypes = [_vp]
_lib.q4k_selftest_wait_timeout.restype = ctypes.c_int
_lib.q4k_embed_lookup_f32.argtypes = [_vp, ctypes.c_ulonglong, ctypes.c_int, ctypes.c_int,
                                      ctypes.c_int, ctypes.c_uint, ctypes.c_float, _vp, _vp]
_lib.q4k_embed_lookup_f32.restype = ctypes.c_int
_lib.q4k_embed_gather_f32.argtypes = [_vp, ctypes.c_ulonglong, ctypes.c_int, ctypes.c_int, _vp,
                                      ctypes.c_int, ctypes.c_float, _vp, _vp]
_lib.q4k_embed_gather_f32.restype = ctypes.c_int


_lib.q4k_dequant_f16.argtypes = [_vp, _vp, ctypes.c_int, ctypes.c_int, _vp]
_lib.q4k_dequant_f16.restype = ctypes.c_int
_lib.q4k_f32_to_f16.argtypes = [_vp, _vp, ctypes.c_ulonglong, _vp]
_lib.q4k_f32_to_f16.restype = ctypes.c_int
_lib.q4k_gemm_f16.argtypes = [_vp, _vp, _vp, ctypes.c_int, ctypes.c_int, ctypes.c_int, _vp]
_lib.q4k_gemm_f16.restype = ctypes.c_int
_lib.q4k_prefill_f16.argtypes = [_vp, _vp, _vp, _vp, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                 _vp]
_lib.q4k_prefill_f16.restype = ctypes.c_int
_lib.q4k_prefill_f16_noalloc.argtypes = [_vp, _vp, _vp, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                         _vp]
_lib.q4k_prefill_f16_noalloc.restype = ctypes.c_int


def library() -> ctypes.CDLL:
    return _lib


def _ptr(t, dtype: str | None = None, name: str = "", min_bytes: int = 0) -> int | None:
    """Device address of a tensor (or a raw integer address, passed through
    unchecked: the caller vouches for it).

    A tensor must be a contiguous CUDA tensor on the current CUDA device (the
    library launches there and cannot tell a host or foreign pointer from a
    raw address) holding at least `min_bytes` bytes; with `dtype` ("float32",
    "int32", "uint8") its element type must match, since the library reads raw
    bytes. Anything else raises before the C call."""
    if t is None:
        return None
    if isinstance(t, int):
        return t
    if dtype is not None and str(t.dtype).replace("torch.", "") != dtype:
        raise TypeError(f"{name} must be a {dtype} tensor, got {t.dtype}")
    if not t.is_cuda:
        raise ValueError(f"{name or 'tensor'} must be a CUDA tensor, got device {t.device}")
    import torch
    if t.device.index != torch.cuda.current_device():
        raise ValueError(f"{name or 'tensor'} is on {t.device}, but the current CUDA device is "
                         f"cuda:{torch.cuda.current_device()}")
    if not t.is_contiguous():
        raise ValueError(f"{name or 'tensor'} must be contiguous")
    have = t.numel() * t.element_size()
    if have < min_bytes:
        raise ValueError(f"{name or 'tensor'} holds {have} bytes, the call needs {min_bytes}")
    return t.data_ptr()


def _need(count: int, item: int, valid: bool) -> int:
    """Bytes a buffer must hold, or 0 where the C library will refuse the
    call's sizes anyway (its status is then the answer)."""
    return count * item if valid and count > 0 else 0


def _gemv_sizes_valid(m: int, n: int, k: int) -> bool:
    return 1 <= m <= Q4K_MAX_M and q4k_weight_bytes(n, k) > 0


def _stream(stream) -> int | None:
    if stream is None:
        import torch
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


def q4k_weight_bytes(n: int, k: int) -> int:
    return _lib.q4k_weight_bytes(int(n), int(k))


def q4k_status_string(status: int) -> str:
    return _lib.q4k_status_string(int(status)).decode()


def q4k_last_cuda_error() -> int:
    return _lib.q4k_last_cuda_error()


def q4k_gemv_plan_for(m: int, n: int, k: int, num_sms: int) -> dict:
    plan = q4k_gemv_plan()
    st = _lib.q4k_gemv_plan_for(int(m), int(n), int(k), int(num_sms), ctypes.byref(plan))
    if st != Q4K_OK:
        raise Q4KError(st, "q4k_gemv_plan_for")
    return plan.as_dict()


def q4k_gemv_swiglu_plan_for(m: int, n: int, k: int, num_sms: int) -> dict:
    plan = q4k_gemv_plan()
    st = _lib.q4k_gemv_swiglu_plan_for(int(m), int(n), int(k), int(num_sms), ctypes.byref(plan))
    if st != Q4K_OK:
        raise Q4KError(st, "q4k_gemv_swiglu_plan_for")
    return plan.as_dict()


def q4k_selftest_wait_timeout(stream=None) -> None:
    """Enqueues the bounded-wait self-test kernel (raises Q4K_FAULT_COPY_TIMEOUT)."""
    st = _lib.q4k_selftest_wait_timeout(_stream(stream))
    if st != Q4K_OK:
        raise Q4KError(st, "q4k_selftest_wait_timeout")


def q4k_device_fault_flags() -> int:
    """Reads and clears the current device's kernel fault flags (synchronises)."""
    v = ctypes.c_uint(0)
    st = _lib.q4k_device_fault_flags(ctypes.byref(v))
    if st != Q4K_OK:
        raise Q4KError(st, "q4k_device_fault_flags")
    return v.value


def q4k_gemv_status(w, x, y, m: int, n: int, k: int, stream=None, flags: int = 0) -> int:
    """Raw status of the C call (no exception; tensor checks still raise)."""
    ok = _gemv_sizes_valid(m, n, k)
    args = (_ptr(w, None, "w", _need(q4k_weight_bytes(n, k), 1, ok)),
            _ptr(x, "float32", "x", _need(m * k, 4, ok)),
            _ptr(y, "float32", "y", _need(m * n, 4, ok)), int(m), int(n), int(k))
    if flags == 0:
        return _lib.q4k_gemv(*args, _stream(stream))
    return _lib.q4k_gemv_ex(*args, int(flags), _stream(stream))


def q4k_gemv(w, x, y, m: int, n: int, k: int, stream=None, x_ready: bool = False) -> None:
    """y[m, n] = W[n, k] x[m, k] on `stream` (default: torch's current stream).
    x_ready: x is not written by the work still pending on `stream`
    (Q4K_GEMV_X_READY: it may be read before that work finishes)."""
    st = q4k_gemv_status(w, x, y, m, n, k, stream, Q4K_GEMV_X_READY if x_ready else 0)
    if st != Q4K_OK:
        raise Q4KError(st, "q4k_gemv")


def q4k_gemv_swiglu_status(w_gate, w_up, x, y, m: int, n: int, k: int, stream=None) -> int:
    ok = _gemv_sizes_valid(m, n, k)
    wb = _need(q4k_weight_bytes(n, k), 1, ok)
    return _lib.q4k_gemv_swiglu(_ptr(w_gate, None, "w_gate", wb), _ptr(w_up, None, "w_up", wb),
                                _ptr(x, "float32", "x", _need(m * k, 4, ok)),
                                _ptr(y, "float32", "y", _need(m * n, 4, ok)), int(m), int(n),
                                int(k), _stream(stream))


def q4k_gemv_swiglu(w_gate, w_up, x, y, m: int, n: int, k: int, stream=None) -> None:
    """y[m, n] = silu(W_gate x) * (W_up x) on `stream` (default: torch's current stream)."""
    st = q4k_gemv_swiglu_status(w_gate, w_up, x, y, m, n, k, stream)
    if st != Q4K_OK:
        raise Q4KError(st, "q4k_gemv_swiglu")


def q4k_dequant_f32_status(w, out, n: int, k: int, stream=None) -> int:
    ok = q4k_weight_bytes(n, k) > 0
    return _lib.q4k_dequant_f32(_ptr(w, None, "w", _need(q4k_weight_bytes(n, k), 1, ok)),
                                _ptr(out, "float32", "out", _need(n * k, 4, ok)), int(n), int(k),
                                _stream(stream))


def q4k_dequant_f32(w, out, n: int, k: int, stream=None) -> None:
    """out[n, k] = dequantised W (f32) on `stream` (default: torch's current stream)."""
    st = q4k_dequant_f32_status(w, out, n, k, stream)
    if st != Q4K_OK:
        raise Q4KError(st, "q4k_dequant_f32")


def _nbytes(t, given) -> int:
    if given is not None:
        return int(given)
    if t is None or isinstance(t, int):
        raise ValueError("table_bytes is required with a raw address")
    return t.numel() * t.element_size()


def q4k_embed_lookup_f32_status(table, rows: int, cols: int, hidden: int, token: int,
                                embed_scale: float, out, stream=None,
                                table_bytes: int | None = None) -> int:
    """Raw status of the C call (no exception). table_bytes defaults to the
    tensor's size; pass it explicitly with a raw pointer."""
    ok = hidden > 0 and hidden % Q4K_QK == 0
    return _lib.q4k_embed_lookup_f32(_ptr(table, None, "table"), _nbytes(table, table_bytes),
                                     int(rows), int(cols), int(hidden), int(token) & 0xFFFFFFFF,
                                     float(embed_scale),
                                     _ptr(out, "float32", "out", _need(hidden, 4, ok)),
                                     _stream(stream))


def q4k_embed_lookup_f32(table, rows: int, cols: int, hidden: int, token: int,
                         embed_scale: float, out, stream=None,
                         table_bytes: int | None = None) -> None:
    """out[hidden] = row `token` of the Q4_K table [rows, cols], dequantised, x embed_scale."""
    st = q4k_embed_lookup_f32_status(table, rows, cols, hidden, token, embed_scale, out, stream,
                                     table_bytes)
    if st != Q4K_OK:
        raise Q4KError(st, "q4k_embed_lookup_f32")


def q4k_embed_gather_f32_status(table, rows: int, hidden: int, tokens, n_tokens: int,
                                embed_scale: float, out, stream=None,
                                table_bytes: int | None = None) -> int:
    ok = hidden > 0 and hidden % Q4K_QK == 0 and n_tokens > 0
    return _lib.q4k_embed_gather_f32(_ptr(table, None, "table"), _nbytes(table, table_bytes),
                                     int(rows), int(hidden),
                                     _ptr(tokens, "int32", "tokens", _need(n_tokens, 4, ok)),
                                     int(n_tokens), float(embed_scale),
                                     _ptr(out, "float32", "out", _need(n_tokens * hidden, 4, ok)),
                                     _stream(stream))


def q4k_embed_gather_f32(table, rows: int, hidden: int, tokens, n_tokens: int,
                         embed_scale: float, out, stream=None,
                         table_bytes: int | None = None) -> None:
    """out[n_tokens, hidden] = rows tokens[i] (int32, device) of the table, x embed_scale.
    A token outside the table gives a zero row and raises Q4K_FAULT_TOKEN_RANGE."""
    st = q4k_embed_gather_f32_status(table, rows, hidden, tokens, n_tokens, embed_scale, out,
                                     stream, table_bytes)
    if st != Q4K_OK:
        raise Q4KError(st, "q4k_embed_gather_f32")


# --------------------------------------------------------------------------- prefill (fp16)

def _gemm_sizes_valid(m: int, n: int, k: int) -> bool:
    return m > 0 and n > 0 and k > 0 and k % Q4K_GEMM_K_MULTIPLE == 0


def q4k_dequant_f16_status(w, out, n: int, k: int, stream=None) -> int:
    ok = q4k_weight_bytes(n, k) > 0
    return _lib.q4k_dequant_f16(_ptr(w, None, "w", _need(q4k_weight_bytes(n, k), 1, ok)),
                                _ptr(out, "float16", "out", _need(n * k, 2, ok)), int(n), int(k),
                                _stream(stream))


def q4k_dequant_f16(w, out, n: int, k: int, stream=None) -> None:
    """out[n, k] (float16) = the fp16 mirror of the Q4_K matrix W."""
    st = q4k_dequant_f16_status(w, out, n, k, stream)
    if st != Q4K_OK:
        raise Q4KError(st, "q4k_dequant_f16")


def q4k_f32_to_f16_status(x, out, count: int, stream=None) -> int:
    ok = count > 0
    return _lib.q4k_f32_to_f16(_ptr(x, "float32", "x", _need(count, 4, ok)),
                               _ptr(out, "float16", "out", _need(count, 2, ok)), int(count),
                               _stream(stream))


def q4k_f32_to_f16(x, out, count: int, stream=None) -> None:
    """out[:count] (float16) = RNE binary16 of x[:count] (float32)."""
    st = q4k_f32_to_f16_status(x, out, count, stream)
    if st != Q4K_OK:
        raise Q4KError(st, "q4k_f32_to_f16")


def q4k_gemm_f16_status(w16, x16, y, m: int, n: int, k: int, stream=None) -> int:
    ok = _gemm_sizes_valid(m, n, k)
    return _lib.q4k_gemm_f16(_ptr(w16, "float16", "w_f16", _need(n * k, 2, ok)),
                             _ptr(x16, "float16", "x_f16", _need(m * k, 2, ok)),
                             _ptr(y, "float32", "y", _need(m * n, 4, ok)), int(m), int(n), int(k),
                             _stream(stream))


def q4k_gemm_f16(w16, x16, y, m: int, n: int, k: int, stream=None) -> None:
    """y[m, n] = x16[m, k] @ w16[n, k]^T (fp16 operands, f32 accumulation and output)."""
    st = q4k_gemm_f16_status(w16, x16, y, m, n, k, stream)
    if st != Q4K_OK:
        raise Q4KError(st, "q4k_gemm_f16")


def q4k_prefill_f16_status(w16, x, scratch, y, m: int, n: int, k: int, stream=None) -> int:
    ok = _gemm_sizes_valid(m, n, k)
    return _lib.q4k_prefill_f16(_ptr(w16, "float16", "w_f16", _need(n * k, 2, ok)),
                                _ptr(x, "float32", "x", _need(m * k, 4, ok)),
                                _ptr(scratch, None, "x_f16_scratch", _need(m * k, 2, ok)),
                                _ptr(y, "float32", "y", _need(m * n, 4, ok)), int(m), int(n),
                                int(k), _stream(stream))


def q4k_prefill_f16(w16, x, scratch, y, m: int, n: int, k: int, stream=None) -> None:
    """y[m, n] = fp16(x[m, k]) @ w16[n, k]^T; `scratch` (m*k*2 bytes) receives fp16(x)."""
    st = q4k_prefill_f16_status(w16, x, scratch, y, m, n, k, stream)
    if st != Q4K_OK:
        raise Q4KError(st, "q4k_prefill_f16")


def q4k_prefill_f16_noalloc_status(w16, x, y, m: int, n: int, k: int, stream=None) -> int:
    """Raw status of the C call (no exception; tensor checks still raise)."""
    ok = _gemm_sizes_valid(m, n, k) and m * k <= Q4K_PREFILL_NOALLOC_MAX_ELEMS
    return _lib.q4k_prefill_f16_noalloc(_ptr(w16, "float16", "w_f16", _need(n * k, 2, ok)),
                                        _ptr(x, "float32", "x", _need(m * k, 4, ok)),
                                        _ptr(y, "float32", "y", _need(m * n, 4, ok)), int(m),
                                        int(n), int(k), _stream(stream))


def q4k_prefill_f16_noalloc(w16, x, y, m: int, n: int, k: int, stream=None) -> None:
    """y[m, n] = fp16(x[m, k]) @ w16[n, k]^T using the library's fixed scratch
    (for callers that cannot allocate device memory; m*k <=
    Q4K_PREFILL_NOALLOC_MAX_ELEMS; calls that overlap on the GPU race)."""
    st = q4k_prefill_f16_noalloc_status(w16, x, y, m, n, k, stream)
    if st != Q4K_OK:
        raise Q4KError(st, "q4k_prefill_f16_noalloc")
