"""CPU oracle for GGUF Q4_K dequantisation and Q4_K GEMV (ctypes front end).

TEST INFRASTRUCTURE. Only `tests/`, `__graft_entry__.smoke()` and the
`cpu_baseline` / `--impl reference` legs of `bench.py` may import this package.
The product library (`gguf_quant_dequant_q4k_b200`) never imports, loads or
calls it, and the two share no code.

The arithmetic lives in `q4k_oracle.c` (plain C, built with gcc); this file only
compiles it and marshals numpy arrays. The C file's header states what each
function follows on the pages and the format readings it takes.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(_HERE, "q4k_oracle.c")
LIB = os.path.join(_HERE, "libq4k_oracle.so")

_u8p = ctypes.POINTER(ctypes.c_uint8)
_f32p = ctypes.POINTER(ctypes.c_float)
_f64p = ctypes.POINTER(ctypes.c_double)
_i32p = ctypes.POINTER(ctypes.c_int32)
_i64p = ctypes.POINTER(ctypes.c_int64)
_u16p = ctypes.POINTER(ctypes.c_uint16)

CFLAGS = ["-O2", "-fPIC", "-shared", "-std=c11", "-ffp-contract=off", "-fno-fast-math",
          "-pthread"]


def build(src: str = SRC, out: str = LIB, force: bool = False) -> str:
    """Compile `src` with gcc into the shared library `out` (only if stale)."""
    if (not force and os.path.exists(out)
            and os.path.getmtime(out) >= os.path.getmtime(src)):
        return out
    tmp = out + ".tmp%d" % os.getpid()
    subprocess.run(["gcc", *CFLAGS, src, "-o", tmp, "-lm"], check=True)
    os.replace(tmp, out)
    return out


def _p(arr: np.ndarray, ptype):
    return arr.ctypes.data_as(ptype)


def _check_shape(w: np.ndarray, n: int, k: int) -> None:
    if k <= 0 or k % 256 or n <= 0:
        raise ValueError(f"bad Q4_K shape n={n} k={k}")
    if w.dtype != np.uint8 or not w.flags.c_contiguous or w.size != n * (k // 256) * 144:
        raise ValueError("w must be contiguous uint8 of n*(k/256)*144 bytes")


def _rows(rows, n: int) -> np.ndarray:
    rows = np.ascontiguousarray(rows, dtype=np.int64).reshape(-1)
    if rows.size and (rows.min() < 0 or rows.max() >= n):
        raise ValueError("row index out of range")
    return rows


class Oracle:
    """One loaded copy of the oracle library."""

    def __init__(self, path: str):
        L = ctypes.CDLL(path)
        L.q4k_oracle_half_to_double.argtypes = [ctypes.c_uint16]
        L.q4k_oracle_half_to_double.restype = ctypes.c_double
        L.q4k_oracle_unpack.argtypes = [_u8p, _u16p, _u16p, _i32p, _i32p, _i32p]
        L.q4k_oracle_unpack.restype = None
        L.q4k_oracle_pack.argtypes = [ctypes.c_uint16, ctypes.c_uint16, _i32p, _i32p, _i32p,
                                      _u8p]
        L.q4k_oracle_pack.restype = None
        L.q4k_oracle_dequant_f32.argtypes = [_u8p, ctypes.c_int64, ctypes.c_int64, _f32p]
        L.q4k_oracle_dequant_f32.restype = None
        L.q4k_oracle_dequant_rows.argtypes = [_u8p, ctypes.c_int64, _i64p, ctypes.c_int64,
                                              _f32p]
        L.q4k_oracle_dequant_rows.restype = None
        L.q4k_oracle_gemv.argtypes = [_u8p, _f32p, ctypes.c_int32, ctypes.c_int64,
                                      ctypes.c_int64, _f64p, _f64p, ctypes.c_int32]
        L.q4k_oracle_gemv.restype = ctypes.c_int
        L.q4k_oracle_gemv_rows.argtypes = [_u8p, _f32p, ctypes.c_int32, ctypes.c_int64, _i64p,
                                           ctypes.c_int64, _f64p, _f64p]
        L.q4k_oracle_gemv_rows.restype = None
        L.q4k_oracle_embed_validate.argtypes = [ctypes.c_uint64] * 5
        L.q4k_oracle_embed_validate.restype = ctypes.c_int
        L.q4k_oracle_embed_lookup.argtypes = [_u8p] + [ctypes.c_uint64] * 5 + [ctypes.c_float,
                                                                              _f32p]
        L.q4k_oracle_embed_lookup.restype = ctypes.c_int
        L.q4k_oracle_float_to_half.argtypes = [ctypes.c_float]
        L.q4k_oracle_float_to_half.restype = ctypes.c_uint16
        L.q4k_oracle_floats_to_half.argtypes = [_f32p, ctypes.c_int64, _u16p]
        L.q4k_oracle_floats_to_half.restype = None
        L.q4k_oracle_dequant_f16.argtypes = [_u8p, ctypes.c_int64, ctypes.c_int64, _u16p]
        L.q4k_oracle_dequant_f16.restype = None
        self.L = L
        self.path = path

    def half_to_double(self, bits: int) -> float:
        return self.L.q4k_oracle_half_to_double(int(bits) & 0xFFFF)

    def unpack(self, sb: np.ndarray):
        """One 144-byte superblock -> (d_bits, dmin_bits, sc[8], m[8], q[256])."""
        sb = np.ascontiguousarray(sb, dtype=np.uint8).reshape(-1)
        if sb.size != 144:
            raise ValueError("a superblock is 144 bytes")
        d = ctypes.c_uint16()
        dm = ctypes.c_uint16()
        sc = np.zeros(8, np.int32)
        mn = np.zeros(8, np.int32)
        q = np.zeros(256, np.int32)
        self.L.q4k_oracle_unpack(_p(sb, _u8p), ctypes.byref(d), ctypes.byref(dm),
                                 _p(sc, _i32p), _p(mn, _i32p), _p(q, _i32p))
        return d.value, dm.value, sc, mn, q

    def pack(self, d_bits: int, dmin_bits: int, sc, mn, q) -> np.ndarray:
        """Integer fields -> one 144-byte superblock (the inverse of `unpack`)."""
        sc = np.ascontiguousarray(sc, dtype=np.int32)
        mn = np.ascontiguousarray(mn, dtype=np.int32)
        q = np.ascontiguousarray(q, dtype=np.int32)
        out = np.zeros(144, np.uint8)
        self.L.q4k_oracle_pack(int(d_bits), int(dmin_bits), _p(sc, _i32p), _p(mn, _i32p),
                               _p(q, _i32p), _p(out, _u8p))
        return out

    def dequant_f32(self, w: np.ndarray, n: int, k: int) -> np.ndarray:
        """Dequantised W as an (n, k) float32 array."""
        w = np.ascontiguousarray(w, dtype=np.uint8).reshape(-1)
        _check_shape(w, n, k)
        out = np.empty((n, k), np.float32)
        self.L.q4k_oracle_dequant_f32(_p(w, _u8p), n, k, _p(out, _f32p))
        return out

    def dequant_rows(self, w: np.ndarray, n: int, k: int, rows) -> np.ndarray:
        """Dequantised rows `rows` of W as a (len(rows), k) float32 array."""
        w = np.ascontiguousarray(w, dtype=np.uint8).reshape(-1)
        _check_shape(w, n, k)
        rows = _rows(rows, n)
        out = np.empty((rows.size, k), np.float32)
        self.L.q4k_oracle_dequant_rows(_p(w, _u8p), k, _p(rows, _i64p), rows.size,
                                       _p(out, _f32p))
        return out

    def gemv(self, w: np.ndarray, x: np.ndarray, n: int, k: int, nthreads: int = 1):
        """(y, a): y = W x in double, a = sum |w x| per element; both (m, n) float64."""
        w = np.ascontiguousarray(w, dtype=np.uint8).reshape(-1)
        _check_shape(w, n, k)
        x = np.ascontiguousarray(x, dtype=np.float32).reshape(-1, k)
        m = x.shape[0]
        y = np.empty((m, n), np.float64)
        a = np.empty((m, n), np.float64)
        rc = self.L.q4k_oracle_gemv(_p(w, _u8p), _p(x, _f32p), m, n, k, _p(y, _f64p),
                                    _p(a, _f64p), int(nthreads))
        if rc != 0:
            raise RuntimeError("oracle could not start its threads")
        return y, a

    def gemv_rows(self, w: np.ndarray, x: np.ndarray, n: int, k: int, rows):
        """(y, a) for the listed rows only: both (m, len(rows)) float64."""
        w = np.ascontiguousarray(w, dtype=np.uint8).reshape(-1)
        _check_shape(w, n, k)
        x = np.ascontiguousarray(x, dtype=np.float32).reshape(-1, k)
        rows = _rows(rows, n)
        m = x.shape[0]
        y = np.empty((m, rows.size), np.float64)
        a = np.empty((m, rows.size), np.float64)
        self.L.q4k_oracle_gemv_rows(_p(w, _u8p), _p(x, _f32p), m, k, _p(rows, _i64p),
                                    rows.size, _p(y, _f64p), _p(a, _f64p))
        return y, a

    def floats_to_half(self, x: np.ndarray) -> np.ndarray:
        """binary16 RNE bit patterns (uint16) of float32 values, same shape."""
        x = np.ascontiguousarray(x, dtype=np.float32)
        out = np.empty(x.shape, np.uint16)
        self.L.q4k_oracle_floats_to_half(_p(x.reshape(-1), _f32p), x.size,
                                         _p(out.reshape(-1), _u16p))
        return out

    def dequant_f16(self, w: np.ndarray, n: int, k: int) -> np.ndarray:
        """The fp16 mirror of W: (n, k) uint16 binary16 bit patterns."""
        w = np.ascontiguousarray(w, dtype=np.uint8).reshape(-1)
        _check_shape(w, n, k)
        out = np.empty((n, k), np.uint16)
        self.L.q4k_oracle_dequant_f16(_p(w, _u8p), n, k, _p(out, _u16p))
        return out

    def half_values(self, bits: np.ndarray) -> np.ndarray:
        """float64 values of binary16 bit patterns (through half_to_double)."""
        table = np.array([self.half_to_double(b) for b in range(65536)], np.float64) \
            if not hasattr(self, "_half_table") else self._half_table
        self._half_table = table
        return table[np.asarray(bits, np.uint16).astype(np.int64)]

    def gemm_f16(self, w16: np.ndarray, x16: np.ndarray, rows=None):
        """Prefill GEMM reference on fp16 operands ("memra-engine 0.83.1,
        src/f16_ffi.rs", `memra_f16_pp_gemm_pre`: y = x16 W16^T, fp16 inputs,
        f32 output): y[i][r] = sum_k w16[r][k] * x16[i][k] and a[i][r] =
        sum_k |w16[r][k] * x16[i][k]|, both in float64 from the exact binary16
        values (a double matmul: every product is exact, the sums are
        double-rounded only). w16 (n, k) and x16 (m, k) are uint16 bit
        patterns; `rows` restricts the output columns to those rows of W.
        Returns (y, a), each (m, len(rows) or n) float64."""
        wv = self.half_values(w16 if rows is None else np.asarray(w16)[np.asarray(rows)])
        xv = self.half_values(x16)
        return xv @ wv.T, np.abs(xv) @ np.abs(wv).T

    def embed_validate(self, table_bytes: int, rows: int, cols: int, hidden: int,
                       token: int) -> int:
        """Which of the embedding-table rules fails (EMBED_* codes; EMBED_OK = 0)."""
        return self.L.q4k_oracle_embed_validate(table_bytes, rows, cols, hidden, token)

    def embed_lookup(self, table: np.ndarray, rows: int, cols: int, hidden: int, token: int,
                     embed_scale: float, table_bytes: int | None = None):
        """(status, out): out = row `token` dequantised, times embed_scale (float32,
        `hidden` values), or None when a rule fails."""
        table = np.ascontiguousarray(table, dtype=np.uint8).reshape(-1)
        nbytes = table.size if table_bytes is None else int(table_bytes)
        out = np.zeros(max(int(hidden), 1), np.float32)
        st = self.L.q4k_oracle_embed_lookup(_p(table, _u8p), nbytes, rows, cols, hidden, token,
                                            float(embed_scale), _p(out, _f32p))
        return st, (out[:hidden] if st == EMBED_OK else None)


# q4k_oracle_embed_validate results
EMBED_OK, EMBED_SHAPE, EMBED_TOKEN, EMBED_WIDTH, EMBED_OVERFLOW, EMBED_SIZE = range(6)

_default: Oracle | None = None


def default() -> Oracle:
    """The oracle built from `q4k_oracle.c` in this directory."""
    global _default
    if _default is None:
        _default = Oracle(build())
    return _default


def half_to_double(bits):
    return default().half_to_double(bits)


def unpack(sb):
    return default().unpack(sb)


def pack(d_bits, dmin_bits, sc, mn, q):
    return default().pack(d_bits, dmin_bits, sc, mn, q)


def dequant_f32(w, n, k):
    return default().dequant_f32(w, n, k)


def dequant_rows(w, n, k, rows):
    return default().dequant_rows(w, n, k, rows)


def gemv(w, x, n, k, nthreads=1):
    return default().gemv(w, x, n, k, nthreads)


def gemv_rows(w, x, n, k, rows):
    return default().gemv_rows(w, x, n, k, rows)


def embed_validate(table_bytes, rows, cols, hidden, token):
    return default().embed_validate(table_bytes, rows, cols, hidden, token)


def embed_lookup(table, rows, cols, hidden, token, embed_scale, table_bytes=None):
    return default().embed_lookup(table, rows, cols, hidden, token, embed_scale, table_bytes)


def swiglu_gemv(w_gate, w_up, x, n, k, nthreads=1):
    """Fused gate/up GEMV with SwiGLU ("realizar 0.8.5" kernel cache page,
    `FusedGateUpSwigluHwDp4aQ4KGemv { k: hidden_dim, n: intermediate_dim }`):
    g = W_gate x and u = W_up x by the oracle GEMV (double), then
    out = silu(g) * u = g / (1 + exp(-g)) * u in double.
    Returns (out, g, u, a_g, a_u), all (m, n) float64 (a_*: sums of |w x|)."""
    g, a_g = gemv(w_gate, x, n, k, nthreads)
    u, a_u = gemv(w_up, x, n, k, nthreads)
    with np.errstate(over="ignore"):
        silu = g / (1.0 + np.exp(-g))
    return silu * u, g, u, a_g, a_u


def swiglu_tolerance(g, u, a_g, a_u, out):
    """Per-element bound for a GPU SwiGLU GEMV against `swiglu_gemv`. The GPU's
    g and u each carry the GEMV bound t = 1e-4 * sum|w x| + 1e-6; silu' lies in
    [-0.1, 1.1], so silu(g) moves by at most 1.1 t_g; the f32 epilogue (exp,
    divide, multiply) adds a few ulps of the result:
      1.1 t_g (|u| + t_u) + (|silu(g)| + 1.1 t_g) t_u + 1e-6 |out| + 1e-30."""
    tg = tolerance(a_g)
    tu = tolerance(a_u)
    with np.errstate(over="ignore"):
        silu = np.abs(g / (1.0 + np.exp(-g)))
    return 1.1 * tg * (np.abs(u) + tu) + (silu + 1.1 * tg) * tu + 1e-6 * np.abs(out) + 1e-30


def floats_to_half(x):
    return default().floats_to_half(x)


def dequant_f16(w, n, k):
    return default().dequant_f16(w, n, k)


def half_values(bits):
    return default().half_values(bits)


def gemm_f16(w16, x16, rows=None):
    return default().gemm_f16(w16, x16, rows)


def gemm_f16_tolerance(a: np.ndarray, k: int) -> np.ndarray:
    """Per-element bound for a GPU fp16 GEMM with f32 accumulation against
    `gemm_f16`: the products of two binary16 values are exact in f32 (22
    significant bits), so the only error is the accumulation of k products in
    f32: at most k * u * sum|w x| for recursive summation with unit roundoff u,
    taken here as 2^-23 (twice f32's 2^-24, allowing accumulation by
    truncation rather than rounding), plus 1e-6 for the final store."""
    return k * 2.0 ** -23 * np.asarray(a) + 1e-6


def tolerance(a: np.ndarray) -> np.ndarray:
    """Per-element GEMV bound |y_gpu - y_ref| <= 1e-4 * sum|w x| + 1e-6."""
    return 1e-4 * np.asarray(a) + 1e-6
