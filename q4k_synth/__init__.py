"""Seeded synthetic inputs for Q4_K GEMV / dequant: the one module that both the
CPU oracle's tests and the CUDA path's tests and benchmark draw their inputs from.

It holds none of the method's arithmetic: it never decodes a superblock, never
dequantises and never forms a dot product. It only lays random numbers into the
byte positions of the Q4_K superblock, so that the oracle and the GPU see the
same bytes.

Superblock byte positions used here (GGUF Q4_K, 144 bytes per 256 weights; the
144-byte size is the one the "memra-engine 0.83.1, src/f16_ffi.rs" page checks in
`build_q8_f16` and names in the `memra_q4_K_dequant_f16` declaration):

    bytes   0..1    d     (IEEE binary16, little-endian)
    bytes   2..3    dmin  (IEEE binary16, little-endian)
    bytes   4..15   12 bytes of packed 6-bit sub-block scales and mins
    bytes  16..143  128 bytes of 4-bit quants

Value distributions (the synthetic workload of the decode shapes):
  * d, dmin: a float64 drawn from U[1e-3, 2e-2], rounded to binary16 by
    round-to-nearest-even (numpy's float64 -> float16 conversion);
  * the 12 scale bytes and 128 quant bytes: independent uniform bytes 0..255;
  * x: standard normal float64 rounded to float32.

Draw order from one numpy PCG64 stream per seed: all d values, all dmin values,
all scale bytes (superblock-major), all quant bytes (superblock-major), then x
(vector-major).
"""
from __future__ import annotations

import numpy as np

QK_K = 256          # weights per superblock
BLOCK_BYTES = 144   # bytes per superblock

# Byte offsets of the fields inside one superblock (see the module docstring).
OFF_D, OFF_DMIN, OFF_SCALES, OFF_QS = 0, 2, 4, 16

# The shapes of the decode-GEMV sweep (N, K), by model class.
SHAPES_TINY = [(256, 1024)]
SHAPES_1P5B = [(8960, 1536), (1536, 8960), (1536, 1536)]
SHAPES_7B = [(11008, 4096), (4096, 11008), (4096, 4096)]
SHAPES_8B = [(4096, 14336), (128256, 4096)]
SHAPES_MULTIVEC = [(14336, 4096), (4096, 14336)]
# One 8B-class decode layer: q, k, v, o, gate, up, down (N, K).
LAYER_8B = [(4096, 4096), (1024, 4096), (1024, 4096), (4096, 4096),
            (14336, 4096), (14336, 4096), (4096, 14336)]

# Seeds per shape, in the order of the lists above.
SEEDS = {
    (256, 1024): 0,
    (8960, 1536): 1, (1536, 8960): 2, (1536, 1536): 3,
    (11008, 4096): 4, (4096, 11008): 5, (4096, 4096): 6,
    (4096, 14336): 7, (128256, 4096): 8,
}
SEED_MULTIVEC = {(14336, 4096): 9, (4096, 14336): 10}


def layer_seed(layer: int, proj: int) -> int:
    """Seed of projection `proj` (0..6 = q,k,v,o,gate,up,down) of decode layer `layer`."""
    return 1000 + 7 * layer + proj


def weight_bytes(n: int, k: int) -> int:
    if n <= 0 or k <= 0 or k % QK_K:
        raise ValueError(f"bad Q4_K shape n={n} k={k}")
    return n * (k // QK_K) * BLOCK_BYTES


def _rng(seed: int) -> np.random.Generator:
    return np.random.Generator(np.random.PCG64(seed))


def _f16_bits(rng: np.random.Generator, count: int, lo: float, hi: float) -> np.ndarray:
    v = rng.uniform(lo, hi, count)                # float64 sample
    return v.astype(np.float16).view(np.uint16)   # RNE to binary16, as raw bits


def fill_superblocks(rng: np.random.Generator, nsb: int,
                     d_range=(1e-3, 2e-2), dmin_range=(1e-3, 2e-2)) -> np.ndarray:
    """`nsb` random superblocks as a (nsb, 144) uint8 array."""
    out = np.empty((nsb, BLOCK_BYTES), dtype=np.uint8)
    d = _f16_bits(rng, nsb, *d_range)
    dmin = _f16_bits(rng, nsb, *dmin_range)
    out[:, OFF_D:OFF_D + 2] = d.astype('<u2').view(np.uint8).reshape(nsb, 2)
    out[:, OFF_DMIN:OFF_DMIN + 2] = dmin.astype('<u2').view(np.uint8).reshape(nsb, 2)
    out[:, OFF_SCALES:OFF_QS] = rng.integers(0, 256, (nsb, 12), dtype=np.uint8)
    out[:, OFF_QS:] = rng.integers(0, 256, (nsb, 128), dtype=np.uint8)
    return out


def q4k_problem(n: int, k: int, m: int = 1, seed: int = 0):
    """(w, x): w = N*(K/256)*144 uint8 bytes (row-major by output row), x = (m, K) float32."""
    nbytes = weight_bytes(n, k)
    rng = _rng(seed)
    w = fill_superblocks(rng, nbytes // BLOCK_BYTES).reshape(-1)
    x = rng.standard_normal(m * k).astype(np.float32).reshape(m, k)
    return w, x


def x_vectors(k: int, m: int, seed: int) -> np.ndarray:
    """Only activations: (m, K) float32 N(0,1) from their own seeded stream."""
    return _rng(seed).standard_normal(m * k).astype(np.float32).reshape(m, k)


def random_bytes(nbytes: int, seed: int) -> np.ndarray:
    """Uniform raw bytes (every field random, including d and dmin bit patterns)."""
    return _rng(seed).integers(0, 256, nbytes, dtype=np.uint8)
