"""Pins for the CPU oracle: checks against things other than the oracle itself.

Each `check_*` takes a loaded `oracle.Oracle` and raises AssertionError if the
oracle disagrees with what the format, the mathematics or a library routine
fixes. `test_oracle_pins.py` runs them on the oracle; `test_oracle_mutants.py`
runs them on copies of the oracle with a planted mistake and requires that at
least one check fails for every mistake.

Sources of each expectation:
  * binary16 decoding  -> numpy's float16 (a library routine) over all 65536
    bit patterns, plus hand-derived values;
  * field layout       -> hand-built superblocks whose dequantised values are
    derived by hand below (closed forms), a bit-by-bit map of the 12 scale
    bytes, and a nibble-by-nibble position map;
  * unpack/pack        -> round trips in both directions (bijection of the
    144 bytes with the integer fields);
  * GEMV               -> exact rational arithmetic from the unpacked integer
    fields (brute force), numpy matmul of the dequantised matrix, unit and zero
    vectors, per-vector independence.
The readings the layout checks encode are those stated in the oracle's header
(GGUF block_q4_K): d, dmin, S[12], Q[128]; get_scale_min_k4 packing; byte
Q[32g+l] holds weight 64g+l (low nibble) and 64g+32+l (high nibble).
"""
from __future__ import annotations

import os
from fractions import Fraction

import numpy as np

import q4k_synth

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")

# binary16 bit patterns used below
H_ONE, H_HALF, H_QUARTER, H_EIGHTH = 0x3C00, 0x3800, 0x3400, 0x3000


def _block(d_bits, dmin_bits, S, Q):
    b = np.zeros(144, np.uint8)
    b[0], b[1] = d_bits & 0xFF, d_bits >> 8
    b[2], b[3] = dmin_bits & 0xFF, dmin_bits >> 8
    b[4:16] = np.asarray(S, np.uint8)
    b[16:144] = np.asarray(Q, np.uint8)
    return b


# --------------------------------------------------------------------------- binary16

def check_half_all_patterns(o):
    bits = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    ref = bits.view(np.float16).astype(np.float64)
    got = np.array([o.half_to_double(int(b)) for b in bits])
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(got), nan), "NaN patterns differ"
    assert np.array_equal(got[~nan], ref[~nan]), "binary16 values differ from numpy"
    assert np.array_equal(np.signbit(got[~nan]), np.signbit(ref[~nan])), "sign of zero"


def check_half_known(o):
    table = {
        0x3C00: 1.0, 0x3800: 0.5, 0xC000: -2.0, 0x7BFF: 65504.0,
        0x0400: 2.0 ** -14,                 # smallest normal
        0x0001: 2.0 ** -24,                 # smallest subnormal
        0x03FF: 1023 * 2.0 ** -24,          # largest subnormal
        0x3555: 1365 * 2.0 ** -12,          # 0.333251953125
        0x7C00: float("inf"), 0xFC00: float("-inf"),
    }
    for b, v in table.items():
        assert o.half_to_double(b) == v, hex(b)
    assert np.signbit(o.half_to_double(0x8000)) and o.half_to_double(0x8000) == 0.0


# --------------------------------------------------------------------------- layout

def check_scale_bit_map(o):
    """Set one bit of the 12 scale bytes at a time; exactly one 6-bit field may
    change, by the power of two the packing assigns to that bit.

    Bit map (byte i of S, bit b), written in the bit -> field direction:
      i in 0..3  : b < 6 -> sc[i]   bit b ;  b >= 6 -> sc[i+4] bit b-2
      i in 4..7  : b < 6 -> m[i-4]  bit b ;  b >= 6 -> m[i]    bit b-2
      i in 8..11 : b < 4 -> sc[i-4] bit b ;  b >= 4 -> m[i-4]  bit b-4
    """
    for i in range(12):
        for b in range(8):
            S = np.zeros(12, np.uint8)
            S[i] = 1 << b
            _, _, sc, mn, q = o.unpack(_block(0, 0, S, np.zeros(128, np.uint8)))
            if i < 4:
                field, j, bit = ("sc", i, b) if b < 6 else ("sc", i + 4, b - 2)
            elif i < 8:
                field, j, bit = ("m", i - 4, b) if b < 6 else ("m", i, b - 2)
            else:
                field, j, bit = ("sc", i - 4, b) if b < 4 else ("m", i - 4, b - 4)
            exp_sc = np.zeros(8, np.int64)
            exp_m = np.zeros(8, np.int64)
            (exp_sc if field == "sc" else exp_m)[j] = 1 << bit
            assert np.array_equal(sc, exp_sc) and np.array_equal(mn, exp_m), (i, b, sc, mn)
            assert not q.any()


def check_nibble_map(o):
    """sc_j = 1, m_j = 0, d = 1, dmin = 0: the dequantised block equals q. Setting
    one nibble of Q to 15 must set exactly one weight: the low nibble of byte b
    is weight 64*(b//32) + b%32, the high nibble is that index + 32."""
    S = np.array([1, 1, 1, 1, 0, 0, 0, 0, 1, 1, 1, 1], np.uint8)
    for b in range(128):
        for high in (0, 1):
            Q = np.zeros(128, np.uint8)
            Q[b] = 0xF0 if high else 0x0F
            v = o.dequant_f32(_block(H_ONE, 0, S, Q), 1, 256)[0]
            t = 64 * (b // 32) + (b % 32) + 32 * high
            exp = np.zeros(256, np.float32)
            exp[t] = 15.0
            assert np.array_equal(v, exp), (b, high)


def check_closed_forms(o):
    zero_q = np.zeros(128, np.uint8)
    ff = np.full(12, 0xFF, np.uint8)
    # 1) every scale byte 0xFF -> sc_j = m_j = 63; quants all zero -> -dmin*63.
    v = o.dequant_f32(_block(H_ONE, H_HALF, ff, zero_q), 1, 256)[0]
    assert np.all(v == np.float32(-31.5)), v[:4]
    # 2) same scales, every nibble 15 -> 1*63*15 - 0.5*63 = 913.5.
    v = o.dequant_f32(_block(H_ONE, H_HALF, ff, np.full(128, 0xFF, np.uint8)), 1, 256)[0]
    assert np.all(v == np.float32(913.5)), v[:4]
    # 3) only the top two bits of S[0..7] set: sc_0..3 = m_0..3 = 0 and
    #    sc_4..7 = m_4..7 = 0b110000 = 48. With q = 1 everywhere (bytes 0x11):
    #    weights 0..127 -> 0, weights 128..255 -> 48 - 0.5*48 = 24.
    S = np.array([0xC0] * 8 + [0] * 4, np.uint8)
    v = o.dequant_f32(_block(H_ONE, H_HALF, S, np.full(128, 0x11, np.uint8)), 1, 256)[0]
    assert np.all(v[:128] == 0) and np.all(v[128:] == np.float32(24.0)), v[::32]
    # 4) distinct fields per sub-block. S[0..3] = 1,2,3,4 (sc_0..3),
    #    S[4..7] = 1,3,5,7 (m_0..3), S[8..11] = 0x65,0x76,0x87,0x98
    #    (sc_4..7 = 5,6,7,8 low nibbles; m_4..7 = 6,7,8,9 high nibbles).
    #    Bytes 0x21: q = 1 in even sub-blocks (low nibbles), q = 2 in odd ones.
    #    d = 0.25, dmin = 0.125: value_j = 0.25*sc_j*q_j - 0.125*m_j.
    S = np.array([1, 2, 3, 4, 1, 3, 5, 7, 0x65, 0x76, 0x87, 0x98], np.uint8)
    v = o.dequant_f32(_block(H_QUARTER, H_EIGHTH, S, np.full(128, 0x21, np.uint8)), 1, 256)[0]
    expect = [0.125, 0.625, 0.125, 1.125, 0.5, 2.125, 0.75, 2.875]
    for j in range(8):
        assert np.all(v[32 * j:32 * j + 32] == np.float32(expect[j])), (j, v[32 * j])
    # 5) cancelling block: sc = 4, q = 15, m = 60, d = dmin -> every weight is 0.
    #    S[0..3] = 4, S[4..7] = 60 | (3 << 6) (m_j = 60 and top bits of m_4..7 = 3),
    #    S[0..3] also carry top bits of sc_4..7 = 0; S[8..11]: sc_4..7 low = 4,
    #    m_4..7 low nibble 60 & 15 = 12 -> 0xC4. m_4..7 = 12 | (3 << 4) = 60.
    S = np.array([4, 4, 4, 4, 60 | 0xC0, 60 | 0xC0, 60 | 0xC0, 60 | 0xC0,
                  0xC4, 0xC4, 0xC4, 0xC4], np.uint8)
    v = o.dequant_f32(_block(0x2E66, 0x2E66, S, np.full(128, 0xFF, np.uint8)), 1, 256)[0]
    assert np.all(v == 0), v[::32]


# --------------------------------------------------------------------------- unpack <-> pack

def check_pack_roundtrip(o, count=1500, seed=11):
    rng = np.random.default_rng(seed)
    for _ in range(count):
        d, dm = (int(v) for v in rng.integers(0, 65536, 2))
        sc = rng.integers(0, 64, 8)
        mn = rng.integers(0, 64, 8)
        q = rng.integers(0, 16, 256)
        d2, dm2, sc2, mn2, q2 = o.unpack(o.pack(d, dm, sc, mn, q))
        assert (d2, dm2) == (d, dm)
        assert np.array_equal(sc2, sc) and np.array_equal(mn2, mn) and np.array_equal(q2, q)
    # every value of every 6-bit field, one field at a time
    for j in range(8):
        for val in range(64):
            for which in (0, 1):
                sc = np.zeros(8, np.int64)
                mn = np.zeros(8, np.int64)
                (sc if which == 0 else mn)[j] = val
                _, _, sc2, mn2, _ = o.unpack(o.pack(0, 0, sc, mn, np.zeros(256)))
                assert np.array_equal(sc2, sc) and np.array_equal(mn2, mn), (j, val, which)


def check_unpack_pack_bytes(o, count=1500, seed=12):
    rng = np.random.default_rng(seed)
    for _ in range(count):
        b = rng.integers(0, 256, 144).astype(np.uint8)
        assert np.array_equal(o.pack(*o.unpack(b)), b)


# --------------------------------------------------------------------------- GEMV

def _exact_weight(d_bits, dmin_bits, sc, mn, q):
    """Exact rational d*sc*q - dmin*m, and its f32 rounding as a Fraction."""
    d = Fraction(float(np.uint16(d_bits).view(np.float16)))
    dmin = Fraction(float(np.uint16(dmin_bits).view(np.float16)))
    w = d * int(sc) * int(q) - dmin * int(mn)
    wd = float(w)
    assert Fraction(wd) == w, "value not exact in double"
    return Fraction(float(np.float32(wd)))


def check_bruteforce_gemv(o, seed=13):
    """Tiny N, K: y from the unpacked integer fields in exact rational arithmetic
    (dequantised weights rounded once to f32, as the format's f32 value) versus
    the oracle's double GEMV on the packed bytes."""
    rng = np.random.default_rng(seed)
    for n, k in [(1, 256), (3, 256), (2, 512), (4, 512)]:
        nsb = k // 256
        fields = []
        blocks = []
        for _ in range(n * nsb):
            d = int(np.float16(rng.uniform(1e-3, 2e-2)).view(np.uint16))
            dm = int(np.float16(rng.uniform(1e-3, 2e-2)).view(np.uint16))
            sc, mn, q = rng.integers(0, 64, 8), rng.integers(0, 64, 8), rng.integers(0, 16, 256)
            fields.append((d, dm, sc, mn, q))
            blocks.append(o.pack(d, dm, sc, mn, q))
        w = np.concatenate(blocks)
        x = rng.standard_normal((2, k)).astype(np.float32)
        y, a = o.gemv(w, x, n, k)
        for i in range(2):
            for r in range(n):
                s = Fraction(0)
                for b in range(nsb):
                    d, dm, sc, mn, q = fields[r * nsb + b]
                    for t in range(256):
                        s += _exact_weight(d, dm, sc[t // 32], mn[t // 32], q[t]) * \
                            Fraction(float(x[i, 256 * b + t]))
                err = abs(Fraction(y[i, r]) - s)
                assert err <= Fraction(k * 2.0 ** -52) * Fraction(a[i, r]), (n, k, i, r)


def check_gemv_vs_matmul(o, seed=14):
    for n, k, m in [(5, 256, 1), (33, 768, 3), (17, 1024, 8)]:
        w, x = q4k_synth.q4k_problem(n, k, m, seed)
        y, a = o.gemv(w, x, n, k)
        ref = x.astype(np.float64) @ o.dequant_f32(w, n, k).astype(np.float64).T
        assert np.all(np.abs(y - ref) <= 1e-12 * a + 1e-300), (n, k, m)
        absref = np.abs(x.astype(np.float64)) @ np.abs(o.dequant_f32(w, n, k).astype(np.float64)).T
        assert np.allclose(a, absref, rtol=1e-12, atol=0), (n, k, m)


def check_unit_and_zero_vectors(o, seed=15):
    n, k = 9, 512
    w, _ = q4k_synth.q4k_problem(n, k, 1, seed)
    deq = o.dequant_f32(w, n, k)
    for col in (0, 1, 31, 32, 63, 64, 255, 256, 300, 511):
        x = np.zeros((1, k), np.float32)
        x[0, col] = 1.0
        y, _ = o.gemv(w, x, n, k)
        assert np.array_equal(y[0], deq[:, col].astype(np.float64)), col
    y, a = o.gemv(w, np.zeros((1, k), np.float32), n, k)
    assert not y.any() and not a.any()


def check_vectors_independent(o, seed=16):
    n, k, m = 7, 512, 5
    w, x = q4k_synth.q4k_problem(n, k, m, seed)
    y, a = o.gemv(w, x, n, k)
    for i in range(m):
        yi, ai = o.gemv(w, x[i:i + 1], n, k)
        assert np.array_equal(yi[0], y[i]) and np.array_equal(ai[0], a[i])


def check_threads_and_rows(o, seed=17):
    n, k, m = 37, 768, 2
    w, x = q4k_synth.q4k_problem(n, k, m, seed)
    y1, a1 = o.gemv(w, x, n, k, nthreads=1)
    y4, a4 = o.gemv(w, x, n, k, nthreads=4)
    assert np.array_equal(y1, y4) and np.array_equal(a1, a4)
    rows = [0, 5, 36, 5]
    yr, ar = o.gemv_rows(w, x, n, k, rows)
    assert np.array_equal(yr, y1[:, rows]) and np.array_equal(ar, a1[:, rows])
    assert np.array_equal(o.dequant_rows(w, n, k, rows), o.dequant_f32(w, n, k)[rows])


def check_golden(o):
    """Regression values written by tests/golden/make_golden.py (oracle only)."""
    path = os.path.join(GOLDEN, "tiny_256x1024_seed0.txt")
    rows = []
    with open(path) as f:
        for line in f:
            if line.startswith("#") or not line.strip():
                continue
            rows.append([float.fromhex(t) for t in line.split()])
    ref = np.array(rows)               # columns: y, a, dequant[n][0], dequant[n][255]
    w, x = q4k_synth.q4k_problem(256, 1024, 1, q4k_synth.SEEDS[(256, 1024)])
    y, a = o.gemv(w, x, 256, 1024)
    deq = o.dequant_f32(w, 256, 1024)
    assert np.array_equal(y[0], ref[:, 0]) and np.array_equal(a[0], ref[:, 1])
    assert np.array_equal(deq[:, 0].astype(np.float64), ref[:, 2])
    assert np.array_equal(deq[:, 255].astype(np.float64), ref[:, 3])


def check_embed_page_cases(o):
    """The page's own validation test (tests/golden/embed_validation_cases.txt)."""
    path = os.path.join(GOLDEN, "embed_validation_cases.txt")
    n = 0
    with open(path) as f:
        for line in f:
            if line.startswith("#") or not line.strip():
                continue
            *nums, expect = line.split()
            st = o.embed_validate(*[int(v) for v in nums])
            assert (st == 0) == (expect == "ok"), line
            n += 1
    assert n == 4


def check_embed_rules(o):
    """Each validation rule alone, in the page's order (codes: 1 shape, 2 token,
    3 width, 4 overflow, 5 size)."""
    row = 144
    ok = (10 * row, 10, 256, 256, 9)
    assert o.embed_validate(*ok) == 0
    assert o.embed_validate(10 * row, 10, 512, 256, 9) == 1          # cols != hidden
    assert o.embed_validate(10 * row, 10, 256, 256, 10) == 2         # token == rows
    assert o.embed_validate(0, 0, 256, 256, 0) == 2                  # empty table
    assert o.embed_validate(10 * row, 10, 300, 300, 0) == 3          # not whole blocks
    assert o.embed_validate(0, 10, 0, 0, 0) == 3                     # zero width
    assert o.embed_validate(10 * row + 1, 10, 256, 256, 0) == 5      # one byte too many
    assert o.embed_validate(10 * row - 1, 10, 256, 256, 0) == 5      # one byte short
    assert o.embed_validate(20 * 2 * row, 20, 512, 512, 19) == 0     # two blocks per row
    assert o.embed_validate(20 * 2 * row, 20, 512, 512, 20) == 2
    # shape is checked before the token, the token before the width
    assert o.embed_validate(0, 1, 512, 256, 5) == 1
    assert o.embed_validate(0, 1, 300, 300, 5) == 2
    big = 1 << 63
    assert o.embed_validate(0, big, 256, 256, 0) == 4                # rows * row_bytes overflows
    assert o.embed_validate(0, big, 1 << 62, 1 << 62, 0) == 4        # wide rows: table size overflows


def check_embed_values(o, seed=18):
    """Rows 0, mid and last of small tables, several scales, against exact
    arithmetic from the unpacked fields: w = d*sc*q - dmin*m rounded to f32, then
    w * scale rounded to f32."""
    rng = np.random.default_rng(seed)
    for rows, hidden in [(3, 256), (5, 512), (2, 768)]:
        nsb = hidden // 256
        fields, blocks = [], []
        for _ in range(rows * nsb):
            d = int(np.float16(rng.uniform(1e-3, 2e-2)).view(np.uint16))
            dm = int(np.float16(rng.uniform(1e-3, 2e-2)).view(np.uint16))
            sc, mn, q = rng.integers(0, 64, 8), rng.integers(0, 64, 8), rng.integers(0, 16, 256)
            fields.append((d, dm, sc, mn, q))
            blocks.append(o.pack(d, dm, sc, mn, q))
        table = np.concatenate(blocks)
        for token in sorted({0, rows // 2, rows - 1}):
            for scale in (1.0, 2.0, -0.5, 0.0, float(np.float32(0.1234567)), 3.0e-3):
                st, out = o.embed_lookup(table, rows, hidden, hidden, token, scale)
                assert st == 0
                for b in range(nsb):
                    d, dm, sc, mn, q = fields[token * nsb + b]
                    for t in range(0, 256, 7):
                        w = _exact_weight(d, dm, sc[t // 32], mn[t // 32], q[t])
                        ref = np.float32(float(w * Fraction(float(np.float32(scale)))))
                        got = out[b * 256 + t]
                        assert got == ref or (np.isnan(got) and np.isnan(ref)), \
                            (rows, hidden, token, scale, b, t, got, ref)
    # a failed rule writes nothing and returns no row
    st, out = o.embed_lookup(np.zeros(144 * 4, np.uint8), 4, 256, 256, 4, 1.0)
    assert st == 2 and out is None


def check_swiglu_composition(o, seed=19):
    """SwiGLU GEMV: out = g * expit(g) * u with scipy's logistic function (a
    library routine), g and u the GEMVs of the two matrices; special cases
    silu(0) = 0, a zero up-projection gives 0, and silu(g) -> g for large g."""
    import oracle as oracle_mod
    from scipy.special import expit
    saved = oracle_mod._default
    oracle_mod._default = o
    try:
        n, k, m = 21, 768, 3
        wg, x = q4k_synth.q4k_problem(n, k, m, seed)
        wu, _ = q4k_synth.q4k_problem(n, k, 1, seed + 1)
        out, g, u, a_g, a_u = oracle_mod.swiglu_gemv(wg, wu, x, n, k)
        g2, _ = o.gemv(wg, x, n, k)
        u2, _ = o.gemv(wu, x, n, k)
        assert np.array_equal(g, g2) and np.array_equal(u, u2)
        assert np.allclose(out, g * expit(g) * u, rtol=1e-14, atol=0)
        zero, *_ = oracle_mod.swiglu_gemv(wg, wu, np.zeros((1, k), np.float32), n, k)
        assert not zero.any()
        same, gg, uu, *_ = oracle_mod.swiglu_gemv(wg, wg, 50.0 * x[:1], n, k)
        big = gg[0] > 40
        assert big.any() and np.allclose(same[0][big], gg[0][big] ** 2, rtol=1e-15)
    finally:
        oracle_mod._default = saved


# --------------------------------------------------------------------------- fp16 mirror

def check_float_to_half_vs_numpy(o, seed=20):
    """binary32 -> binary16 RNE against numpy's float32 -> float16 conversion (a
    library routine) on random bit patterns, on every binary16 value, on the
    midpoints between neighbouring binary16 values and just either side of them."""
    rng = np.random.default_rng(seed)
    h = np.arange(0x7C00, dtype=np.uint32).astype(np.uint16)
    hv = h.view(np.float16).astype(np.float64)
    mids = (hv[:-1] + hv[1:]) / 2                      # exact in float32 below 2^16
    mids32 = mids.astype(np.float32)
    assert np.array_equal(mids32.astype(np.float64), mids)
    near = np.concatenate([np.nextafter(mids32, np.float32(0)), mids32,
                           np.nextafter(mids32, np.float32(np.inf))])
    rand = rng.integers(0, 2 ** 32, 400_000, dtype=np.uint64).astype(np.uint32).view(np.float32)
    special = np.array([0.0, -0.0, 65504, 65519.996, 65520, 65536, 1e30, -1e30, np.inf, -np.inf,
                        2.0 ** -24, 2.0 ** -25, 3 * 2.0 ** -25, 2.0 ** -26, 1e-45, -1e-45],
                       np.float32)
    for x in (hv.astype(np.float32), near, rand, special, -near):
        got = o.floats_to_half(x)
        with np.errstate(over="ignore"):
            ref = x.astype(np.float16).view(np.uint16)
        nan = np.isnan(x)
        assert np.array_equal(got[~nan], ref[~nan]), \
            f"{int((got[~nan] != ref[~nan]).sum())} conversions differ from numpy"
        assert np.all(np.isnan(got[nan].view(np.float16)))


def check_float_to_half_known(o):
    """Hand-derived roundings: ties go to the even bit pattern, 65520 overflows."""
    table = {1.0: 0x3C00, 65504.0: 0x7BFF, 65519.99: 0x7BFF, 65520.0: 0x7C00,
             2.0 ** -24: 0x0001, 2.0 ** -25: 0x0000, 3 * 2.0 ** -25: 0x0002,
             5 * 2.0 ** -25: 0x0002, 1 + 2.0 ** -11: 0x3C00, 1 + 3 * 2.0 ** -11: 0x3C02,
             -2.0: 0xC000, 2.0 ** -14: 0x0400, 1023 * 2.0 ** -24: 0x03FF,
             (2047 / 2) * 2.0 ** -24: 0x0400}
    for v, bits in table.items():
        assert int(o.floats_to_half(np.array([v], np.float32))[0]) == bits, (v, hex(bits))


def check_dequant_f16(o, seed=21):
    """The mirror is the binary16 rounding of the pinned f32 dequantisation:
    against numpy's conversion of the oracle's f32 values, and a closed form."""
    n, k = 6, 512
    w, _ = q4k_synth.q4k_problem(n, k, 1, seed)
    got = o.dequant_f16(w, n, k)
    assert np.array_equal(got, o.dequant_f32(w, n, k).astype(np.float16).view(np.uint16))
    ff = np.full(12, 0xFF, np.uint8)
    blk = _block(H_ONE, H_HALF, ff, np.full(128, 0xFF, np.uint8))   # every weight 913.5
    assert np.all(o.dequant_f16(blk, 1, 256) == np.float16(913.5).view(np.uint16))
    blk = _block(H_ONE, H_HALF, ff, np.zeros(128, np.uint8))        # every weight -31.5
    assert np.all(o.dequant_f16(blk, 1, 256) == np.float16(-31.5).view(np.uint16))


def check_gemm_f16(o, seed=22):
    """fp16 GEMM reference: exact rational sums of the binary16 products on a
    tiny problem, unit vectors giving columns, and |.| sums."""
    rng = np.random.default_rng(seed)
    n, m, k = 3, 2, 16
    w16 = rng.integers(0, 0x7C00, (n, k)).astype(np.uint16) | \
        (rng.integers(0, 2, (n, k)).astype(np.uint16) << 15)
    x16 = rng.integers(0x2000, 0x5000, (m, k)).astype(np.uint16)
    y, a = o.gemm_f16(w16, x16)
    for i in range(m):
        for r in range(n):
            ex = sum(Fraction(float(np.uint16(w16[r, t]).view(np.float16))) *
                     Fraction(float(np.uint16(x16[i, t]).view(np.float16))) for t in range(k))
            ab = sum(abs(Fraction(float(np.uint16(w16[r, t]).view(np.float16))) *
                         Fraction(float(np.uint16(x16[i, t]).view(np.float16)))) for t in range(k))
            assert abs(Fraction(y[i, r]) - ex) <= abs(ex) * Fraction(1, 2 ** 50), (i, r)
            assert abs(Fraction(a[i, r]) - ab) <= ab * Fraction(1, 2 ** 50), (i, r)
    eye = np.zeros((k, k), np.uint16)
    eye[np.arange(k), np.arange(k)] = 0x3C00                        # binary16 1.0
    cols, _ = o.gemm_f16(w16, eye)
    assert np.array_equal(cols, np.array([[float(np.uint16(b).view(np.float16)) for b in row]
                                          for row in w16]).T)
    sub, _ = o.gemm_f16(w16, x16, rows=[2, 0])
    assert np.array_equal(sub, y[:, [2, 0]])


ALL_CHECKS = [
    check_half_all_patterns, check_half_known, check_scale_bit_map, check_nibble_map,
    check_closed_forms, check_pack_roundtrip, check_unpack_pack_bytes, check_bruteforce_gemv,
    check_gemv_vs_matmul, check_unit_and_zero_vectors, check_vectors_independent,
    check_threads_and_rows, check_golden, check_embed_page_cases, check_embed_rules,
    check_embed_values, check_swiglu_composition, check_float_to_half_vs_numpy,
    check_float_to_half_known, check_dequant_f16, check_gemm_f16,
]
