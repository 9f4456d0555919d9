"""Hand-built Q4_K matrices for the GPU parity tests: blocks whose weights
stress the per-element accuracy bound (all-zero quants, near-cancelling
scale/min pairs). Built with the oracle's packer (pinned by round trips in
tests/oracle_pins.py); no GPU code here."""
import numpy as np

import oracle


def uniform_block(d_bits, dmin_bits, sc, mn, q):
    """One superblock with sc_j, m_j (sequences of 8) and quant q_j (constant
    within sub-block j) packed by the oracle's packer."""
    qv = np.repeat(np.asarray(q, np.int64), 32)
    return oracle.pack(d_bits, dmin_bits, np.asarray(sc, np.int64), np.asarray(mn, np.int64), qv)


def zero_quant_matrix(n, k):
    # every quant 0: each weight is -dmin * m_j = -dmin (m_j = 1), with
    # d = 0x251F (about 0.0200), dmin = 0x1438 (about 0.00103), sc_j = 50
    b = uniform_block(0x251F, 0x1438, [50] * 8, [1] * 8, [0] * 8)
    return np.tile(b, n * (k // 256))


def near_cancelling_matrix(n, k, seed):
    """Blocks whose weights d*sc_j - dmin*m_j nearly cancel, with d != dmin:
    q_j = 1, sc_j in 40..63, d just above a power of two 2^e and dmin just below
    it (so dmin's lowest mantissa bit is half of d's and 128*d*sc_j + dmin*m_j
    can need 25 bits), m_j = rint(sc_j*d/dmin) <= 63. Each weight is then about
    sc_j*(d - dmin), a few hundredths of d*sc_j."""
    rng = np.random.default_rng(seed)
    nsb = n * (k // 256)
    out = np.empty((nsb, 144), np.uint8)
    for i in range(nsb):
        e = int(rng.integers(-9, -5))                       # d, dmin around 2^-9 .. 2^-6
        d = np.float16(2.0 ** e * (1 + rng.integers(1, 24) / 1024))
        dmin = np.float16(2.0 ** e * (1 - rng.integers(1, 48) / 2048))
        r = float(d) / float(dmin)
        sc = rng.integers(40, int(63 / r) + 1, 8)
        mn = np.clip(np.rint(sc * r), 0, 63).astype(np.int64)
        out[i] = uniform_block(int(d.view(np.uint16)), int(dmin.view(np.uint16)), sc, mn, [1] * 8)
    return out.reshape(-1)
