"""Writes the oracle regression fixture tiny_256x1024_seed0.txt.

Calls only the CPU oracle (and the seeded input generator). The pages print no
worked example for Q4_K, so this file pins the oracle against silent change,
not against the pages: columns are y[n], a[n] = sum|w x|, W[n][0], W[n][255]
of the tiny 256x1024 problem (seed 0), as float.hex.
Run from the repository root: python tests/golden/make_golden.py
"""
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
sys.path.insert(0, ROOT)

import oracle  # noqa: E402
import q4k_synth  # noqa: E402


def main():
    n, k = 256, 1024
    w, x = q4k_synth.q4k_problem(n, k, 1, q4k_synth.SEEDS[(n, k)])
    y, a = oracle.gemv(w, x, n, k)
    deq = oracle.dequant_f32(w, n, k)
    out = os.path.join(os.path.dirname(os.path.abspath(__file__)), "tiny_256x1024_seed0.txt")
    with open(out, "w") as f:
        f.write("# written by tests/golden/make_golden.py from the CPU oracle only\n")
        f.write("# tiny Q4_K GEMV N=256 K=1024 m=1 seed 0; columns: y a W[n][0] W[n][255]\n")
        for r in range(n):
            f.write(" ".join(float(v).hex() for v in
                             (y[0, r], a[0, r], deq[r, 0], deq[r, 255])) + "\n")


if __name__ == "__main__":
    main()
