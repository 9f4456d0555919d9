"""The seeded input generator: reproducible, right sizes, right distributions (CPU)."""
import numpy as np

import q4k_synth


def test_sizes_match_the_q4k_size_rule():
    # 144 bytes = 2 (d) + 2 (dmin) + 12 (scales) + 128 (quants) per 256 weights
    assert q4k_synth.BLOCK_BYTES == 2 + 2 + 12 + 128
    for (n, k) in (q4k_synth.SHAPES_TINY + q4k_synth.SHAPES_1P5B + q4k_synth.SHAPES_7B
                   + q4k_synth.SHAPES_8B):
        w, x = q4k_synth.q4k_problem(n, k, 1, 0) if n * k <= 1 << 24 else (None, None)
        assert q4k_synth.weight_bytes(n, k) == n * k // 256 * 144
        if w is not None:
            assert w.size == n * k // 256 * 144 and x.shape == (1, k)
    assert q4k_synth.weight_bytes(128256, 4096) == 295_501_824
    assert sum(q4k_synth.weight_bytes(n, k) for n, k in q4k_synth.LAYER_8B) == 122_683_392


def test_reproducible_and_seed_dependent():
    a = q4k_synth.q4k_problem(64, 512, 2, 5)
    b = q4k_synth.q4k_problem(64, 512, 2, 5)
    c = q4k_synth.q4k_problem(64, 512, 2, 6)
    assert np.array_equal(a[0], b[0]) and np.array_equal(a[1], b[1])
    assert not np.array_equal(a[0], c[0])


def test_value_distributions():
    w, x = q4k_synth.q4k_problem(512, 4096, 1, 3)
    sb = w.reshape(-1, 144)
    d = sb[:, 0:2].copy().view('<f2').astype(np.float64).ravel()
    dmin = sb[:, 2:4].copy().view('<f2').astype(np.float64).ravel()
    for v in (d, dmin):
        assert v.min() >= np.float16(1e-3) and v.max() <= np.float16(2e-2)
        assert abs(v.mean() - 0.0105) < 5e-4
    rest = sb[:, 4:].ravel()
    assert rest.min() == 0 and rest.max() == 255 and abs(rest.mean() - 127.5) < 1.0
    assert abs(x.mean()) < 0.05 and abs(x.std() - 1.0) < 0.05 and x.dtype == np.float32
