"""Parity of the integer tensor-core GEMV (q4k_gemv with m = 1..4 on tall
matrices, Q4K_KERNEL_I8) with the CPU oracle, on a B200.

Bound: |y_gpu - y_ref| <= 1e-4 * sum|w x| + 1e-6 per element (y_ref in double),
as for every q4k_gemv path. The cases here are the ones its number format and
launch shape add: x is scaled per 256-element block by the block's largest
magnitude and split into base-128 digits (dynamic range inside a block, tiny,
huge, subnormal and zero blocks, non-finite values); CTAs own whole 128-row
tiles (a ragged last tile, one and several superblock columns per tile, an odd
column count, the largest K whose digit image fits shared memory); each
item's sums are split between two epilogue warps and added at the tile's end.
Two to four vectors share each decoded superblock (base-256 digits of every
vector in one MMA operand, vector 3 unused for m = 3); each epilogue warp sums
its own vectors, and cut tiles publish a piece per vector.
"""
import numpy as np
import pytest

import oracle
import q4k_synth

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def q4k():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import gguf_quant_dequant_q4k_b200 as lib
    return lib


def dev(a):
    return torch.from_numpy(np.ascontiguousarray(a)).cuda()


def gpu_gemv(q4k, w, x, n, k):
    x = np.asarray(x, np.float32).reshape(-1, k)
    m = x.shape[0]
    assert q4k.q4k_gemv_plan_for(m, n, k, 148)["kernel"] == q4k.Q4K_KERNEL_I8
    y = torch.full((m, n), float("nan"), dtype=torch.float32, device="cuda")
    q4k.q4k_gemv(dev(w), dev(x), y, m, n, k)
    torch.cuda.synchronize()
    return y.cpu().numpy()


def assert_gemv_close(y, yref, a, what=""):
    err = np.abs(y.astype(np.float64) - yref)
    tol = oracle.tolerance(a)
    bad = ~(err <= tol)
    assert not bad.any(), (f"{what}: {bad.sum()} elements out of tolerance; worst "
                           f"err/tol={np.nanmax(err / tol):.3g}")


def sampled(n, count, seed):
    rng = np.random.default_rng(seed)
    return np.unique(np.concatenate([[0, 1, 127, 128, n - 128, n - 1], rng.integers(0, n, count)]))


@pytest.mark.parametrize("n,k", [(296 * 128 - 51, 512), (296 * 128, 768), (148 * 128 * 3 - 5, 1024)])
def test_i8_ragged_tiles(q4k, n, k):
    """Two or three tiles per CTA, a 77-row last tile; 2, 3 and 4 superblock
    columns per tile (an odd count moves the tile end between the epilogue
    warps' items)."""
    w, x = q4k_synth.q4k_problem(n, k, 1, n % 1000 + k)
    y = gpu_gemv(q4k, w, x, n, k)
    yref, a = oracle.gemv(w, x, n, k, nthreads=8)
    assert_gemv_close(y, yref, a, f"{n}x{k}")


@pytest.mark.parametrize("n,k", [(11008, 4096), (4096, 14336), (3000, 15872), (4096 + 77, 8192)])
def test_i8_cut_tiles(q4k, n, k):
    """Fewer tiles than a whole-tile split needs: equal item ranges, tiles cut
    between CTAs and finished from their pieces (in CTA order) by the last CTA
    to publish one; a ragged last tile; identical bits on a second call (the
    stream's scratch counters are left zero by each launch)."""
    w, x = q4k_synth.q4k_problem(n, k, 1, q4k_synth.SEEDS.get((n, k), n + k))
    y = gpu_gemv(q4k, w, x, n, k)
    y2 = gpu_gemv(q4k, w, x, n, k)
    assert np.array_equal(y.view(np.uint32), y2.view(np.uint32))
    yref, a = oracle.gemv(w, x, n, k, nthreads=8)
    assert_gemv_close(y, yref, a, f"{n}x{k}")


def test_i8_one_column_tiles(q4k):
    """K = 256: every item ends a tile (1185 tiles, 8 or 9 per CTA)."""
    n, k = 1184 * 128 + 1, 256
    w, x = q4k_synth.q4k_problem(n, k, 1, 11)
    y = gpu_gemv(q4k, w, x, n, k)
    yref, a = oracle.gemv(w, x, n, k, nthreads=8)
    assert_gemv_close(y, yref, a, "K = 256")


def test_i8_largest_k(q4k):
    """K = 62 * 256, the longest row whose digit image fits beside four weight
    stages; one tile per CTA."""
    n, k = 148 * 128, 62 * 256
    w, x = q4k_synth.q4k_problem(n, k, 1, 62)
    y = gpu_gemv(q4k, w, x, n, k)
    rows = sampled(n, 120, 5)
    yref, a = oracle.gemv_rows(w, x, n, k, rows)
    assert_gemv_close(y[:, rows], yref, a, "K = 15872")


def test_i8_block_dynamic_range(q4k):
    """Blocks scaled by 1e-30 and 1e30, a block of subnormals, an all-zero
    block, a block whose largest value is 2^20 times its others, a block of
    equal values."""
    n, k = 296 * 128, 2048
    w, x = q4k_synth.q4k_problem(n, k, 1, 77)
    x = x.reshape(k).copy()
    x[0:256] *= np.float32(1e-30)
    x[256:512] *= np.float32(1e30)
    x[512:768] = (np.arange(256, dtype=np.float32) - 128) * np.float32(1e-43)
    x[768:1024] = 0.0
    x[1024 + 17] = np.float32(2.0 ** 20)
    x[1280:1536] = np.float32(1.0)
    y = gpu_gemv(q4k, w, x, n, k)
    yref, a = oracle.gemv(w, x, n, k, nthreads=8)
    assert_gemv_close(y, yref, a, "dynamic range")


@pytest.mark.parametrize("t", [0, 31, 32, 255, 256 + 100, 2047])
def test_i8_unit_vector_is_exact_column(q4k, t):
    """x = e_t scales to 2^32 (one digit 16): y is d*sc*q - dmin*m formed
    exactly and rounded once, i.e. the f32 dequantised column, bit for bit
    (low and high nibbles, first and last sub-blocks)."""
    n, k = 296 * 128 - 3, 2048
    w, _ = q4k_synth.q4k_problem(n, k, 1, 32)
    x = np.zeros(k, np.float32)
    x[t] = 1.0
    y = gpu_gemv(q4k, w, x, n, k)
    col = oracle.dequant_f32(w, n, k).reshape(n, k)[:, t].copy()
    assert np.array_equal(y[0].view(np.uint32), col.view(np.uint32))


def test_i8_unit_vectors_every_column(q4k):
    """x = e_c for every column c of K = 512: each y is the dequantised column
    bit for bit."""
    n, k = 296 * 128 - 77, 512
    w, _ = q4k_synth.q4k_problem(n, k, 1, 36)
    deq = oracle.dequant_f32(w, n, k).reshape(n, k)
    wt = dev(w)
    x = torch.zeros((k, 1, k), dtype=torch.float32, device="cuda")
    x[torch.arange(k), 0, torch.arange(k)] = 1.0
    y = torch.full((k, 1, n), float("nan"), dtype=torch.float32, device="cuda")
    for c in range(k):
        q4k.q4k_gemv(wt, x[c], y[c], 1, n, k)
    torch.cuda.synchronize()
    got = y[:, 0, :].cpu().numpy()
    assert np.array_equal(got.view(np.uint32), deq.T.copy().view(np.uint32))


@pytest.mark.parametrize("bad", [np.inf, -np.inf, np.nan])
def test_i8_non_finite_vector_is_nan(q4k, bad):
    n, k = 296 * 128, 1024
    w, x = q4k_synth.q4k_problem(n, k, 1, 5)
    x = x.reshape(k).copy()
    x[700] = bad
    y = gpu_gemv(q4k, w, x, n, k)
    assert np.isnan(y).all()


def test_i8_deterministic_and_rows_only(q4k):
    """Two calls give identical bits; nothing outside y's n floats is written."""
    n, k = 296 * 128 - 51, 1536
    w, x = q4k_synth.q4k_problem(n, k, 1, 9)
    wt, xt = dev(w), dev(x.reshape(1, k))
    guard = 64
    buf = torch.full((n + 2 * guard,), 7.0, dtype=torch.float32, device="cuda")
    y = buf[guard:guard + n]
    q4k.q4k_gemv(wt, xt, y, 1, n, k)
    first = y.clone()
    q4k.q4k_gemv(wt, xt, y, 1, n, k)
    torch.cuda.synchronize()
    assert torch.equal(first.view(torch.int32), y.view(torch.int32))
    assert (buf[:guard] == 7.0).all() and (buf[guard + n:] == 7.0).all()
    yref, a = oracle.gemv(w, x, n, k, nthreads=8)
    assert_gemv_close(y.cpu().numpy().reshape(1, n), yref, a, "rows")


def test_i8_lm_head_sampled(q4k):
    """The 128256 x 4096 LM head: 1002 tiles, 7 on most CTAs; 200 sampled rows."""
    n, k = 128256, 4096
    w, x = q4k_synth.q4k_problem(n, k, 1, q4k_synth.SEEDS[(n, k)])
    y = gpu_gemv(q4k, w, x, n, k)
    rows = sampled(n, 200, 3)
    yref, a = oracle.gemv_rows(w, x, n, k, rows)
    assert_gemv_close(y[:, rows], yref, a, "LM head")


def test_i8_graph_capture_and_two_streams(q4k):
    """Calls captured in a CUDA graph replay to the eager result; calls on two
    streams at once both match it."""
    n, k = 296 * 128, 1024
    w, x = q4k_synth.q4k_problem(n, k, 1, 17)
    wt, xt = dev(w), dev(x.reshape(1, k))
    eager = torch.empty((1, n), dtype=torch.float32, device="cuda")
    q4k.q4k_gemv(wt, xt, eager, 1, n, k)
    torch.cuda.synchronize()
    s = torch.cuda.Stream()
    ys = [torch.full((1, n), float("nan"), device="cuda") for _ in range(3)]
    with torch.cuda.stream(s):
        q4k.q4k_gemv(wt, xt, ys[0], 1, n, k, stream=s)
    s.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=s):
        for y in ys:
            q4k.q4k_gemv(wt, xt, y, 1, n, k, stream=s)
    for y in ys:
        y.fill_(float("nan"))
    torch.cuda.synchronize()
    with torch.cuda.stream(s):
        g.replay()
        g.replay()
    s.synchronize()
    for y in ys:
        assert torch.equal(y.view(torch.int32), eager.view(torch.int32))
    del g
    s1, s2 = torch.cuda.Stream(), torch.cuda.Stream()
    y1 = torch.full((1, n), float("nan"), device="cuda")
    y2 = torch.full((1, n), float("nan"), device="cuda")
    torch.cuda.synchronize()
    for _ in range(5):
        q4k.q4k_gemv(wt, xt, y1, 1, n, k, stream=s1)
        q4k.q4k_gemv(wt, xt, y2, 1, n, k, stream=s2)
    torch.cuda.synchronize()
    assert torch.equal(y1.view(torch.int32), eager.view(torch.int32))
    assert torch.equal(y2.view(torch.int32), eager.view(torch.int32))
    yref, a = oracle.gemv(w, x, n, k, nthreads=8)
    assert_gemv_close(eager.cpu().numpy(), yref, a, "eager")


# ------------------------------------------------------------ 2 to 4 vectors

@pytest.mark.parametrize("m", [2, 3, 4])
@pytest.mark.parametrize("n,k", [(296 * 128 - 51, 512), (11008, 4096), (4096 + 77, 8192), (3000, 15872),
                                 (20000, 2304)])
def test_i8_vectors_ragged_and_cut_tiles(q4k, n, k, m):
    """Whole tiles with a ragged last one; tiles cut between CTAs with a piece
    per vector; 62 superblock columns; an odd 9 (two columns per item for two
    vectors, the padded column skipped). Identical bits on a second call."""
    w, x = q4k_synth.q4k_problem(n, k, m, n % 1000 + k + m)
    y = gpu_gemv(q4k, w, x, n, k)
    y2 = gpu_gemv(q4k, w, x, n, k)
    assert np.array_equal(y.view(np.uint32), y2.view(np.uint32))
    yref, a = oracle.gemv(w, x, n, k, nthreads=8)
    assert_gemv_close(y, yref, a, f"{n}x{k} m={m}")


@pytest.mark.parametrize("m", [3, 4])
def test_i8_vectors_dynamic_range(q4k, m):
    """Each vector its own scales: one at 1e-30, one at 1e30, one with a
    subnormal block, a zero block and a 2^20 outlier; the last one unchanged."""
    n, k = 296 * 128, 2048
    w, x = q4k_synth.q4k_problem(n, k, m, 78)
    x = x.reshape(m, k).copy()
    x[0] *= np.float32(1e-30)
    x[1] *= np.float32(1e30)
    x[2, 512:768] = (np.arange(256, dtype=np.float32) - 128) * np.float32(1e-43)
    x[2, 768:1024] = 0.0
    x[2, 1024 + 17] = np.float32(2.0 ** 20)
    y = gpu_gemv(q4k, w, x, n, k)
    yref, a = oracle.gemv(w, x, n, k, nthreads=8)
    assert_gemv_close(y, yref, a, f"dynamic range m={m}")


@pytest.mark.parametrize("m", [2, 4])
def test_i8_vectors_unit_columns(q4k, m):
    """x_v = e_(t_v): every y_v is the f32 dequantised column t_v, bit for bit
    (the unit scales to 2^29, one base-256 digit 32)."""
    n, k = 296 * 128 - 3, 2048
    w, _ = q4k_synth.q4k_problem(n, k, 1, 33)
    ts = [0, 255, 256 + 100, 2047][:m]
    x = np.zeros((m, k), np.float32)
    for v, t in enumerate(ts):
        x[v, t] = 1.0
    y = gpu_gemv(q4k, w, x, n, k)
    deq = oracle.dequant_f32(w, n, k).reshape(n, k)
    for v, t in enumerate(ts):
        assert np.array_equal(y[v].view(np.uint32), deq[:, t].copy().view(np.uint32)), (v, t)


def test_i8_vectors_non_finite_stays_in_its_vector(q4k):
    """A NaN in vector 1 makes all of y_1 NaN and leaves the others exact to
    the bound."""
    n, k, m = 11008, 4096, 4
    w, x = q4k_synth.q4k_problem(n, k, m, 6)
    x = x.reshape(m, k).copy()
    x[1, 3000] = np.nan
    y = gpu_gemv(q4k, w, x, n, k)
    assert np.isnan(y[1]).all()
    keep = [0, 2, 3]
    yref, a = oracle.gemv(w, x[keep], n, k, nthreads=8)
    assert_gemv_close(y[keep], yref, a, "other vectors")


def test_i8_vectors_rows_only(q4k):
    """Nothing outside y's m x n floats is written."""
    n, k, m = 4096, 14336, 3
    w, x = q4k_synth.q4k_problem(n, k, m, 10)
    wt, xt = dev(w), dev(x.reshape(m, k))
    guard = 64
    buf = torch.full((m * n + 2 * guard,), 7.0, dtype=torch.float32, device="cuda")
    y = buf[guard:guard + m * n].view(m, n)
    q4k.q4k_gemv(wt, xt, y, m, n, k)
    torch.cuda.synchronize()
    assert (buf[:guard] == 7.0).all() and (buf[guard + m * n:] == 7.0).all()
    rows = sampled(n, 60, 4)
    yref, a = oracle.gemv_rows(w, x, n, k, rows)
    assert_gemv_close(y.cpu().numpy()[:, rows], yref, a, "rows m=3")


@pytest.mark.parametrize("m", [2, 4])
def test_i8_vectors_lm_head_sampled(q4k, m):
    """The 128256 x 4096 LM head with two and four vectors; 100 sampled rows."""
    n, k = 128256, 4096
    w, x = q4k_synth.q4k_problem(n, k, m, 12 + m)
    y = gpu_gemv(q4k, w, x, n, k)
    rows = sampled(n, 100, 7)
    yref, a = oracle.gemv_rows(w, x, n, k, rows)
    assert_gemv_close(y[:, rows], yref, a, f"LM head m={m}")


def test_i8_vectors_graph_capture_and_two_streams(q4k):
    """Four vectors on cut tiles: graph replays and two concurrent streams give
    the eager bits (each stream's piece scratch holds four vectors)."""
    n, k, m = 11008, 4096, 4
    w, x = q4k_synth.q4k_problem(n, k, m, 18)
    wt, xt = dev(w), dev(x.reshape(m, k))
    eager = torch.empty((m, n), dtype=torch.float32, device="cuda")
    q4k.q4k_gemv(wt, xt, eager, m, n, k)
    torch.cuda.synchronize()
    s = torch.cuda.Stream()
    y = torch.full((m, n), float("nan"), device="cuda")
    with torch.cuda.stream(s):
        q4k.q4k_gemv(wt, xt, y, m, n, k, stream=s)
    s.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=s):
        q4k.q4k_gemv(wt, xt, y, m, n, k, stream=s)
    y.fill_(float("nan"))
    for _ in range(3):
        g.replay()
    torch.cuda.synchronize()
    assert torch.equal(y.view(torch.int32), eager.view(torch.int32))
    s1, s2 = torch.cuda.Stream(), torch.cuda.Stream()
    y1 = torch.full((m, n), float("nan"), device="cuda")
    y2 = torch.full((m, n), float("nan"), device="cuda")
    with torch.cuda.stream(s1):
        q4k.q4k_gemv(wt, xt, y1, m, n, k, stream=s1)
    with torch.cuda.stream(s2):
        q4k.q4k_gemv(wt, xt, y2, m, n, k, stream=s2)
    torch.cuda.synchronize()
    assert torch.equal(y1.view(torch.int32), eager.view(torch.int32))
    assert torch.equal(y2.view(torch.int32), eager.view(torch.int32))
    del g


@pytest.mark.parametrize("m,k,depth,cpi", [(2, 256, 8, 1), (2, 1792, 8, 1), (2, 6912, 6, 1), (2, 11264, 4, 1),
                                           (1, 7168, 6, 1), (3, 5632, 4, 1), (4, 3584, 6, 1)])
def test_i8_every_instantiation(q4k, m, k, depth, cpi):
    """One whole 128-row tile per CTA (N = 148 * 128) with the digit image
    growing with K: each ring depth / items-of-one-column variant of the
    kernel the launch rule picks, checked on the first and last tiles and
    sampled rows."""
    n = 148 * 128
    p = q4k.q4k_gemv_plan_for(m, n, k, 148)
    assert p["kernel"] == q4k.Q4K_KERNEL_I8 and p["depth"] == depth and p["slices"] == cpi, p
    w, x = q4k_synth.q4k_problem(n, k, m, k + m)
    y = gpu_gemv(q4k, w, x, n, k)
    rows = np.unique(np.concatenate([np.arange(128), np.arange(n - 128, n), sampled(n, 80, k)]))
    yref, a = oracle.gemv_rows(w, x, n, k, rows)
    assert_gemv_close(y[:, rows], yref, a, f"{n}x{k} m={m}")


def test_i8_no_fault_flags(q4k):
    assert q4k.q4k_device_fault_flags() == 0
