"""Parity of the tensor-core batched GEMV (q4k_gemv with m >= 3 vectors) with
the CPU oracle, on a B200.

Bound: |y_gpu - y_ref| <= 1e-4 * sum|w x| + 1e-6 per element (y_ref in double),
as for every q4k_gemv path. The cases here are the ones its number format and
its launch shape add: x is scaled per 256-element block by the block's largest
magnitude and split into base-128 digits (dynamic range inside a block, tiny,
huge, subnormal and zero blocks, non-finite values), vectors run in groups of
16 padded to 8 or 16, and CTAs own equal ranges of (128-row tile, superblock
column) items (several tiles per CTA, tiles cut between CTAs, a ragged last
tile).
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
    x = np.ascontiguousarray(x, np.float32).reshape(-1, k)
    m = x.shape[0]
    assert q4k.q4k_gemv_plan_for(m, n, k, 148)["kernel"] == q4k.Q4K_KERNEL_TC
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


@pytest.mark.parametrize("m", [3, 5, 8, 9, 15, 16, 17, 31, 32, 33, 64])
@pytest.mark.parametrize("n,k", [(130, 1024), (257, 2048), (1, 256)])
def test_tc_group_sizes(q4k, n, k, m):
    """Padding to 8 or 16 vectors, groups of 16, one- and two-tile matrices."""
    w, x = q4k_synth.q4k_problem(n, k, m, 3 * m + n)
    y = gpu_gemv(q4k, w, x, n, k)
    yref, a = oracle.gemv(w, x, n, k)
    assert_gemv_close(y, yref, a, f"{n}x{k} m={m}")


def test_tc_persistent_tiles_ragged(q4k):
    """More 128-row tiles than SMs (two or three per CTA) and a 77-row last tile."""
    n, k, m = 148 * 128 * 2 + 77, 512, 5
    w, x = q4k_synth.q4k_problem(n, k, m, 41)
    y = gpu_gemv(q4k, w, x, n, k)
    yref, a = oracle.gemv(w, x, n, k, nthreads=8)
    assert_gemv_close(y, yref, a, f"{n}x{k} m={m}")


@pytest.mark.parametrize("n,k", [(128, 8192), (3, 65536), (300, 1536), (1536, 1536)])
def test_tc_tiles_cut_between_ctas(q4k, n, k):
    """Tiles cut between CTAs: one tile over 32 CTAs (one superblock column
    each), one over all 148, and tiles of several pieces; the pieces are added
    in CTA order by whichever CTA finishes a tile last."""
    m = 5
    w, x = q4k_synth.q4k_problem(n, k, m, n + k)
    y = gpu_gemv(q4k, w, x, n, k)
    yref, a = oracle.gemv(w, x, n, k, nthreads=8)
    assert_gemv_close(y, yref, a, f"{n}x{k}")
    y2 = gpu_gemv(q4k, w, x, n, k)
    assert np.array_equal(y.view(np.uint32), y2.view(np.uint32)), "order of the piece sums"


def test_tc_block_dynamic_range(q4k):
    """Blocks scaled by 1e-30 and 1e30, a block of subnormals, an all-zero
    block, and a block whose largest value is 2^20 times its others (those are
    rounded at 2^-34 of the block's scale)."""
    n, k, m = 200, 2048, 4
    w, x = q4k_synth.q4k_problem(n, k, m, 77)
    x = x.reshape(m, k).copy()
    x[0, 0:256] *= np.float32(1e-30)
    x[1, 256:512] *= np.float32(1e30)
    x[2, 512:768] = (np.arange(256, dtype=np.float32) - 128) * np.float32(1e-43)
    x[3, 768:1024] = 0.0
    x[0, 1024 + 17] = np.float32(2.0 ** 20)
    x[1, 1280:1536] = np.float32(1.0)
    y = gpu_gemv(q4k, w, x, n, k)
    yref, a = oracle.gemv(w, x, n, k)
    assert_gemv_close(y, yref, a, "dynamic range")


def test_tc_unit_vectors_are_exact_columns(q4k):
    """x = e_t scales to 2^32 (one digit 16): y is d*sc*q - dmin*m formed
    exactly and rounded once, i.e. the f32 dequantised column, bit for bit."""
    n, k = 257, 2048
    w, _ = q4k_synth.q4k_problem(n, k, 1, 32)
    deq = oracle.dequant_f32(w, n, k).reshape(n, k)
    cols = np.arange(0, k, 37)[:48]
    x = np.zeros((len(cols), k), np.float32)
    x[np.arange(len(cols)), cols] = 1.0
    y = gpu_gemv(q4k, w, x, n, k)
    assert np.array_equal(y.view(np.uint32), deq[:, cols].T.copy().view(np.uint32))


def test_tc_non_finite_vector_is_nan(q4k):
    """An inf or NaN in a vector makes that vector's outputs NaN; the other
    vectors of the launch are unaffected."""
    n, k, m = 70, 1024, 4
    w, x = q4k_synth.q4k_problem(n, k, m, 5)
    x = x.reshape(m, k).copy()
    x[1, 300] = np.inf
    x[3, 1000] = np.nan
    y = gpu_gemv(q4k, w, x, n, k)
    assert np.isnan(y[1]).all() and np.isnan(y[3]).all()
    keep = [0, 2]
    yref, a = oracle.gemv(w, x[keep], n, k)
    assert_gemv_close(y[keep], yref, a, "finite vectors")


def test_tc_deterministic_and_rows_only(q4k):
    """Two calls give identical bits; nothing outside y's m x n floats is written."""
    n, k, m = 300, 1536, 6
    w, x = q4k_synth.q4k_problem(n, k, m, 9)
    wt, xt = dev(w), dev(x.reshape(m, k))
    guard = 64
    buf = torch.full((m * n + 2 * guard,), 7.0, dtype=torch.float32, device="cuda")
    y = buf[guard:guard + m * n]
    q4k.q4k_gemv(wt, xt, y, m, n, k)
    first = y.clone()
    q4k.q4k_gemv(wt, xt, y, m, n, k)
    torch.cuda.synchronize()
    assert torch.equal(first.view(torch.int32), y.view(torch.int32))
    assert (buf[:guard] == 7.0).all() and (buf[guard + m * n:] == 7.0).all()
    yref, a = oracle.gemv(w, x, n, k)
    assert_gemv_close(y.cpu().numpy().reshape(m, n), yref, a, "rows")


def test_tc_lm_head_sampled(q4k):
    """m = 5 on the 128256 x 4096 LM head: 16032 items over the CTAs, several
    tiles per CTA and a cut tile at most CTA boundaries; 40 sampled rows."""
    n, k, m = 128256, 4096, 5
    w, x = q4k_synth.q4k_problem(n, k, m, 8)
    y = gpu_gemv(q4k, w, x, n, k)
    rows = np.unique(np.concatenate([[0, 127, 128, n - 1], np.random.default_rng(3).integers(0, n, 36)]))
    yref, a = oracle.gemv_rows(w, x, n, k, rows)
    assert_gemv_close(y[:, rows], yref, a, "LM head m=5")


def test_tc_graph_capture_and_two_streams(q4k):
    """Calls captured in a CUDA graph (the call's stream-ordered workspace
    becomes graph memory nodes) replay to the eager result; calls on two
    streams at once (one workspace each) both match it."""
    n, k, m = 1000, 2048, 6
    w, x = q4k_synth.q4k_problem(n, k, m, 17)
    wt, xt = dev(w), dev(x.reshape(m, k))
    eager = torch.empty((m, n), dtype=torch.float32, device="cuda")
    q4k.q4k_gemv(wt, xt, eager, m, n, k)
    torch.cuda.synchronize()
    s = torch.cuda.Stream()
    ys = [torch.full((m, n), float("nan"), device="cuda") for _ in range(3)]
    with torch.cuda.stream(s):   # warm-up outside capture
        q4k.q4k_gemv(wt, xt, ys[0], m, n, k, stream=s)
    s.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=s):
        for y in ys:
            q4k.q4k_gemv(wt, xt, y, m, n, k, stream=s)
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
    y1 = torch.full((m, n), float("nan"), device="cuda")
    y2 = torch.full((m, n), float("nan"), device="cuda")
    torch.cuda.synchronize()
    for _ in range(5):
        q4k.q4k_gemv(wt, xt, y1, m, n, k, stream=s1)
        q4k.q4k_gemv(wt, xt, y2, m, n, k, stream=s2)
    torch.cuda.synchronize()
    assert torch.equal(y1.view(torch.int32), eager.view(torch.int32))
    assert torch.equal(y2.view(torch.int32), eager.view(torch.int32))
    yref, a = oracle.gemv(w, x, n, k)
    assert_gemv_close(eager.cpu().numpy(), yref, a, "eager")


def test_tc_no_fault_flags(q4k):
    assert q4k.q4k_device_fault_flags() == 0
