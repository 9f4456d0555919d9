"""Parity of the CUDA path (through the C ABI) with the CPU oracle, on a B200.

GEMV: |y_gpu - y_ref| <= 1e-4 * sum|w x| + 1e-6 per element (y_ref in double).
Dequant: bit-exact f32 (NaN compared as NaN: its payload is not part of the
format's value).
"""
import os

import numpy as np
import pytest

import oracle
import q4k_synth
import special_blocks

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

NTHREADS = max(1, len(os.sched_getaffinity(0)))


@pytest.fixture(scope="module")
def q4k():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import gguf_quant_dequant_q4k_b200 as lib
    return lib


def dev(a):
    return torch.from_numpy(np.ascontiguousarray(a)).cuda()


def gpu_gemv(q4k, w, x, n, k, wt=None):
    x = np.ascontiguousarray(x, np.float32).reshape(-1, k)
    m = x.shape[0]
    wt = dev(w) if wt is None else wt
    xt = dev(x)
    y = torch.full((m, n), float("nan"), dtype=torch.float32, device="cuda")
    q4k.q4k_gemv(wt, xt, y, m, n, k)
    torch.cuda.synchronize()
    return y.cpu().numpy()


def gpu_dequant(q4k, w, n, k, wt=None):
    wt = dev(w) if wt is None else wt
    out = torch.full((n, k), float("nan"), dtype=torch.float32, device="cuda")
    q4k.q4k_dequant_f32(wt, out, n, k)
    torch.cuda.synchronize()
    return out


def assert_gemv_close(y, yref, a, what=""):
    err = np.abs(y.astype(np.float64) - yref)
    tol = oracle.tolerance(a)
    bad = ~(err <= tol)
    assert not bad.any(), (f"{what}: {bad.sum()} elements out of tolerance; worst "
                           f"err/tol={np.nanmax(err / tol):.3g}")


def assert_bitexact(got, ref, what=""):
    got = np.asarray(got, np.float32)
    ref = np.asarray(ref, np.float32)
    gn, rn = np.isnan(got), np.isnan(ref)
    assert np.array_equal(gn, rn), f"{what}: NaN positions differ"
    gb, rb = got[~gn].view(np.uint32), ref[~rn].view(np.uint32)
    bad = gb != rb
    assert not bad.any(), f"{what}: {bad.sum()} values differ bitwise"


# --------------------------------------------------------------------------- dequant

@pytest.mark.parametrize("n,k", [(1, 256), (3, 768), (33, 256), (256, 1024), (1536, 1536),
                                 (8960, 1536), (4096, 11008)])
def test_dequant_bitexact(q4k, n, k):
    w, _ = q4k_synth.q4k_problem(n, k, 1, q4k_synth.SEEDS.get((n, k), 100 + n))
    got = gpu_dequant(q4k, w, n, k).cpu().numpy()
    assert_bitexact(got, oracle.dequant_f32(w, n, k), f"{n}x{k}")


def test_dequant_raw_random_bytes(q4k):
    """Every byte random, d and dmin included: subnormals, infinities, NaNs."""
    n, k = 64, 1024
    w = q4k_synth.random_bytes(n * (k // 256) * 144, 21)
    assert_bitexact(gpu_dequant(q4k, w, n, k).cpu().numpy(), oracle.dequant_f32(w, n, k))


def test_dequant_lm_head_sampled_rows(q4k):
    n, k = 128256, 4096
    w, _ = q4k_synth.q4k_problem(n, k, 1, q4k_synth.SEEDS[(n, k)])
    out = gpu_dequant(q4k, w, n, k)
    rows = np.unique(np.concatenate([[0, 1, n - 2, n - 1],
                                     np.random.default_rng(3).integers(0, n, 60)]))
    got = out[torch.from_numpy(rows).cuda()].cpu().numpy()
    assert_bitexact(got, oracle.dequant_rows(w, n, k, rows))


# --------------------------------------------------------------------------- GEMV, m = 1

CONFIG_SHAPES = (q4k_synth.SHAPES_TINY + q4k_synth.SHAPES_1P5B + q4k_synth.SHAPES_7B
                 + q4k_synth.SHAPES_8B)


@pytest.mark.parametrize("n,k", CONFIG_SHAPES)
def test_gemv_config_shapes(q4k, n, k):
    w, x = q4k_synth.q4k_problem(n, k, 1, q4k_synth.SEEDS[(n, k)])
    y = gpu_gemv(q4k, w, x, n, k)
    yref, a = oracle.gemv(w, x, n, k, nthreads=NTHREADS)
    assert_gemv_close(y, yref, a, f"{n}x{k}")


@pytest.mark.parametrize("n,k", [(1, 256), (2, 256), (5, 512), (7, 768), (31, 1280),
                                 (33, 2304), (37, 8960), (129, 256), (1, 14336), (3, 11008),
                                 (97, 4352), (300, 3840), (149, 1024), (77, 1536), (40, 4096),
                                 (147, 20480), (1000, 20480), (64, 20736), (2, 30720), (5, 30976), (2, 32768),
                                 (1000, 28672), (150, 23040), (7, 20736)])
def test_gemv_ragged_shapes(q4k, n, k):
    w, x = q4k_synth.q4k_problem(n, k, 1, 1000 + n + k)
    y = gpu_gemv(q4k, w, x, n, k)
    yref, a = oracle.gemv(w, x, n, k)
    assert_gemv_close(y, yref, a, f"{n}x{k}")


# --------------------------------------------------------------------------- GEMV, m > 1

@pytest.mark.parametrize("m", range(1, 9))
@pytest.mark.parametrize("n,k", [(33, 512), (200, 1792)])
def test_gemv_every_m_small(q4k, n, k, m):
    w, x = q4k_synth.q4k_problem(n, k, m, 7 * m + n)
    y = gpu_gemv(q4k, w, x, n, k)
    yref, a = oracle.gemv(w, x, n, k)
    assert_gemv_close(y, yref, a, f"{n}x{k} m={m}")


@pytest.mark.parametrize("m", [1, 2, 4, 8])
@pytest.mark.parametrize("n,k", q4k_synth.SHAPES_MULTIVEC)
def test_gemv_multivector_shapes(q4k, n, k, m):
    w, x = q4k_synth.q4k_problem(n, k, m, q4k_synth.SEED_MULTIVEC[(n, k)])
    y = gpu_gemv(q4k, w, x, n, k)
    yref, a = oracle.gemv(w, x, n, k, nthreads=NTHREADS)
    assert_gemv_close(y, yref, a, f"{n}x{k} m={m}")


@pytest.mark.parametrize("n,k", [(75904, 256), (100000, 20480), (151936, 20480), (64, 28672)])
def test_gemv_tall_two_slices_sampled(q4k, n, k):
    """Very tall matrices (512 or more rows per CTA) that the integer
    tensor-core kernel does not take (K beyond its digit image, or too few
    superblock columns per CTA with whole tiles uneven) and K beyond 20480
    (one vector) run two quant slices per lane on the streaming kernel; the
    oracle checks sampled rows, including every CTA boundary region."""
    plan = q4k.q4k_gemv_plan_for(1, n, k, torch.cuda.get_device_properties(0).multi_processor_count)
    assert plan["slices"] == 2
    w, x = q4k_synth.q4k_problem(n, k, 1, 60 + n % 97)
    y = gpu_gemv(q4k, w, x, n, k)
    assert np.isfinite(y).all()
    rng = np.random.default_rng(n)
    per = -(-n // plan["grid"])
    edges = np.clip(np.arange(0, n, per)[:, None] + np.array([-1, 0, 1])[None, :], 0, n - 1)
    rows = np.unique(np.concatenate([edges.reshape(-1)[::7], rng.integers(0, n, 40), [0, n - 1]]))
    yref, a = oracle.gemv_rows(w, x, n, k, rows)
    assert_gemv_close(y[:, rows], yref, a, f"{n}x{k}")


@pytest.mark.parametrize("m,n,k", [(3, 40, 20736), (4, 33, 14336), (4, 300, 7680), (3, 300, 7936),
                                   (5, 77, 15616), (1, 9, 40960), (2, 17, 33024), (1, 4096, 61440),
                                   (7, 150, 11008), (4, 1, 14336), (3, 5, 8192)])
def test_gemv_k_chunks_and_vector_groups(q4k, m, n, k):
    """K beyond one team: one or two vectors run as K-chunks of strided row
    segments on the streaming kernel, later chunks adding into y (one vector
    on a matrix with enough superblock columns per SM, 4096 x 61440, runs on
    the integer tensor-core kernel instead); three or more run on the
    tensor-core kernel, which takes any K; y starts as NaN, so the first
    launch must overwrite it."""
    plan = q4k.q4k_gemv_plan_for(m, n, k, torch.cuda.get_device_properties(0).multi_processor_count)
    expected = (q4k.Q4K_KERNEL_I8 if (m, n, k) == (1, 4096, 61440) else q4k.Q4K_KERNEL_STREAM) if m <= 2 \
        else q4k.Q4K_KERNEL_TC
    assert plan["kernel"] == expected
    w, x = q4k_synth.q4k_problem(n, k, m, 70 + m + n)
    y = gpu_gemv(q4k, w, x, n, k)
    if n * k <= 4096 * 61440 // 8:
        yref, a = oracle.gemv(w, x, n, k, nthreads=NTHREADS)
        assert_gemv_close(y, yref, a, f"{m}x{n}x{k}")
    else:
        rows = np.unique(np.concatenate([[0, n - 1], np.random.default_rng(n).integers(0, n, 30)]))
        yref, a = oracle.gemv_rows(w, x, n, k, rows)
        assert_gemv_close(y[:, rows], yref, a, f"{m}x{n}x{k}")


@pytest.mark.parametrize("m", [9, 12, 16, 17, 32, 64])
@pytest.mark.parametrize("n,k", [(33, 512), (200, 1792), (40, 20736)])
def test_gemv_batches_beyond_eight(q4k, n, k, m):
    """m > 8: vector tiles (pairs on the streaming kernel; eights on the general
    kernel for K = 20736)."""
    w, x = q4k_synth.q4k_problem(n, k, m, 11 * m + n)
    y = gpu_gemv(q4k, w, x, n, k)
    yref, a = oracle.gemv(w, x, n, k)
    assert_gemv_close(y, yref, a, f"{n}x{k} m={m}")


@pytest.mark.parametrize("m", [16, 32])
@pytest.mark.parametrize("n,k", q4k_synth.SHAPES_MULTIVEC)
def test_gemv_batched_multivector_shapes_sampled(q4k, n, k, m):
    """m = 16 and 32 on the multi-vector shapes; the oracle checks 24 sampled rows."""
    w, x = q4k_synth.q4k_problem(n, k, m, q4k_synth.SEED_MULTIVEC[(n, k)] + m)
    y = gpu_gemv(q4k, w, x, n, k)
    rng = np.random.default_rng(m)
    rows = np.unique(np.concatenate([[0, n - 1], rng.integers(0, n, 22)]))
    yref, a = oracle.gemv_rows(w, x, n, k, rows)
    assert_gemv_close(y[:, rows], yref, a, f"{n}x{k} m={m}")


def test_gemv_32_layer_sweep_sampled(q4k):
    """All 224 projections of the 32-layer 8B-class decode sweep, each layer's
    weights seeded independently; the oracle checks 8 sampled rows of each."""
    rng = np.random.default_rng(5)
    for layer in range(32):
        for proj, (n, k) in enumerate(q4k_synth.LAYER_8B):
            w, x = q4k_synth.q4k_problem(n, k, 1, q4k_synth.layer_seed(layer, proj))
            y = gpu_gemv(q4k, w, x, n, k)
            assert np.isfinite(y).all()
            rows = np.unique(np.concatenate([[0, n - 1], rng.integers(0, n, 6)]))
            yref, a = oracle.gemv_rows(w, x, n, k, rows)
            assert_gemv_close(y[:, rows], yref, a, f"layer {layer} proj {proj}")


# --------------------------------------------------------------------------- special inputs

def test_gemv_zero_vector_gives_exact_zero(q4k):
    n, k = 300, 4096
    w, _ = q4k_synth.q4k_problem(n, k, 1, 31)
    y = gpu_gemv(q4k, w, np.zeros((1, k), np.float32), n, k)
    assert (y == 0).all()


def test_gemv_unit_vectors_give_columns(q4k):
    n, k = 257, 2048
    w, _ = q4k_synth.q4k_problem(n, k, 1, 32)
    deq = oracle.dequant_f32(w, n, k)
    cols = [0, 31, 32, 63, 64, 255, 256, 1000, 2047]
    x = np.zeros((len(cols), k), np.float32)
    for i, c in enumerate(cols[:8]):
        x[i, c] = 1.0
    y = gpu_gemv(q4k, w, x[:8], n, k)
    for i, c in enumerate(cols[:8]):
        assert_gemv_close(y[i], deq[:, c].astype(np.float64), np.abs(deq[:, c]).astype(np.float64),
                          f"column {c}")


def _gpu_columns(q4k, wt, n, k, cols, m):
    """y for x = e_c, c in `cols`, as calls of m vectors each (the last call may
    hold fewer). Returns (len(cols), n)."""
    cols = np.asarray(cols)
    eye = torch.zeros((len(cols), k), dtype=torch.float32, device="cuda")
    eye[torch.arange(len(cols), device="cuda"), torch.from_numpy(cols).cuda()] = 1.0
    y = torch.full((len(cols), n), float("nan"), dtype=torch.float32, device="cuda")
    for i0 in range(0, len(cols), m):
        mi = min(m, len(cols) - i0)
        q4k.q4k_gemv(wt, eye[i0:i0 + mi], y[i0:i0 + mi], mi, n, k)
    torch.cuda.synchronize()
    return y.cpu().numpy()


def _assert_columns(y, deq, cols, what):
    ref = deq[:, cols].T.astype(np.float64)
    assert_gemv_close(y, ref, np.abs(ref), what)


@pytest.mark.parametrize("m", [1, 2, 64])
def test_gemv_unit_vectors_every_column(q4k, m):
    """x = e_c for every column c of a 257 x 2048 matrix: y must be column c of
    the dequantised matrix within 1e-4 |w| + 1e-6 per element. m = 1 runs the
    one-vector kernel, m = 2 and 64 the two-vector kernel (64 = 32 pairs)."""
    n, k = 257, 2048
    w, _ = q4k_synth.q4k_problem(n, k, 1, 32)
    deq = oracle.dequant_f32(w, n, k)
    cols = np.arange(k)
    y = _gpu_columns(q4k, dev(w), n, k, cols, m)
    _assert_columns(y, deq, cols, f"every column, m={m}")


@pytest.mark.parametrize("n,k", [(33, 20736), (75904, 256)])
def test_gemv_unit_vectors_every_column_two_slices(q4k, n, k):
    """The two-slice one-vector kernel (K beyond 20480, or 512+ rows per CTA),
    x = e_c for every column."""
    plan = q4k.q4k_gemv_plan_for(1, n, k, torch.cuda.get_device_properties(0).multi_processor_count)
    assert plan["slices"] == 2
    w, _ = q4k_synth.q4k_problem(n, k, 1, 36)
    deq = oracle.dequant_f32(w, n, k)
    cols = np.arange(k)
    y = _gpu_columns(q4k, dev(w), n, k, cols, 1)
    _assert_columns(y, deq, cols, f"every column, {n}x{k}")


@pytest.mark.parametrize("m", [1, 2, 3])
@pytest.mark.parametrize("n,k", [(40, 4096), (7, 14336), (300, 1536), (33, 20736)])
def test_gemv_zero_quant_blocks(q4k, n, k, m):
    """All-zero quants (weights exactly -dmin*m_j) with a large d*sc: y = W 1
    and y = W x for x ~ N(0,1) within the per-element bound."""
    w = special_blocks.zero_quant_matrix(n, k)
    deq = oracle.dequant_f32(w, n, k)
    assert (deq == np.float32(-float(np.uint16(0x1438).view(np.float16)))).all()
    x = np.ones((m, k), np.float32)
    x[1:] = q4k_synth.x_vectors(k, m - 1, 61 + m)
    y = gpu_gemv(q4k, w, x, n, k)
    yref, a = oracle.gemv(w, x, n, k)
    assert_gemv_close(y, yref, a, f"zero quants {n}x{k} m={m}")


@pytest.mark.parametrize("m", [1, 2, 3])
@pytest.mark.parametrize("n,k", [(40, 4096), (5, 14336), (149, 1024), (20, 20736)])
def test_gemv_near_cancelling_blocks(q4k, n, k, m):
    """Weights that nearly cancel with d != dmin (so B_j's rounding is not
    exact), against all-ones and N(0,1) activations."""
    w = special_blocks.near_cancelling_matrix(n, k, 62 + n)
    x = np.ones((m, k), np.float32)
    x[1:] = 10 * q4k_synth.x_vectors(k, m - 1, 63 + m)
    y = gpu_gemv(q4k, w, x, n, k)
    yref, a = oracle.gemv(w, x, n, k)
    assert_gemv_close(y, yref, a, f"near-cancelling {n}x{k} m={m}")


def test_gemv_near_cancelling_every_column(q4k):
    n, k = 65, 2048
    w = special_blocks.near_cancelling_matrix(n, k, 64)
    deq = oracle.dequant_f32(w, n, k)
    wt = dev(w)
    cols = np.arange(k)
    for m in (1, 2):
        _assert_columns(_gpu_columns(q4k, wt, n, k, cols, m), deq, cols,
                        f"near-cancelling columns m={m}")


def _cancelling_block():
    # sc_j = 4, m_j = 60, every q = 15, d = dmin  =>  every weight is exactly 0
    S = np.array([4, 4, 4, 4, 60 | 0xC0, 60 | 0xC0, 60 | 0xC0, 60 | 0xC0,
                  0xC4, 0xC4, 0xC4, 0xC4], np.uint8)
    b = np.zeros(144, np.uint8)
    b[0:2] = b[2:4] = np.array([0x66, 0x2E], np.uint8)   # binary16 0x2E66, about 0.1
    b[4:16] = S
    b[16:] = 0xFF
    return b


def test_gemv_cancelling_blocks(q4k):
    """Rows whose weights are all exactly 0 by cancellation (d*sc*q == dmin*m):
    the contract's bound there is the 1e-6 absolute floor."""
    n, k = 40, 4096
    w, x = q4k_synth.q4k_problem(n, k, 2, 33)
    sb = w.reshape(n, k // 256, 144)
    sb[::3] = _cancelling_block()          # every third row cancels exactly
    w = sb.reshape(-1)
    yref, a = oracle.gemv(w, x, n, k)
    assert (yref[:, ::3] == 0).all()
    y = gpu_gemv(q4k, w, x * 10, n, k)      # large activations stress the floor
    yref, a = oracle.gemv(w, x * 10, n, k)
    assert_gemv_close(y, yref, a, "cancelling")


def test_gemv_deterministic(q4k):
    n, k = 4096, 11008
    w, x = q4k_synth.q4k_problem(n, k, 3, 34)
    wt = dev(w)
    y1 = gpu_gemv(q4k, w, x, n, k, wt=wt)
    y2 = gpu_gemv(q4k, w, x, n, k, wt=wt)
    assert np.array_equal(y1.view(np.uint32), y2.view(np.uint32))


def test_gemv_offsets_guard_band_and_stream(q4k):
    """W at a 16-byte (not 256-byte) offset inside a larger buffer, y with guard
    elements around it, launched on a side stream: only y[0:m*n] changes."""
    n, k, m = 77, 1536, 3
    w, x = q4k_synth.q4k_problem(n, k, m, 35)
    wbuf = torch.zeros(w.size + 64, dtype=torch.uint8, device="cuda")
    wbuf[16:16 + w.size] = dev(w)
    xbuf = torch.zeros(m * k + 8, dtype=torch.float32, device="cuda")
    xbuf[4:4 + m * k] = dev(x.reshape(-1))
    ybuf = torch.full((m * n + 64,), 7.0, dtype=torch.float32, device="cuda")
    s = torch.cuda.Stream()
    with torch.cuda.stream(s):
        q4k.q4k_gemv(wbuf.data_ptr() + 16, xbuf.data_ptr() + 16, ybuf.data_ptr() + 4 * 32,
                     m, n, k, stream=s)
    s.synchronize()
    yb = ybuf.cpu().numpy()
    assert (yb[:32] == 7.0).all() and (yb[32 + m * n:] == 7.0).all()
    yref, a = oracle.gemv(w, x, n, k)
    assert_gemv_close(yb[32:32 + m * n].reshape(m, n), yref, a, "offsets")


def test_invalid_arguments_on_gpu_enqueue_nothing(q4k):
    n, k = 16, 512
    wt = torch.zeros(q4k.q4k_weight_bytes(n, k), dtype=torch.uint8, device="cuda")
    xt = torch.zeros(k, dtype=torch.float32, device="cuda")
    y = torch.full((n,), 3.0, device="cuda")
    assert q4k.q4k_gemv_status(wt, xt, y, 65, n, k) == q4k.Q4K_ERR_UNSUPPORTED_M
    # x and y hold one vector: the binding refuses a tensor too small for 9;
    # through raw addresses the library finds y overlapping x
    with pytest.raises(ValueError):
        q4k.q4k_gemv_status(wt, xt, y, 9, n, k)
    assert (q4k.q4k_gemv_status(wt.data_ptr(), xt.data_ptr(), y.data_ptr(), 9, n, k)
            == q4k.Q4K_ERR_OVERLAP)
    with pytest.raises(ValueError):   # weights short of n*(k/256)*144 bytes
        q4k.q4k_gemv_status(wt[:-16], xt, y, 1, n, k)
    with pytest.raises(ValueError):   # a strided view is not a dense row-major buffer
        q4k.q4k_gemv_status(wt, torch.zeros(2 * k, device="cuda")[::2], y, 1, n, k)
    with pytest.raises(ValueError):   # dequant output too small
        q4k.q4k_dequant_f32_status(wt, torch.zeros(n * k - 1, device="cuda"), n, k)
    assert q4k.q4k_gemv_status(wt.data_ptr() + 8, xt, y, 1, n, k) == q4k.Q4K_ERR_ALIGN
    assert q4k.q4k_gemv_status(wt, xt, y, 1, n, 500) == q4k.Q4K_ERR_SHAPE
    torch.cuda.synchronize()
    assert (y == 3.0).all()


@pytest.mark.parametrize("n,k", [(149, 1024), (40, 4096), (1000, 20480)])
def test_gemv_two_vectors_team_split(q4k, n, k):
    w, x = q4k_synth.q4k_problem(n, k, 2, 40 + n)
    y = gpu_gemv(q4k, w, x, n, k)
    yref, a = oracle.gemv(w, x, n, k)
    assert_gemv_close(y, yref, a, f"{n}x{k} m=2")


@pytest.mark.parametrize("m", [1, 2])
@pytest.mark.parametrize("n,k", [(1, 14336), (3, 8960), (7, 11008), (5, 8192), (1, 4096),
                                 (2, 1536), (8, 14336), (16, 8960), (40, 4096), (100, 2048)])
def test_gemv_small_n_cluster_split(q4k, n, k, m):
    """Small N: for N < 8 and K >= 8192 rows are split across the two CTAs of a
    thread-block cluster (split-K) and finished through distributed shared
    memory; the other shapes run one CTA per row."""
    plan = q4k.q4k_gemv_plan_for(m, n, k, torch.cuda.get_device_properties(0).multi_processor_count)
    w, x = q4k_synth.q4k_problem(n, k, m, 50 + n + m)
    y = gpu_gemv(q4k, w, x, n, k)
    yref, a = oracle.gemv(w, x, n, k)
    assert_gemv_close(y, yref, a, f"{n}x{k} m={m} cluster={plan['cluster']}")


@pytest.mark.parametrize("m,n,k", [(1, 1536, 1536), (2, 4096, 4096), (1, 64, 61696), (1, 148 * 128, 512),
                                   (1, 4096, 14336), (2, 11008, 4096), (4, 11008, 4096), (8, 300, 2048)])
def test_gemv_x_ready_same_bits(q4k, m, n, k):
    """Q4K_GEMV_X_READY (x read before the preceding kernel finishes) gives
    the plain call's bits on every path: streaming (one and two vectors,
    K-chunks), integer kernel (whole and cut tiles, two and four vectors),
    and the batched kernel, which ignores it."""
    w, x = q4k_synth.q4k_problem(n, k, m, 90 + m + n % 97)
    wt, xt = dev(w), dev(np.asarray(x, np.float32).reshape(m, k))
    y0 = torch.full((m, n), float("nan"), device="cuda")
    y1 = torch.full((m, n), float("nan"), device="cuda")
    q4k.q4k_gemv(wt, xt, y0, m, n, k)
    q4k.q4k_gemv(wt, xt, y1, m, n, k, x_ready=True)
    torch.cuda.synchronize()
    assert torch.equal(y0.view(torch.int32), y1.view(torch.int32))
    rows = np.unique(np.concatenate([[0, n - 1], np.random.default_rng(n).integers(0, n, 40)]))
    yref, a = oracle.gemv_rows(w, x, n, k, rows)
    assert_gemv_close(y1.cpu().numpy()[:, rows], yref, a, f"x_ready {m}x{n}x{k}")


def test_gemv_x_ready_chain(q4k):
    """A chain on one stream, eager and in a CUDA graph: q = Wq x; k = Wk x
    and v = Wv x flagged (x is not written by the pending work); h = Wo q
    unflagged (q is). Every output matches the oracle."""
    d = 2048
    x = q4k_synth.x_vectors(d, 1, 5)
    mats = [q4k_synth.q4k_problem(d, d, 1, 60 + i)[0] for i in range(4)]
    wq, wk, wv, wo = (dev(w) for w in mats)
    xt = dev(x.reshape(1, d))
    outs = [torch.full((1, d), float("nan"), device="cuda") for _ in range(4)]
    s = torch.cuda.Stream()

    def chain():
        q4k.q4k_gemv(wq, xt, outs[0], 1, d, d, stream=s)
        q4k.q4k_gemv(wk, xt, outs[1], 1, d, d, stream=s, x_ready=True)
        q4k.q4k_gemv(wv, xt, outs[2], 1, d, d, stream=s, x_ready=True)
        q4k.q4k_gemv(wo, outs[0], outs[3], 1, d, d, stream=s)

    def check():
        torch.cuda.synchronize()
        got = [o.cpu().numpy() for o in outs]
        for i, w in enumerate(mats[:3]):
            yref, a = oracle.gemv(w, x, d, d)
            assert_gemv_close(got[i], yref, a, f"projection {i}")
        yref, a = oracle.gemv(mats[3], got[0], d, d)
        assert_gemv_close(got[3], yref, a, "dependent projection")

    with torch.cuda.stream(s):
        chain()
    check()
    for o in outs:
        o.fill_(float("nan"))
    s.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=s):
        chain()
    for o in outs:
        o.fill_(float("nan"))
    torch.cuda.synchronize()
    g.replay()
    check()
    del g


def test_no_kernel_fault_flags(q4k):
    """No bounded wait on a bulk copy gave up during any of the runs above."""
    assert q4k.q4k_device_fault_flags() == 0
