"""Parity of the fused gate/up SwiGLU GEMV (through the C ABI) with the CPU
oracle (g, u by the oracle GEMV in double, then silu(g) * u in double), on a
B200, within oracle.swiglu_tolerance."""
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


def problem(n, k, m, seed):
    wg, x = q4k_synth.q4k_problem(n, k, m, seed)
    wu, _ = q4k_synth.q4k_problem(n, k, 1, seed + 1)
    return wg, wu, x


def gpu_swiglu(q4k, wg, wu, x, n, k):
    x = np.ascontiguousarray(x, np.float32).reshape(-1, k)
    m = x.shape[0]
    y = torch.full((m, n), float("nan"), dtype=torch.float32, device="cuda")
    q4k.q4k_gemv_swiglu(torch.from_numpy(wg).cuda(), torch.from_numpy(wu).cuda(),
                        torch.from_numpy(x).cuda(), y, m, n, k)
    torch.cuda.synchronize()
    return y.cpu().numpy()


def assert_swiglu_close(y, wg, wu, x, n, k, what, rows=None):
    if rows is None:
        ref, g, u, a_g, a_u = oracle.swiglu_gemv(wg, wu, x, n, k, nthreads=NTHREADS)
    else:
        g, a_g = oracle.gemv_rows(wg, x, n, k, rows)
        u, a_u = oracle.gemv_rows(wu, x, n, k, rows)
        ref = g / (1.0 + np.exp(-g)) * u
        y = y[:, rows]
    tol = oracle.swiglu_tolerance(g, u, a_g, a_u, ref)
    err = np.abs(y.astype(np.float64) - ref)
    bad = ~(err <= tol)
    assert not bad.any(), f"{what}: {bad.sum()} out of tolerance, worst {np.nanmax(err / tol):.3g}"


@pytest.mark.parametrize("m", [1, 2, 3])
@pytest.mark.parametrize("n,k", [(1, 256), (3, 4096), (7, 14336), (149, 1024), (300, 3840),
                                 (1000, 2048), (64, 20736)])
def test_swiglu_matches_oracle(q4k, n, k, m):
    wg, wu, x = problem(n, k, m, 300 + n + m)
    y = gpu_swiglu(q4k, wg, wu, x, n, k)
    assert_swiglu_close(y, wg, wu, x, n, k, f"{n}x{k} m={m}")


@pytest.mark.parametrize("m", [1, 2, 8])
def test_swiglu_ffn_shape(q4k, m):
    """The 8B-class FFN gate/up shape, 14336 x 4096, all rows."""
    n, k = 14336, 4096
    wg, wu, x = problem(n, k, m, 310 + m)
    y = gpu_swiglu(q4k, wg, wu, x, n, k)
    assert_swiglu_close(y, wg, wu, x, n, k, f"FFN m={m}")


def test_swiglu_7b_ffn_sampled(q4k):
    n, k = 11008, 4096
    wg, wu, x = problem(n, k, 1, 320)
    y = gpu_swiglu(q4k, wg, wu, x, n, k)
    rows = np.unique(np.concatenate([[0, n - 1], np.random.default_rng(1).integers(0, n, 40)]))
    assert_swiglu_close(y, wg, wu, x, n, k, "7B FFN", rows=rows)


def test_swiglu_batches_beyond_eight(q4k):
    n, k = 200, 1792
    wg, wu, x = problem(n, k, 12, 330)
    y = gpu_swiglu(q4k, wg, wu, x, n, k)
    assert_swiglu_close(y, wg, wu, x, n, k, "m=12")


def test_swiglu_same_matrix_and_zero_vector(q4k):
    """gate == up (one buffer passed twice) and x = 0 (y = silu(0) * 0 = 0)."""
    n, k = 500, 4096
    wg, _, x = problem(n, k, 1, 340)
    wt = torch.from_numpy(wg).cuda()
    y = torch.full((1, n), float("nan"), dtype=torch.float32, device="cuda")
    q4k.q4k_gemv_swiglu(wt, wt, torch.from_numpy(x).cuda(), y, 1, n, k)
    torch.cuda.synchronize()
    assert_swiglu_close(y.cpu().numpy(), wg, wg, x, n, k, "gate == up")
    q4k.q4k_gemv_swiglu(wt, wt, torch.zeros((1, k), device="cuda"), y, 1, n, k)
    torch.cuda.synchronize()
    assert not y.cpu().numpy().any()


def test_swiglu_matches_separate_gemvs(q4k):
    """The fused call against two q4k_gemv calls and the same f32 epilogue
    written with torch: the GEMV sums differ only in rounding order."""
    n, k = 4096, 4096
    wg, wu, x = problem(n, k, 1, 350)
    y = gpu_swiglu(q4k, wg, wu, x, n, k)
    g = torch.empty((1, n), device="cuda")
    u = torch.empty((1, n), device="cuda")
    xt = torch.from_numpy(x).cuda()
    q4k.q4k_gemv(torch.from_numpy(wg).cuda(), xt, g, 1, n, k)
    q4k.q4k_gemv(torch.from_numpy(wu).cuda(), xt, u, 1, n, k)
    sep = (g / (1 + torch.exp(-g)) * u).cpu().numpy().astype(np.float64)
    ref, go, uo, a_g, a_u = oracle.swiglu_gemv(wg, wu, x, n, k, nthreads=NTHREADS)
    tol = oracle.swiglu_tolerance(go, uo, a_g, a_u, ref)
    assert np.all(np.abs(y - sep) <= 2 * tol)    # both within tol of the reference
    assert q4k.q4k_device_fault_flags() == 0


def _swiglu_columns(q4k, wg, wu, n, k, m):
    """y for x = e_c for every column c, m vectors per call."""
    eye = torch.eye(k, dtype=torch.float32, device="cuda")
    y = torch.full((k, n), float("nan"), dtype=torch.float32, device="cuda")
    gt, ut = torch.from_numpy(wg).cuda(), torch.from_numpy(wu).cuda()
    for i0 in range(0, k, m):
        mi = min(m, k - i0)
        q4k.q4k_gemv_swiglu(gt, ut, eye[i0:i0 + mi], y[i0:i0 + mi], mi, n, k)
    torch.cuda.synchronize()
    return y.cpu().numpy()


@pytest.mark.parametrize("m", [1, 2, 64])
def test_swiglu_unit_vectors_every_column(q4k, m):
    """x = e_c for every column of a 257 x 2048 gate (the seed-32 matrix) and
    an up matrix: y = silu(gate column) * (up column) within the bound."""
    n, k = 257, 2048
    wg, _ = q4k_synth.q4k_problem(n, k, 1, 32)
    wu, _ = q4k_synth.q4k_problem(n, k, 1, 37)
    y = _swiglu_columns(q4k, wg, wu, n, k, m)
    x = np.eye(k, dtype=np.float32)
    assert_swiglu_close(y, wg, wu, x, n, k, f"every column m={m}")


@pytest.mark.parametrize("m", [1, 2])
@pytest.mark.parametrize("n,k", [(40, 4096), (300, 1536)])
def test_swiglu_zero_quant_and_near_cancelling(q4k, n, k, m):
    """Gate of all-zero-quant blocks (weights exactly -dmin*m_j) and up of
    near-cancelling blocks, and the other way round, with x = 1 and N(0,1)."""
    wz = special_blocks.zero_quant_matrix(n, k)
    wc = special_blocks.near_cancelling_matrix(n, k, 70 + n)
    x = np.ones((m, k), np.float32)
    x[1:] = q4k_synth.x_vectors(k, m - 1, 71 + m)
    for wg, wu, what in ((wz, wc, "zero/near"), (wc, wz, "near/zero")):
        y = gpu_swiglu(q4k, wg, wu, x, n, k)
        assert_swiglu_close(y, wg, wu, x, n, k, f"{what} {n}x{k} m={m}")


def test_swiglu_near_cancelling_every_column(q4k):
    n, k = 65, 2048
    wg = special_blocks.near_cancelling_matrix(n, k, 72)
    wu = special_blocks.zero_quant_matrix(n, k)
    x = np.eye(k, dtype=np.float32)
    for m in (1, 2):
        y = _swiglu_columns(q4k, wg, wu, n, k, m)
        assert_swiglu_close(y, wg, wu, x, n, k, f"near-cancelling columns m={m}")
