"""Parity of the prefill path (fp16 mirror, f32 -> fp16 convert, tcgen05 GEMM)
with the CPU oracle, through the C ABI, on a B200.

Mirror and convert: bit-exact (NaN compared as NaN). GEMM: against the exact
products of the fp16 operands summed in double (oracle.gemm_f16), within
oracle.gemm_f16_tolerance (k * 2^-23 * sum|w x| + 1e-6); where every partial
sum is an integer below 2^24 the f32 result must be exact."""
import os

import numpy as np
import pytest

import oracle
import q4k_synth

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


def bits16(t):
    return t.cpu().contiguous().view(torch.int16).numpy().view(np.uint16)


def assert_same_half(got, ref, what=""):
    gn = np.isnan(got.view(np.float16))
    rn = np.isnan(ref.view(np.float16))
    assert np.array_equal(gn, rn), f"{what}: NaN positions differ"
    bad = got[~gn] != ref[~rn]
    assert not bad.any(), f"{what}: {int(bad.sum())} binary16 values differ"


def gpu_gemm(q4k, w16, x16, m, n, k):
    y = torch.full((m, n), float("nan"), dtype=torch.float32, device="cuda")
    q4k.q4k_gemm_f16(dev(w16).view(torch.float16), dev(x16).view(torch.float16), y, m, n, k)
    torch.cuda.synchronize()
    return y.cpu().numpy()


def assert_gemm_close(y, yref, a, k, what=""):
    err = np.abs(y.astype(np.float64) - yref)
    tol = oracle.gemm_f16_tolerance(a, k)
    bad = ~(err <= tol)
    assert not bad.any(), (f"{what}: {int(bad.sum())} of {bad.size} out of tolerance; worst "
                           f"err/tol {np.nanmax(err / tol):.3g}")
    # typical error far inside the worst-case bound (a layout slip is not)
    rel = err / np.maximum(a, 1e-30)
    assert np.median(rel) < 2.0 ** -16, f"{what}: median relative error {np.median(rel):.3g}"


# --------------------------------------------------------------------------- mirror, convert

@pytest.mark.parametrize("n,k", [(1, 256), (33, 512), (256, 1024), (1536, 1536), (4096, 4096),
                                 (1000, 14336)])
def test_dequant_f16_bitexact(q4k, n, k):
    w, _ = q4k_synth.q4k_problem(n, k, 1, 500 + n)
    out = torch.empty((n, k), dtype=torch.float16, device="cuda")
    q4k.q4k_dequant_f16(dev(w), out, n, k)
    torch.cuda.synchronize()
    assert_same_half(bits16(out), oracle.dequant_f16(w, n, k), f"{n}x{k}")


def test_dequant_f16_raw_random_bytes(q4k):
    """Every byte random (d and dmin too): subnormals, infinities, NaNs, and
    values beyond binary16's range."""
    n, k = 64, 1024
    w = q4k_synth.random_bytes(n * (k // 256) * 144, 501)
    out = torch.empty((n, k), dtype=torch.float16, device="cuda")
    q4k.q4k_dequant_f16(dev(w), out, n, k)
    torch.cuda.synchronize()
    assert_same_half(bits16(out), oracle.dequant_f16(w, n, k), "raw bytes")


@pytest.mark.parametrize("count", [1, 3, 4, 5, 1001, 4096, (1 << 20) + 3])
def test_f32_to_f16_bitexact(q4k, count):
    rng = np.random.default_rng(count)
    x = rng.standard_normal(count).astype(np.float32) * np.float32(100.0)
    x[::7] = rng.integers(0, 2 ** 32, x[::7].size, dtype=np.uint64).astype(np.uint32).view(np.float32)
    out = torch.empty(count, dtype=torch.float16, device="cuda")
    q4k.q4k_f32_to_f16(dev(x), out, count)
    torch.cuda.synchronize()
    assert_same_half(bits16(out), oracle.floats_to_half(x), f"count {count}")


# --------------------------------------------------------------------------- GEMM

def small_int_operands(m, n, k, seed):
    """fp16 operands holding integers in [-8, 8]: every product and partial sum
    (|sum| <= 64 k < 2^24) is exact in f32, so the GEMM must be exact."""
    rng = np.random.default_rng(seed)
    w = rng.integers(-8, 9, (n, k)).astype(np.float16).view(np.uint16)
    x = rng.integers(-8, 9, (m, k)).astype(np.float16).view(np.uint16)
    return w, x


@pytest.mark.parametrize("m,n,k", [(1, 1, 64), (5, 7, 64), (128, 128, 256), (129, 130, 320),
                                   (256, 128, 1024), (300, 257, 512), (257, 384, 4096),
                                   (512, 256, 14336),
                                   # tile widths the launch picks on 148 SMs: 256, 128 and
                                   # 64 tokens per CTA, and ragged edges of each
                                   (512, 14336, 256), (512, 4096, 256), (512, 1024, 256),
                                   (509, 14300, 192), (500, 4000, 320), (511, 1000, 128)])
def test_gemm_f16_exact_on_integers(q4k, m, n, k):
    w16, x16 = small_int_operands(m, n, k, m * 7 + n)
    y = gpu_gemm(q4k, w16, x16, m, n, k)
    yref, _ = oracle.gemm_f16(w16, x16)
    assert np.array_equal(y.astype(np.float64), yref), \
        f"{m}x{n}x{k}: {int((y != yref).sum())} of {y.size} differ"


def test_gemm_f16_unit_vectors_give_columns(q4k):
    """x16 = rows of the identity: y[i][r] is w16[r][i] exactly."""
    n, k = 300, 1024
    w, _ = q4k_synth.q4k_problem(n, k, 1, 510)
    w16 = oracle.dequant_f16(w, n, k)
    m = k
    x16 = np.zeros((m, k), np.uint16)
    x16[np.arange(m), np.arange(k)] = 0x3C00
    y = gpu_gemm(q4k, w16, x16, m, n, k)
    assert np.array_equal(y.astype(np.float64), oracle.half_values(w16).T)


@pytest.mark.parametrize("m,n,k", [(1, 128, 256), (64, 1000, 1536), (200, 512, 4096),
                                   (512, 1024, 4096), (333, 640, 2048)])
def test_gemm_f16_mirror_of_q4k(q4k, m, n, k):
    """The whole prefill route on synthetic Q4_K weights: mirror, convert, GEMM."""
    w, _ = q4k_synth.q4k_problem(n, k, 1, 520 + m)
    x = q4k_synth.x_vectors(k, m, 521 + m)
    wt = dev(w)
    w16 = torch.empty((n, k), dtype=torch.float16, device="cuda")
    x16 = torch.empty((m, k), dtype=torch.float16, device="cuda")
    y = torch.full((m, n), float("nan"), dtype=torch.float32, device="cuda")
    q4k.q4k_dequant_f16(wt, w16, n, k)
    q4k.q4k_f32_to_f16(dev(x), x16, m * k)
    q4k.q4k_gemm_f16(w16, x16, y, m, n, k)
    torch.cuda.synchronize()
    w16o = oracle.dequant_f16(w, n, k)
    x16o = oracle.floats_to_half(x)
    assert_same_half(bits16(w16), w16o, "mirror")
    assert_same_half(bits16(x16), x16o, "activations")
    yref, a = oracle.gemm_f16(w16o, x16o)
    assert_gemm_close(y.cpu().numpy(), yref, a, k, f"{m}x{n}x{k}")


@pytest.mark.parametrize("n,k", [(4096, 4096), (1024, 4096), (14336, 4096), (4096, 14336)])
def test_prefill_8b_shapes_sampled(q4k, n, k):
    """The 8B-class projections at m = 512 tokens through q4k_prefill_f16 (one
    call: convert into the caller's scratch, then the GEMM); the scratch holds
    fp16(x) exactly, y equals q4k_gemm_f16's bit for bit, and sampled rows of W
    are checked against the oracle."""
    m = 512
    w, _ = q4k_synth.q4k_problem(n, k, 1, 530 + n + k)
    x = q4k_synth.x_vectors(k, m, 531)
    w16 = torch.empty((n, k), dtype=torch.float16, device="cuda")
    q4k.q4k_dequant_f16(dev(w), w16, n, k)
    xt = dev(x)
    scratch = torch.empty(m * k * 2, dtype=torch.uint8, device="cuda")
    y = torch.full((m, n), float("nan"), dtype=torch.float32, device="cuda")
    q4k.q4k_prefill_f16(w16, xt, scratch, y, m, n, k)
    y2 = torch.full((m, n), float("nan"), dtype=torch.float32, device="cuda")
    q4k.q4k_gemm_f16(w16, scratch.view(torch.float16).view(m, k), y2, m, n, k)
    torch.cuda.synchronize()
    x16o = oracle.floats_to_half(x)
    assert_same_half(scratch.cpu().numpy().view(np.uint16).reshape(m, k), x16o, "scratch")
    yg = y.cpu().numpy()
    assert np.array_equal(yg.view(np.uint32), y2.cpu().numpy().view(np.uint32))
    rng = np.random.default_rng(n + k)
    rows = np.unique(np.concatenate([[0, 127, 128, n - 1], rng.integers(0, n, 28)]))
    w16o = oracle.dequant_f16(w, n, k)
    yref, a = oracle.gemm_f16(w16o, x16o, rows=rows)
    assert_gemm_close(yg[:, rows], yref, a, k, f"{n}x{k} m={m}")


def test_gemm_offsets_and_stream(q4k):
    """Operands at 16-byte (not 256-byte) offsets, y inside a guard band, on a
    side stream: only y changes."""
    m, n, k = 70, 130, 256
    w16, x16 = small_int_operands(m, n, k, 540)
    wb = torch.zeros(n * k + 64, dtype=torch.float16, device="cuda")
    xb = torch.zeros(m * k + 64, dtype=torch.float16, device="cuda")
    wb[8:8 + n * k] = dev(w16).view(torch.float16).reshape(-1)
    xb[8:8 + m * k] = dev(x16).view(torch.float16).reshape(-1)
    yb = torch.full((m * n + 64,), 7.0, dtype=torch.float32, device="cuda")
    s = torch.cuda.Stream()
    with torch.cuda.stream(s):
        q4k.q4k_gemm_f16(wb.data_ptr() + 16, xb.data_ptr() + 16, yb.data_ptr() + 4 * 32,
                         m, n, k, stream=s)
    s.synchronize()
    yv = yb.cpu().numpy()
    assert (yv[:32] == 7.0).all() and (yv[32 + m * n:] == 7.0).all()
    yref, _ = oracle.gemm_f16(w16, x16)
    assert np.array_equal(yv[32:32 + m * n].reshape(m, n).astype(np.float64), yref)


def test_prefill_no_fault_flags(q4k):
    assert q4k.q4k_device_fault_flags() == 0
