"""q4k_prefill_f16_noalloc, the prefill entry point for callers that cannot
allocate device memory (it keeps the fp16 activations in a fixed array inside
the library instead of a caller-provided scratch), against q4k_prefill_f16 on
the same inputs, through the C ABI, on a B200. Named to be collected last: it
must pass both alone in a fresh process and after every other test."""
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


def _problem(q4k, m, n, k, seed):
    w, _ = q4k_synth.q4k_problem(n, k, 1, seed)
    x = q4k_synth.x_vectors(k, m, seed + 1)
    w16 = torch.empty((n, k), dtype=torch.float16, device="cuda")
    q4k.q4k_dequant_f16(torch.from_numpy(w).cuda(), w16, n, k)
    return w, x, w16, torch.from_numpy(x).cuda()


def test_noalloc_matches_scratch_entry_point_two_calls(q4k):
    """Two calls in a row with different shapes (the second reuses the fixed
    array the first filled): each output matches q4k_prefill_f16's within the
    GEMM tolerance of the other prefill tests (k * 2^-23 * sum|w x| + 1e-6,
    against the oracle's exact sums of the fp16 products)."""
    for (m, n, k, seed) in [(512, 1024, 4096, 600), (300, 640, 2048, 610)]:
        w, x, w16, xt = _problem(q4k, m, n, k, seed)
        y_ref = torch.full((m, n), float("nan"), dtype=torch.float32, device="cuda")
        scratch = torch.empty(m * k * 2, dtype=torch.uint8, device="cuda")
        q4k.q4k_prefill_f16(w16, xt, scratch, y_ref, m, n, k)
        y = torch.full((m, n), float("nan"), dtype=torch.float32, device="cuda")
        q4k.q4k_prefill_f16_noalloc(w16, xt, y, m, n, k)
        torch.cuda.synchronize()
        yv, yr = y.cpu().numpy().astype(np.float64), y_ref.cpu().numpy().astype(np.float64)
        _, a = oracle.gemm_f16(oracle.dequant_f16(w, n, k), oracle.floats_to_half(x))
        tol = oracle.gemm_f16_tolerance(a, k)
        assert np.all(np.isfinite(yv))
        assert np.all(np.abs(yv - yr) <= tol), f"{m}x{n}x{k}: outside the GEMM tolerance"


def test_noalloc_refuses_beyond_its_scratch(q4k):
    """m * k above the fixed array is refused before anything is enqueued."""
    k = 4096
    m = q4k.Q4K_PREFILL_NOALLOC_MAX_ELEMS // k + 1
    n = 128
    w16 = torch.zeros((n, k), dtype=torch.float16, device="cuda")
    x = torch.zeros((m, k), dtype=torch.float32, device="cuda")
    y = torch.full((m, n), 5.0, dtype=torch.float32, device="cuda")
    st = q4k.q4k_prefill_f16_noalloc_status(w16.data_ptr(), x.data_ptr(), y.data_ptr(), m, n, k)
    assert st == q4k.Q4K_ERR_CAPACITY
    torch.cuda.synchronize()
    assert bool((y == 5.0).all())
    assert q4k.q4k_device_fault_flags() == 0
