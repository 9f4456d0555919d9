"""Failure detection on a B200 without a GPU fault: a kernel's bounded wait on
an mbarrier phase that nothing completes gives up, raises the copy-timeout
flag and returns; the host reads the flag and the context stays usable."""
import time

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


def test_bounded_wait_gives_up_and_reports(q4k):
    assert q4k.q4k_device_fault_flags() == 0
    t0 = time.perf_counter()
    q4k.q4k_selftest_wait_timeout()
    torch.cuda.synchronize()
    elapsed = time.perf_counter() - t0
    assert elapsed < 30.0
    assert q4k.q4k_device_fault_flags() == q4k.Q4K_FAULT_COPY_TIMEOUT
    assert q4k.q4k_device_fault_flags() == 0          # read clears
    # the context is still usable: a GEMV right after is correct
    n, k = 300, 4096
    w, x = q4k_synth.q4k_problem(n, k, 1, 77)
    y = torch.empty((1, n), device="cuda")
    q4k.q4k_gemv(torch.from_numpy(w).cuda(), torch.from_numpy(x).cuda(), y, 1, n, k)
    torch.cuda.synchronize()
    yref, a = oracle.gemv(w, x, n, k)
    assert np.all(np.abs(y.cpu().numpy() - yref) <= oracle.tolerance(a))
    assert q4k.q4k_device_fault_flags() == 0
