"""The benchmark's multi-rank logic on CPU: world-size-2 gloo ranks (no GPU).

bench.py runs N independent replicas of the sweep ("replicas only": the
GEMV has no exchange step), one per GPU; its time is the slowest rank's (max
over ranks) and its value the bytes all ranks streamed over that time. The
reference arm runs on rank 0 only.
"""
import os
import socket

import pytest

torch = pytest.importorskip("torch")
import torch.distributed as dist  # noqa: E402
import torch.multiprocessing as mp  # noqa: E402

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _load_bench():
    import importlib.util
    spec = importlib.util.spec_from_file_location("bench_under_test", os.path.join(ROOT, "bench.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, times, out_q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    from datetime import timedelta
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=timedelta(seconds=60))
    try:
        bench = _load_bench()
        ms = bench.max_over_ranks(times[rank], world, torch.device("cpu"))
        value = bench.whole_job_gbs(world, 406_356_992, 10, ms)
        dist.barrier()
        out_q.put((rank, ms, value))
    finally:
        dist.destroy_process_group()


def test_two_rank_time_is_the_slowest_rank():
    world = 2
    times = [1.75, 2.5]              # ms: rank 1 is slower
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, times, q)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    got = sorted(q.get(timeout=10) for _ in range(world))
    for rank, ms, value in got:
        assert ms == 2.5
        assert value == pytest.approx(2 * 406_356_992 * 10 / 2.5e-3 / 1e9)


def test_single_rank_needs_no_process_group():
    bench = _load_bench()
    assert bench.max_over_ranks(3.0, 1, None) == 3.0
    assert bench.whole_job_gbs(1, 1_000_000_000, 2, 1000.0) == pytest.approx(2.0)


def test_reference_arm_runs_on_rank_zero_only(monkeypatch, capsys):
    bench = _load_bench()
    monkeypatch.setenv("RANK", "1")

    class Args:
        gpus, steps, warmup = 2, 1, 3
    assert bench.run_reference(Args()) is None
    assert capsys.readouterr().out == ""
