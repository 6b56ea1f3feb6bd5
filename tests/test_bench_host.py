"""Host-side logic of bench.py without a GPU: byte accounting, and the
multi-rank aggregation run as two gloo ranks on the CPU."""
import os
import socket

import pytest

import bench


def test_algorithmic_bytes_per_unit():
    # state 64 KiB read + 64 KiB written, q/k share 256 B, v 256 B, out 512 B, gates 8 B
    assert bench.algorithmic_bytes_per_unit(128, 128, 2) == 132104
    # speculative T = 4: the state is read once per request and written once per token
    assert bench.algorithmic_bytes_per_unit(128, 128, 2, T=4) == 65536 / 4 + 65536 + 256 + 256 + 512 + 8


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out):
    import torch.distributed as dist

    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        elapsed = [10.0, 25.0][rank]  # rank 1 is the slow one
        out[rank] = (bench.max_over_ranks(elapsed, world), bench.job_throughput(1000.0, elapsed, world))
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_and_job_throughput_gloo():
    mp = pytest.importorskip("torch.multiprocessing")
    ctx = mp.get_context("spawn")
    with ctx.Manager() as m:
        out = m.dict()
        port = _free_port()
        procs = [ctx.Process(target=_rank_main, args=(r, 2, port, out)) for r in range(2)]
        for p in procs:
            p.start()
        for p in procs:
            p.join(120)
            assert p.exitcode == 0
        res = dict(out)
    for r in range(2):
        mx, thr = res[r]
        assert mx == 25.0
        assert thr == pytest.approx(2 * 1000.0 / 0.025)


def test_single_rank_aggregation_is_identity():
    assert bench.max_over_ranks(3.5, 1) == 3.5
    assert bench.job_throughput(100.0, 50.0, 1) == pytest.approx(2000.0)


def test_reference_arm_other_ranks_do_no_work(monkeypatch, capsys):
    monkeypatch.setenv("RANK", "1")
    called = []
    monkeypatch.setattr(bench, "oracle_time", lambda *a, **k: called.append(a) or 1.0)

    class A:
        steps, warmup, gpus = 3, 3, 2

    bench.run_reference(A())
    assert not called and capsys.readouterr().out == ""


def test_clock_sampler_summarises_the_timed_window():
    """Samples outside the timed window are ignored; reasons are the union of those inside."""
    s = bench.ClockSampler()
    rows = [(0.5, 1200.0, set()), (1.0, 1965.0, set()), (1.1, 1950.0, {"sw_power_cap"}), (1.2, 1965.0, set()),
            (3.0, 900.0, {"hw_slowdown"})]
    s.rows = [dict(ts=t, sm=sm, sm_max=1965.0, reasons=r) for t, sm, r in rows]
    s.mark(0.9, 1.3)
    c = s.stop()
    assert c["samples"] == 3 and c["window"] == "timed"
    assert c["sm_mhz"] == 1965.0 and c["sm_mhz_min"] == 1950.0 and c["sm_max_mhz"] == 1965.0
    assert c["reasons"] == ["sw_power_cap"]
    empty = bench.ClockSampler()
    assert empty.stop() is None
