"""The bench's multi-process path on CPU: two gloo ranks (replicas) agree on the slowest
rank's time and report the whole job's throughput from it."""
import os
import socket
import sys

import pytest

torch = pytest.importorskip("torch")
import torch.distributed as dist  # noqa: E402
import torch.multiprocessing as mp  # noqa: E402

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank(rank, world, port, local_ms, q):
    sys.path.insert(0, ROOT)
    import bench
    from datetime import timedelta
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=timedelta(seconds=60))
    try:
        ms = bench.max_over_ranks(dist, local_ms[rank], torch, device="cpu")
        dist.barrier()
        q.put((rank, ms, bench.job_throughput(world, 8192, 10, ms)))
    finally:
        dist.destroy_process_group()


def test_two_ranks_take_the_slowest_time_and_sum_the_work():
    world, port = 2, _free_port()
    local_ms = [120.0, 150.0]  # rank 1 is slower
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_rank, args=(r, world, port, local_ms, q)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
    assert all(p.exitcode == 0 for p in procs), [p.exitcode for p in procs]
    got = sorted(q.get(timeout=5) for _ in range(world))
    for rank, ms, value in got:
        assert ms == 150.0
        assert value == pytest.approx(2 * 8192 * 10 / 0.150)


def test_single_process_is_a_no_op():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.max_over_ranks(None, 12.5, torch) == 12.5
    assert bench.job_throughput(1, 8192, 10, 1000.0) == pytest.approx(81920.0)


def test_clock_summary_keeps_only_the_timed_window():
    import datetime
    sys.path.insert(0, ROOT)
    import bench
    t = datetime.datetime(2026, 1, 2, 3, 4, 5)

    def row(dt_ms, mhz, cap="Not Active", thermal="Not Active"):
        ts = (t + datetime.timedelta(milliseconds=dt_ms)).strftime("%Y/%m/%d %H:%M:%S.%f")[:-3]
        return f"{ts}, 0, {mhz}, 1965, 900.1, 0x0, Not Active, {thermal}, Not Active, {cap}"

    lines = [row(0, 1965), row(50, 1965, thermal="Active"),  # idle, before the window
             row(120, 1800, cap="Active"), row(170, 1830, cap="Active"), row(220, 1860),
             row(400, 1965)]  # after it
    got = bench.ClockSampler.summarize(lines, t + datetime.timedelta(milliseconds=100),
                                       t + datetime.timedelta(milliseconds=300))
    assert got["samples"] == 3 and got["window"] == "timed region"
    assert got["sm_mhz"] == 1830 and got["sm_max_mhz"] == 1965
    assert got["reasons"] == ["sw_power_cap"]  # the thermal row lies outside the window
    # no stamped row inside: every row, and the summary says so
    got = bench.ClockSampler.summarize(lines, t + datetime.timedelta(seconds=5), t + datetime.timedelta(seconds=6))
    assert got["window"] == "all samples" and got["samples"] == 6
    assert bench.ClockSampler.summarize([], None, None)["reasons"] == ["no samples"]


def _run_main(monkeypatch, capsys, argv, env):
    sys.path.insert(0, ROOT)
    import bench
    for k, v in env.items():
        monkeypatch.setenv(k, v)
    monkeypatch.setattr(sys, "argv", ["bench.py"] + argv)
    bench.main()
    return capsys.readouterr().out.strip()


def test_reference_arm_times_exactly_k_steps_of_the_oracle(monkeypatch, capsys):
    import json
    out = _run_main(monkeypatch, capsys, ["--impl", "reference", "--steps", "2", "--warmup", "3",
                                          "--oracle-tokens", "8"], {"WORLD_SIZE": "1", "RANK": "0"})
    line = json.loads(out.splitlines()[-1])
    assert line["impl"] == "reference" and line["steps"] == 2 and line["warmup"] == 3
    assert line["unit"] == "tokens/s" and line["higher_is_better"] is True and line["value"] > 0
    assert line["value"] == pytest.approx(8 / (line["ms_per_step"] * 1e-3), rel=1e-9)
    cb = line["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["value"] == line["value"] and cb["cores"] >= 1 and "8 tokens" in cb["sample"]
    assert line["e2e"] == {"value": line["value"], "unit": "tokens/s", "h2d_bytes_per_step": 0,
                           "d2h_bytes_per_step": 0}


def test_reference_arm_runs_on_rank_zero_only(monkeypatch, capsys):
    out = _run_main(monkeypatch, capsys, ["--impl", "reference", "--steps", "1", "--warmup", "3",
                                          "--oracle-tokens", "8"], {"WORLD_SIZE": "2", "RANK": "1"})
    assert out == ""


def test_reference_sample_fits_the_run():
    sys.path.insert(0, ROOT)
    import bench
    for k, w in [(1, 3), (3, 3), (10, 3), (50, 3), (1000, 3)]:
        n = bench.reference_tokens_per_step(k, w)
        assert 64 <= n <= bench.PREFILL_T and n % 64 == 0
        if n > 64:  # the whole run stays near the budget at the oracle's rate
            assert (k + w) * n / bench.ORACLE_EST_TOKENS_S <= bench.REF_BUDGET_S * 1.01
