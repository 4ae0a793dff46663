"""bench.py's host plumbing on CPU: its multi-process reductions on gloo ranks
(world size 2) and its clock sampler against a fake NVML.

The expert layer runs as independent replicas, one per GPU, with no
collective on the data path; bench.py only reduces its timings (max over
ranks) and unit counts (sum over ranks), and lets rank 0 alone run the
reference arm.  These helpers are exercised here with two gloo ranks.
"""
import os
import socket
import sys

import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    sys.path.insert(0, ROOT)
    import bench
    r, w, local, pg = bench.dist_setup(world)
    try:
        assert (r, w, local) == (rank, world, rank) and pg is not None
        ms = bench.max_over_ranks(pg, [10.0 + rank, 7.0 - rank], "cpu")
        units = bench.sum_over_ranks(pg, [1000.0 * (rank + 1)], "cpu")
        bench.barrier(pg)
        out.put((rank, ms, units))
    finally:
        pg.destroy_process_group()


def test_timings_max_and_units_sum_over_two_gloo_ranks():
    ctx = mp.get_context("spawn")
    out = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, out)) for r in range(2)]
    for p in procs:
        p.start()
    got = sorted(out.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, ms, units in got:
        assert ms == [11.0, 7.0]                 # slowest rank decides each timing
        assert units == [3000.0]                 # units of both replicas


def test_reference_arm_runs_on_rank_zero_only(monkeypatch, capsys):
    sys.path.insert(0, ROOT)
    import bench
    monkeypatch.setenv("RANK", "1")
    monkeypatch.setenv("WORLD_SIZE", "2")

    class Args:
        steps, warmup = 1, 0

    bench.run_reference(Args())                  # returns before touching the oracle
    assert capsys.readouterr().out == ""


def test_clock_sampler_reads_nvml_on_a_thread(monkeypatch):
    # a fake NVML (read-only queries): 1700 MHz under a 700 W load with the
    # power-cap reason set, and an idle sample that the summary ignores
    import time
    import types
    sys.path.insert(0, ROOT)
    import bench
    calls = {"n": 0}
    fake = types.SimpleNamespace(
        NVML_CLOCK_SM=1,
        nvmlInit=lambda: None,
        nvmlDeviceGetHandleByUUID=lambda u: "h",
        nvmlDeviceGetHandleByIndex=lambda i: "h",
        nvmlDeviceGetMaxClockInfo=lambda h, c: 1965,
        nvmlDeviceGetClockInfo=lambda h, c: 1700,
        nvmlDeviceGetCurrentClocksEventReasons=lambda h: 0x4,
    )

    def power(h):
        calls["n"] += 1
        return 100_000 if calls["n"] == 1 else 700_000          # milliwatts
    fake.nvmlDeviceGetPowerUsage = power
    monkeypatch.setitem(sys.modules, "pynvml", fake)
    with bench.ClockSampler(0) as clk:
        time.sleep(0.15)
    s = clk.summary()
    assert s["source"].startswith("nvml") and s["samples"] >= 3
    assert s["sm_mhz"] == 1700 and s["sm_max_mhz"] == 1965 and s["reasons"] == ["sw_power_cap"]
