"""bench.py's JSON line keeps its contract, checked on the CPU.

bench.py's own code path runs under a CPU stand-in for the GPU
(tests/fake_gpu.py: inert streams and events, library calls recorded, not
launched) on the tiny layer and a small quantiser workload, so that a change
to the bench's host logic that would raise or drop a key of the line shows
here rather than in a GPU run.  The numbers are those of the stand-in and
mean nothing; the keys, their types and the recorded call sequence do.
"""
import json
import os
import sys

import pytest

from tests.fake_gpu import fake_gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

REQUIRED = {"metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better", "scaling",
            "vs_baseline", "dtype", "data", "config", "roofline", "e2e", "gpu_launches", "clocks"}


@pytest.fixture
def small_bench(monkeypatch):
    sys.path.insert(0, ROOT)
    import bench
    from fp8_moe_numerics_b200 import workloads
    monkeypatch.setitem(workloads.CONFIGS, "quant_small",
                        dict(rows=256, cols=512, x_dist="t4_rowscale", seed=3, sr_seed=0))
    monkeypatch.setattr(bench, "WORKLOAD", "tiny_layer")
    monkeypatch.setattr(bench, "QUANT_WORKLOAD", "quant_small")
    monkeypatch.delenv("RANK", raising=False)
    monkeypatch.delenv("WORLD_SIZE", raising=False)
    return bench


def test_default_line_has_every_contract_key(small_bench, monkeypatch, capsys):
    with fake_gpu(monkeypatch) as calls:
        monkeypatch.setattr(sys, "argv", ["bench.py", "--steps", "2", "--warmup", "3", "--no-cpu-baseline"])
        small_bench.main()
    lines = [ln for ln in capsys.readouterr().out.splitlines() if ln.startswith("{")]
    assert len(lines) == 1
    line = json.loads(lines[-1])
    assert REQUIRED <= set(line)
    assert line["n_gpus"] == 1 and line["steps"] == 2 and line["warmup"] == 3 and line["scaling"] == "weak"
    assert line["higher_is_better"] is True and line["data"].startswith("synthetic")
    assert isinstance(line["config"], dict) and "workload" in line["config"]
    r = line["roofline"]
    assert {"bound", "achieved", "peak", "unit", "frac", "traffic"} <= set(r) and r["bound"] in ("hbm", "tensor", "alu")
    e = line["e2e"]
    assert {"value", "unit", "h2d_bytes_per_step", "d2h_bytes_per_step"} <= set(e)
    assert e["h2d_bytes_per_step"] > 0 and e["d2h_bytes_per_step"] > 0
    assert {"sm_mhz", "sm_max_mhz", "reasons"} <= set(line["clocks"])
    # the step went through the library: routing first, the GEMMs of both passes
    assert calls[0] == "moe_route" and calls.count("grouped_gemm_nvfp4") >= 2 * 5
    assert "grouped_gemm_mxfp8" in calls and "mxfp8_requant_transpose_sr" in calls


def test_kernel_cases_run(small_bench, monkeypatch, capsys):
    for case in ("nvfp4_quantize", "requant", "nvfp4_quantize_sr", "requant_nvfp4", "step_nvfp4_backward"):
        with fake_gpu(monkeypatch) as calls:
            monkeypatch.setattr(sys, "argv", ["bench.py", "--kernel", case])
            small_bench.main()
        out = json.loads(capsys.readouterr().out.strip().splitlines()[-1])
        assert out["kernel"] == case and out["ms"] > 0 and len(calls) >= 4
