"""bench.py keeps its output contract: one JSON line with the metric, the
whole-job value, the timing bookkeeping, the roofline of the dominant launch
(HBM fraction and the row-traffic floor), the end-to-end figure with its
host<->device bytes, the clock record, the launch count and the sub-records
of other workloads.  Short runs (a few seconds of GPU time each)."""
import json
import os
import subprocess
import sys

import pytest
import torch

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")


def _run(*args):
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), *args],
                       capture_output=True, text=True, cwd=ROOT, timeout=600)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [ln for ln in r.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1, r.stdout
    return json.loads(lines[0])


def test_bench_json_contract():
    d = _run("--workload", "decoder", "--steps", "5", "--warmup", "3", "--e2e-steps", "2",
             "--no-cpu-baseline", "--also", "")
    for k in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step",
              "higher_is_better", "scaling", "vs_baseline", "dtype", "data", "config",
              "roofline", "e2e", "gpu_launches", "clocks", "impl"):
        assert k in d, k
    assert d["n_gpus"] == 1 and d["steps"] == 5 and d["warmup"] == 3
    assert d["higher_is_better"] is True and d["scaling"] == "weak" and d["impl"] == "ours"
    assert d["value"] > 0 and d["ms_per_step"] > 0
    assert d["gpu_launches"] == 2 * d["steps"]
    assert "workload" in d["config"] and d["config"]["schedule"].startswith("untiled")
    r = d["roofline"]
    for k in ("bound", "achieved", "peak", "unit", "frac", "traffic"):
        assert k in r, k
    assert r["bound"] == "hbm" and r["unit"] == "GB/s"
    assert abs(r["frac"] - r["achieved"] / r["peak"]) < 1e-9
    assert 0 < r["value_rows_touched"] <= 2 * 17821 * 8
    e = d["e2e"]
    assert e["value"] > 0 and e["h2d_bytes_per_step"] > 0 and e["d2h_bytes_per_step"] > 0
    assert e["unit"] == d["unit"]
    f = d["row_floors"]
    assert f["rows"] > 0 and 0 < f["gather_us"] < f["gather_reduce_us"]
    assert set(d["clocks"]) >= {"sm_mhz", "sm_max_mhz", "reasons"}


def test_bench_graph_and_fused_step():
    d = _run("--workload", "decoder", "--steps", "5", "--warmup", "3", "--graph", "--step",
             "fused", "--no-e2e", "--no-cpu-baseline", "--no-floors", "--also", "")
    assert d["value"] > 0 and "graph" in d["config"]["launch"]
    assert "msda_backward_fused" in d["kernels"]["bwd"]["kernel"]


def test_bench_tiled_schedule_and_sub_records():
    """With --schedule tiled the plan's sort, the tiled forward and the tiled
    backward are three launches per step; the e2e leg runs the same calls; a
    sub-record times another workload on the same schedule."""
    d = _run("--workload", "encoder", "--schedule", "tiled", "--steps", "4", "--warmup", "3",
             "--e2e-steps", "2", "--no-cpu-baseline", "--no-floors", "--also", "encoder_bf16",
             "--also-steps", "3")
    assert d["config"]["schedule"].startswith("tiled")
    assert d["gpu_launches"] == 3 * d["steps"]
    assert "fwd_tiled_kernel" in d["kernels"]["fwd"]["kernel"]
    assert "bwd_tiled_kernel" in d["kernels"]["bwd"]["kernel"]
    assert d["e2e"]["value"] > 0 and "tiled" in d["e2e"]["api"]
    (sub,) = d["also"]
    assert "bf16" in sub["workload"] and sub["fwd_ms"] > 0 and sub["bwd_ms"] > 0
    assert sub["queries_per_s"] > 0 and set(sub["clocks"]) >= {"sm_mhz", "reasons"}
