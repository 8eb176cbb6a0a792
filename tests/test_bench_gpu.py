"""bench.py keeps its output contract: one JSON line with the metric, the
whole-job value, the timing bookkeeping, the roofline of the dominant launch
(HBM fraction and the row-traffic floor), the end-to-end figure with its
host<->device bytes, the clock record and the launch count.  A short run on
the decoder workload (a few seconds of GPU time)."""
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
             "--no-cpu-baseline")
    for k in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step",
              "higher_is_better", "scaling", "vs_baseline", "dtype", "data", "config",
              "roofline", "e2e", "gpu_launches", "clocks", "impl"):
        assert k in d, k
    assert d["n_gpus"] == 1 and d["steps"] == 5 and d["warmup"] == 3
    assert d["higher_is_better"] is True and d["scaling"] == "weak" and d["impl"] == "ours"
    assert d["value"] > 0 and d["ms_per_step"] > 0
    assert d["gpu_launches"] == 2 * d["steps"]
    assert "workload" in d["config"]
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
             "fused", "--no-e2e", "--no-cpu-baseline", "--no-floors")
    assert d["value"] > 0 and "graph" in d["config"]["launch"]
    assert "msda_backward_fused" in d["kernels"]["bwd"]["kernel"]
