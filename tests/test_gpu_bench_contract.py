"""bench.py's JSON line on a GPU: a short run of the default arm prints one
line that carries every key of the benchmark contract, with consistent
values (value = step bytes x K / median pass time, the roofline fraction =
achieved / peak, launches counted per timed pass), for both the graph-replay
and the eager timing."""
import json
import os
import subprocess
import sys

import pytest
import torch

pytestmark = pytest.mark.gpu
ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _bench(*extra):
    cmd = [sys.executable, "bench.py", "--steps", "3", "--warmup", "3", "--repeats", "3",
           "--no-cpu-baseline", *extra]
    out = subprocess.run(cmd, cwd=ROOT, capture_output=True, text=True, timeout=600)
    assert out.returncode == 0, out.stderr[-3000:]
    lines = [l for l in out.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1, out.stdout[-2000:]
    return json.loads(lines[0])


@pytest.mark.parametrize("eager", [False, True], ids=["graph", "eager"])
def test_bench_line_keys_and_consistency(eager):
    if not torch.cuda.is_available():
        pytest.fail("GPU tests need a CUDA device")
    d = _bench(*(["--eager"] if eager else []))
    for k in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step",
              "higher_is_better", "scaling", "vs_baseline", "dtype", "data", "config",
              "roofline", "e2e", "gpu_launches", "clocks", "repeats", "timed"):
        assert k in d, k
    assert d["n_gpus"] == 1 and d["steps"] == 3 and d["warmup"] == 3
    assert d["unit"] == "GB/s" and d["higher_is_better"] is True and d["scaling"] == "weak"
    assert d["config"]["workload"] and "plans" in d["config"]
    step_bytes = d["config"]["bytes_per_step"]
    assert abs(d["value"] - step_bytes / (d["ms_per_step"] / 1e3) / 1e9) <= 1e-3 * d["value"] + 0.05
    assert d["repeats"]["value_min"] <= d["value"] <= d["repeats"]["value_max"]
    r = d["roofline"]
    for k in ("bound", "achieved", "peak", "unit", "frac", "traffic"):
        assert k in r, k
    assert r["bound"] == "hbm" and r["unit"] == "GB/s"
    assert abs(r["frac"] - r["achieved"] / r["peak"]) < 1e-3
    e = d["e2e"]
    for k in ("value", "unit", "h2d_bytes_per_step", "d2h_bytes_per_step"):
        assert k in e, k
    assert e["value"] > 0 and e["h2d_bytes_per_step"] > 0 and e["d2h_bytes_per_step"] > 0
    assert d["gpu_launches"] == 2 * 3 * 3  # two ops per step, K steps, R passes
    c = d["clocks"]
    assert "sm_mhz" in c and "sm_max_mhz" in c and isinstance(c["reasons"], list)
    assert ("eager" in d["timed"]) == eager
