"""The benchmark's own arm on the GPU prints one JSON line with every key of the measurement
contract: the device-timed value, the binding roofline of the dominant kernel, the CPU
oracle baseline, the end-to-end number through host buffers, the launch count and the
clocks sampled during the timed region."""
import json
import os
import subprocess
import sys

import pytest

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

KEYS = {"metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better", "scaling",
        "vs_baseline", "dtype", "data", "config", "roofline", "cpu_baseline", "e2e", "gpu_launches", "clocks"}


def bench_line(*extra):
    cmd = [sys.executable, os.path.join(ROOT, "bench.py"), "--warmup", "3", "--soak", "0", "--cpu-seconds", "1",
           *extra]
    r = subprocess.run(cmd, capture_output=True, text=True, timeout=900, cwd=ROOT)
    assert r.returncode == 0, r.stderr[-3000:]
    lines = [l for l in r.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1, r.stdout[-2000:]
    return json.loads(lines[0])


@pytest.mark.parametrize("extra,unit,bound", [
    (("--workload", "scan_bf16_2x1536x2048", "--steps", "5"), "elems/s", "alu"),
    (("--workload", "decode_bf16_256x5120", "--steps", "50"), "rows/s", "hbm"),
    (("--workload", "conv_bf16_2x1536x2048", "--steps", "5"), "elems/s", "hbm"),
    (("--workload", "scan_f32_1x64x256", "--steps", "5", "--backward"), "elems/s", None),
])
def test_bench_line(cuda_device, extra, unit, bound):
    d = bench_line(*extra)
    assert KEYS <= set(d), KEYS - set(d)
    assert d["unit"] == unit and d["n_gpus"] == 1 and d["value"] > 0 and d["ms_per_step"] > 0
    assert d["higher_is_better"] is True and d["scaling"] == "weak" and d["vs_baseline"] is None
    assert d["config"]["workload"] == extra[1]
    roof = d["roofline"]
    assert {"bound", "achieved", "peak", "unit", "frac", "traffic"} <= set(roof)
    if bound is not None:
        assert roof["bound"] == bound
    assert roof["achieved"] > 0 and roof["peak"] > 0
    assert abs(roof["frac"] - roof["achieved"] / roof["peak"]) < 1e-9
    cb = d["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["value"] > 0 and cb["cores"] >= 1 and cb["sample"]
    e2e = d["e2e"]
    assert e2e["value"] > 0 and e2e["unit"] == unit
    assert e2e["h2d_bytes_per_step"] > 0 and e2e["d2h_bytes_per_step"] > 0
    assert d["gpu_launches"] >= d["steps"]
    clk = d["clocks"]
    assert {"sm_mhz", "sm_max_mhz", "reasons"} <= set(clk)
