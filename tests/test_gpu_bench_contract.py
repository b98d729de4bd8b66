"""The benchmark's output contract: `python bench.py` and `python bench.py
--impl reference` each print one JSON line with the keys and units the
harness reads (run here on the small float32 configuration, as child
processes)."""
import json
import os
import subprocess
import sys

import pytest

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _line(args):
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py")] + args, cwd=ROOT,
                       capture_output=True, text=True, timeout=900)
    assert r.returncode == 0, r.stdout[-2000:] + r.stderr[-2000:]
    lines = [l for l in r.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1, r.stdout[-2000:]
    return json.loads(lines[0])


def test_bench_line_keys():
    d = _line(["--config", "tiny_f32", "--steps", "4", "--warmup", "3"])
    for k in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step",
              "higher_is_better", "scaling", "vs_baseline", "dtype", "data", "config",
              "roofline", "e2e", "gpu_launches", "clocks", "cpu_baseline"):
        assert k in d, k
    assert d["n_gpus"] == 1 and d["steps"] == 4 and d["warmup"] == 3
    assert d["higher_is_better"] is True and d["scaling"] == "weak" and d["value"] > 0
    assert d["config"]["workload"] == "tiny_f32" and d["dtype"] == "f32"
    r = d["roofline"]
    for k in ("bound", "achieved", "peak", "unit", "frac", "traffic"):
        assert k in r, k
    assert r["frac"] == pytest.approx(r["achieved"] / r["peak"])
    e = d["e2e"]
    assert e["unit"] == "tokens/s" and e["value"] > 0
    assert e["h2d_bytes_per_step"] == e["d2h_bytes_per_step"] == 128 * 256 * 4
    assert d["gpu_launches"] > 0 and d["device_status"] == 0
    c = d["cpu_baseline"]
    assert c["kind"] == "oracle" and c["cores"] >= 1 and c["value"] > 0 and c["sample"]
    assert c["one_thread"]["cores"] == 1
    assert {"sm_mhz", "sm_max_mhz", "reasons"} <= set(d["clocks"])


def test_reference_line_keys():
    d = _line(["--impl", "reference", "--config", "tiny_f32", "--steps", "2", "--warmup", "3"])
    assert d["impl"] == "reference" and d["value"] > 0 and d["unit"] == "tokens/s"
    assert d["dtype"] == "f64" and d["config"]["workload"] == "tiny_f32"
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["value"] == d["value"]
    assert d["e2e"] == {"value": d["value"], "unit": "tokens/s", "h2d_bytes_per_step": 0,
                        "d2h_bytes_per_step": 0}
