"""bench.py end to end on one GPU at tiny scale: the JSON line it prints carries
the keys of the benchmark contract (throughput, end-to-end with host copies,
roofline, launches, clocks), for the verify-batch stack and for the many-row
(prefill) mode."""
import json
import os
import subprocess
import sys

import pytest

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _run_bench(*args):
    cmd = [sys.executable, os.path.join(ROOT, "bench.py"), "--layers", "1", "--steps", "2", "--warmup", "1",
           "--no-cpu-baseline", *args]
    out = subprocess.run(cmd, cwd=ROOT, capture_output=True, text=True, timeout=600)
    assert out.returncode == 0, out.stderr[-2000:]
    lines = [l for l in out.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1, out.stdout
    return json.loads(lines[0])


def _check_common(d, m):
    for key in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better",
                "scaling", "vs_baseline", "dtype", "data", "config", "e2e", "roofline", "gpu_launches"):
        assert key in d, key
    assert d["value"] > 0 and d["ms_per_step"] > 0
    assert d["n_gpus"] == 1 and d["steps"] == 2 and d["warmup"] == 1
    assert d["config"]["m"] == m and "workload" in d["config"]
    e2e = d["e2e"]
    assert e2e["value"] > 0 and e2e["h2d_bytes_per_step"] > 0 and e2e["d2h_bytes_per_step"] > 0
    r = d["roofline"]
    for key in ("bound", "achieved", "peak", "unit", "frac", "traffic"):
        assert key in r, key
    assert 0 < r["frac"] < 2
    assert d["gpu_launches"] > 0


def test_bench_verify_stack_json():
    d = _run_bench("--only", "k")
    _check_common(d, 32)
    assert d["roofline"]["bound"] == "hbm" and d["roofline"]["unit"] == "GB/s"
    for m in (32, 1, 8, 16):
        assert d["us_per_layer_m%d" % m] > 0
    assert "issue" in d["roofline"] and "roofline_m1" in d
    assert d["e2e"]["eager"]["value"] > 0
    assert d["config"]["calls"] == "one grouped call per layer"


def test_bench_chained_and_separate_json():
    d = _run_bench("--layers", "2", "--no-extra", "--separate", "--m", "8")
    _check_common(d, 8)
    assert d["config"]["calls"] == "one call per matrix"
    d = _run_bench("--layers", "1")
    assert d["us_per_layer_chain_m32"] > 0 and d["us_per_layer_chain_m1"] > 0


def test_bench_many_row_json():
    d = _run_bench("--only", "k", "--m", "64")
    _check_common(d, 64)
    assert d["roofline"]["bound"] == "tensor" and d["roofline"]["unit"] == "TFLOP/s"
    assert d["tflops"] > 0
