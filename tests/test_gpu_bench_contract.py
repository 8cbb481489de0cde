"""bench.py prints the one JSON line the benchmark contract asks for (small
case on one GPU): required keys, units, and the roofline / cpu_baseline / e2e /
clocks objects."""
import json
import os
import subprocess
import sys

import pytest

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _run(*args):
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), *args], cwd=ROOT, capture_output=True,
                       text=True, timeout=900)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [l for l in r.stdout.splitlines() if l.strip().startswith("{")]
    assert len(lines) == 1, r.stdout[-2000:]
    return json.loads(lines[0])


def test_bench_line_has_the_contract_keys(cuda_device):
    j = _run("--tokens", "65536", "--steps", "5", "--warmup", "3", "--e2e-steps", "1", "--cpu-seconds", "1")
    for k in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better",
              "scaling", "vs_baseline", "dtype", "data", "config", "roofline", "cpu_baseline", "e2e",
              "gpu_launches", "clocks"):
        assert k in j, k
    assert j["n_gpus"] == 1 and j["steps"] == 5 and j["warmup"] == 3
    assert j["higher_is_better"] is True and j["scaling"] == "weak" and j["unit"] == "tokens/s"
    assert j["value"] > 0 and "workload" in j["config"]
    r = j["roofline"]
    for k in ("bound", "achieved", "peak", "unit", "frac", "traffic"):
        assert k in r, k
    assert abs(r["frac"] - r["achieved"] / r["peak"]) < 1e-9
    c = j["cpu_baseline"]
    assert c["kind"] == "oracle" and c["cores"] >= 1 and c["value"] > 0 and c["sample"]
    e = j["e2e"]
    assert e["h2d_bytes_per_step"] == 65536 * 4096 * 2 and e["d2h_bytes_per_step"] > 0 and e["value"] > 0
    assert j["gpu_launches"] == 2 * 5
    assert "sm_mhz" in j["clocks"] and "reasons" in j["clocks"]


def test_smoke_entry_point(cuda_device):
    """__graft_entry__.smoke() runs as the round-end check runs it."""
    sys.path.insert(0, ROOT)
    import __graft_entry__
    __graft_entry__.smoke()
