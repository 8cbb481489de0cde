"""bench.py --impl reference (the CPU oracle on the host's cores) prints the
contract's line with "impl": "reference"; it needs no GPU."""
import json
import os
import subprocess
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_reference_arm_line():
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--steps", "2",
                        "--warmup", "1"], cwd=ROOT, capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [l for l in r.stdout.splitlines() if l.strip().startswith("{")]
    assert len(lines) == 1
    j = json.loads(lines[0])
    assert j["impl"] == "reference" and j["value"] > 0 and j["unit"] == "tokens/s"
    assert j["higher_is_better"] is True and j["steps"] == 2 and j["warmup"] == 1
    assert j["cpu_baseline"]["kind"] == "oracle" and j["cpu_baseline"]["value"] == j["value"]
    assert j["e2e"] == {"value": j["value"], "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}


def test_oracle_suite_child_lines():
    """The CPU half of the benchmark's per-workload oracle suite: the one-thread
    child times tiny, mid and drift; the all-cores child also the dispatch
    workload's router, the tie workload in logits mode and dispatch + combine.
    Each entry names its workload and mode and gives rows, seconds and a
    positive tokens/s (a sample smaller than T is marked extrapolated)."""
    want = {1: [("tiny", "gemm"), ("mid", "gemm"), ("drift", "gemm")],
            2: [("tiny", "gemm"), ("mid", "gemm"), ("drift", "gemm"), ("dispatch", "gemm"), ("ties", "logits"),
                ("dispatch", "dispatch")]}
    for mode, entries in want.items():
        env = dict(os.environ, OMP_NUM_THREADS="1" if mode == 1 else "2")
        r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--suite-cpu-only", str(mode),
                            "--suite-seconds", "0.05"], cwd=ROOT, env=env, capture_output=True, text=True,
                           timeout=600)
        assert r.returncode == 0, r.stderr[-2000:]
        res = json.loads(r.stdout.strip().splitlines()[-1])
        if mode == 1:                                   # the one-thread child also times the bias updates alone
            upd = res.pop()
            assert upd["mode"] == "updates" and upd["smebu_us"] > 0 and upd["sign_us"] > 0
        assert [(e["workload"], e["mode"]) for e in res] == entries
        for e in res:
            assert e["rows"] >= 1 and e["seconds"] > 0 and e["tokens_per_s"] > 0
            assert isinstance(e["extrapolated"], bool)
