"""The CPU oracle timed on every workload beside the GPU path (a measurement
tool, not a test; it needs a GPU):

    python -m tests.oracle_suite [--cpu-seconds 3]

For each workload the oracle (plain fp64 C, `oracle/`) runs on one thread and
on all host cores, in child processes whose OMP_NUM_THREADS fixes the thread
count, on a seeded sample sized for about --cpu-seconds; a sample smaller than
the workload is extrapolated linearly to tokens/s.  The GPU path runs the same
configuration through the public binding with its inputs resident.  One JSON
line: per workload the tokens/s of both and their ratio, plus the bias updates
alone per step.
"""
from __future__ import annotations

import argparse
import json
import os
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

def _cpu_model():
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    return line.split(":", 1)[1].strip()
    except OSError:
        pass
    return "unknown"


SUITE_ENTRIES = [  # (workload, mode)
    ("tiny", "gemm"), ("mid", "gemm"), ("drift", "gemm"), ("ties", "gemm"), ("ties", "logits"),
    ("dispatch", "dispatch"),
]


def oracle_suite_cpu(seconds):
    """CPU half of --oracle-suite (run in a child whose OMP_NUM_THREADS fixes
    the oracle's threads): per entry, the rows timed and the seconds taken.
    Each sample is sized for about `seconds`; a sample smaller than the
    workload is extrapolated linearly (tokens/s)."""
    import numpy as np
    import oracle
    import synth
    oracle.build()
    out = []
    for name, mode in SUITE_ENTRIES:
        c = synth.WORKLOADS[name]
        T, d, Nr, K = c["T"], c["d"], c["Nr"], c["K"]
        cap = T
        if mode == "gemm":
            W = synth.router_weight(Nr, d, seed=synth.BASE_SEED + d)

            def run(rows, seed):
                h = synth.hidden_normal(rows, d, seed=seed, quant8=(name == "ties"))
                b = synth.dead_start_bias(Nr).numpy() if name == "ties" else np.zeros(Nr, np.float32)
                m = np.zeros(Nr, np.float32)
                t0 = time.perf_counter()
                r = oracle.router_gemm(h, W, b, K)
                oracle.smebu(r.counts, b, m)
                return time.perf_counter() - t0
        elif mode == "logits":
            def run(rows, seed):
                x = synth.logits_normal(rows, Nr, seed=seed, quant8=True).numpy()
                b = synth.dead_start_bias(Nr).numpy()
                m = np.zeros(Nr, np.float32)
                t0 = time.perf_counter()
                r = oracle.router_logits(x, b, K)
                oracle.smebu(r.counts, b, m)
                return time.perf_counter() - t0
        else:  # dispatch, identity expert, combine; host memory bounds the sample
            cap = min(T, 16384)

            def run(rows, seed):
                h = synth.hidden_normal(rows, d, seed=seed)
                r = oracle.router_logits(synth.logits_normal(rows, Nr, seed=seed + 1).numpy(),
                                         np.zeros(Nr, np.float32), K)
                t0 = time.perf_counter()
                _, perm, dest = oracle.dispatch(r.idx, Nr)
                X = oracle.gather_rows(h, perm)
                oracle.combine(X, r.gates, dest, want64=False, want32=True)
                return time.perf_counter() - t0
        rows = min(64, cap)  # grow the sample until it takes a measurable share of the budget
        t = run(rows, 1)
        while t < seconds / 8 and rows < cap:
            rows = min(cap, rows * max(2, int(seconds / 8 / max(t, 1e-6))))
            t = run(rows, 1)
        rows = int(min(cap, max(1, rows * seconds / max(t, 1e-6))))
        t = run(rows, 2)
        out.append({"workload": name, "mode": mode, "rows": rows, "seconds": t, "tokens_per_s": rows / t,
                    "extrapolated": rows < T})
    # the bias updates alone, per step, at N_r = 256 on the tie workload's loads
    counts = np.bincount(np.random.default_rng(5).integers(0, 256, 4 * 1048576), minlength=256).astype(np.int64)
    b = synth.dead_start_bias(256).numpy()
    m = np.zeros(256, np.float32)
    reps = 2000
    t0 = time.perf_counter()
    for _ in range(reps):
        oracle.smebu(counts, b, m)
    t_smebu = (time.perf_counter() - t0) / reps
    t0 = time.perf_counter()
    for _ in range(reps):
        oracle.sign_update(counts, b)
    t_sign = (time.perf_counter() - t0) / reps
    out.append({"workload": "ties", "mode": "updates", "smebu_us": t_smebu * 1e6, "sign_us": t_sign * 1e6})
    return out


def oracle_suite(args):
    """Oracle timings on one thread and on all cores beside the GPU path's
    tokens/s on the same configurations (inputs resident on the GPU)."""
    import torch
    import expert_bias_load_b200 as ebl
    import synth
    cpu = {}
    for label, threads in (("one_thread", 1), ("all_cores", os.cpu_count() or 1)):
        env = dict(os.environ, OMP_NUM_THREADS=str(threads))
        r = subprocess.run([sys.executable, "-m", "tests.oracle_suite", "--cpu-only", "--cpu-seconds",
                            str(args.cpu_seconds)], env=env, cwd=ROOT, capture_output=True, text=True, check=True)
        cpu[label] = (threads, json.loads(r.stdout.strip().splitlines()[-1]))
    dev = torch.device("cuda:0")
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(2)]

    def gpu_ms(fn, warmup=3, reps=10):
        for _ in range(warmup):
            fn()
        torch.cuda.synchronize()
        ev[0].record()
        for _ in range(reps):
            fn()
        ev[1].record()
        torch.cuda.synchronize()
        return ev[0].elapsed_time(ev[1]) / reps

    entries = []
    # bias updates alone: one CTA per step; 1000 back-to-back launches per CUDA-event pair
    counts = torch.bincount(torch.randint(0, 256, (4 * 1048576,), generator=torch.Generator().manual_seed(5)),
                            minlength=256).to(torch.int32).to(dev)
    b = synth.dead_start_bias(256, device=dev)
    m = torch.zeros(256, device=dev)
    upd = {"workload": "ties", "step": "bias update alone (N_r = 256)",
           "gpu_smebu_us": gpu_ms(lambda: ebl.smebu_step(counts, b, m), reps=1000) * 1e3,
           "gpu_sign_us": gpu_ms(lambda: ebl.sign_update_step(counts, b, 1e-3), reps=1000) * 1e3,
           "note": "GPU per launch from Python: the host's launch rate bounds it (the kernel itself takes about "
                   "5 us in a launch list)"}
    for label, (threads, res) in cpu.items():
        upd["oracle_" + label + "_smebu_us"] = res[-1]["smebu_us"]
        upd["oracle_" + label + "_sign_us"] = res[-1]["sign_us"]
    for i, (name, mode) in enumerate(SUITE_ENTRIES):
        c = synth.WORKLOADS[name]
        T, d, Nr, K = c["T"], c["d"], c["Nr"], c["K"]
        bias = synth.dead_start_bias(Nr, device=dev) if name == "ties" else torch.zeros(Nr, device=dev)
        m = torch.zeros(Nr, device=dev)
        counts = torch.zeros(Nr, dtype=torch.int32, device=dev)
        idx = torch.empty(T, K, dtype=torch.int32, device=dev)
        g = torch.empty(T, K, device=dev)
        if mode == "gemm":
            h = synth.hidden_normal(T, d, seed=synth.step_seed(name, 0), device=dev, quant8=(name == "ties"))
            W = synth.router_weight(Nr, d, seed=synth.BASE_SEED + d).to(dev)

            def fn():
                ebl.router_forward(h, W, bias, K, counts, topk_idx=idx, gates=g)
                ebl.smebu_step(counts, bias, m, reset_counts=True)
            what = "router (GEMM mode) + SMEBU"
        elif mode == "logits":
            x = synth.logits_normal(T, Nr, seed=synth.step_seed(name, 0), device=dev, quant8=True)

            def fn():
                ebl.router_forward_logits(x, bias, K, counts, topk_idx=idx, gates=g)
                ebl.smebu_step(counts, bias, m, reset_counts=True)
            what = "router (logits mode) + SMEBU"
        else:
            h = synth.hidden_normal(T, d, seed=synth.step_seed(name, 0), device=dev)
            x = synth.logits_normal(T, Nr, seed=synth.step_seed(name, 0) + 1, device=dev)
            tiles = torch.empty((T + 127) // 128, Nr, dtype=torch.int32, device=dev)
            ebl.router_forward_logits(x, torch.zeros(Nr, device=dev), K, counts, topk_idx=idx, gates=g,
                                      tile_counts=tiles)
            del x
            offsets, perm, dest, X = ebl.moe_dispatch(h, idx, Nr, tile_counts=tiles)
            ws = torch.empty(max(16, ebl.dispatch_workspace_bytes(T, Nr)), dtype=torch.uint8, device=dev)
            out = torch.empty(T, d, device=dev)

            def fn():
                ebl.moe_dispatch(h, idx, Nr, tile_counts=tiles, offsets=offsets, perm=perm, dest=dest,
                                 dispatched=X, workspace=ws)
                ebl.moe_combine(X, g, dest, out=out)
            what = "dispatch + identity expert + combine"
        ms = gpu_ms(fn)
        gpu_tps = T / (ms / 1e3)
        e = {"workload": name, "T": T, "d": d, "N_r": Nr, "K": K, "step": what, "gpu_tokens_per_s": gpu_tps,
             "gpu_ms": ms}
        for label, (threads, res) in cpu.items():
            r = res[i]
            e["oracle_" + label] = {"threads": threads, "rows": r["rows"], "seconds": r["seconds"],
                                    "tokens_per_s": r["tokens_per_s"], "extrapolated": r["extrapolated"]}
            e["gpu_over_oracle_" + label] = gpu_tps / r["tokens_per_s"]
        entries.append(e)
        del fn
        torch.cuda.empty_cache()
    entries.append(upd)
    print(json.dumps({"oracle_suite": entries, "cpu_model": _cpu_model(), "nproc": os.cpu_count(),
                      "note": "oracle samples sized for about %.0f s each; a sample smaller than T is "
                              "extrapolated linearly" % args.cpu_seconds}), flush=True)


def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    ap.add_argument("--cpu-seconds", type=float, default=3.0, help="target CPU time of each oracle sample")
    ap.add_argument("--cpu-only", action="store_true", help=argparse.SUPPRESS)
    a = ap.parse_args(argv)
    if a.cpu_only:
        print(json.dumps(oracle_suite_cpu(a.cpu_seconds)), flush=True)
        return
    oracle_suite(a)


if __name__ == "__main__":
    main()
