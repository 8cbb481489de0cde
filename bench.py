"""Benchmark: routed tokens/s of the router step (router GEMM + sigmoid + biased
Top-K + gates + load histogram + SMEBU update) on the tie workload
(T=1,048,576 tokens, d=4096, N_r=256, K=4, hidden on a 1/8 grid, 8 experts
starting at bias -1.0), GEMM mode, bf16 inputs with fp32 accumulation.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

One process per GPU (torchrun for N > 1).  Each rank routes its own batch of T
tokens (weak scaling); the per-expert loads are summed across ranks with one
NCCL all-reduce before the SMEBU step, so every rank applies the same update.
Rank 0 prints one JSON line.  `--impl reference` times the CPU oracle on the
host's cores on a bounded sample of the same workload.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

WORKLOAD = "ties"
METRIC = "routed tokens/s (router+top-K+hist+SMEBU) at N_r=256,K=4; % of roofline"


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=1000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--e2e-steps", type=int, default=3)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-full-step", action="store_true")
    ap.add_argument("--cpu-seconds", type=float, default=12.0, help="target CPU time of the oracle sample")
    ap.add_argument("--suite-seconds", type=float, default=3.0,
                    help="target CPU time of each oracle sample of the per-workload suite (0: skip the suite)")
    ap.add_argument("--suite-cpu-only", type=int, default=0, help=argparse.SUPPRESS)
    ap.add_argument("--tokens", type=int, default=0,
                    help="tokens per GPU (default: the tie workload's 1,048,576); smaller values are for profiling")
    return ap.parse_args()


def measured_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            j = json.load(f)
        return {"hbm_gbs": j["hbm_gbs"], "bf16_tflops": j["bf16_tflops"],
                "bf16_tflops_sustained": j.get("bf16_tflops_sustained"), "source": "measured"}
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0, "source": "fallback"}


def kernel_source_hash(files):
    h = hashlib.sha256()
    for f in files:
        with open(os.path.join(ROOT, f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:16]


ROUTER_SOURCES = ["expert_bias_load_b200/csrc/router_gemm.cu", "expert_bias_load_b200/csrc/ptx.cuh",
                  "expert_bias_load_b200/csrc/topk.cuh"]


def profiled_traffic(workload_key):
    """DRAM bytes per launch of the router kernel from the committed ncu
    summary, if it was taken on the current kernel source; else None."""
    p = os.path.join(ROOT, "profiles", "router_gemm_traffic.json")
    if not os.path.exists(p):
        return None
    with open(p) as f:
        j = json.load(f)
    if j.get("source_hash") != kernel_source_hash(ROUTER_SOURCES):
        return None
    entry = j.get("per_launch", {}).get(workload_key)
    return None if entry is None else float(entry["dram_bytes_full_launch"])


class ClockSampler:
    """SM clock, power and clock-event reasons sampled during the timed region.

    NVML is read from a background thread every 2 ms (the timed region of a
    short run lasts tens of milliseconds); where NVML is not importable,
    nvidia-smi is sampled every 10 ms instead.  Nothing is changed on the GPU:
    only its state is read."""
    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
    # NVML clock-event reason bits
    REASONS = {0x4: "sw_power_cap", 0x8: "hw_slowdown", 0x20: "sw_thermal_slowdown", 0x40: "hw_thermal_slowdown",
               0x80: "hw_power_brake_slowdown"}

    def __init__(self, gpu_index, pci_bus_id=None):
        self.gpu = gpu_index
        self.pci = pci_bus_id
        self.proc = None
        self.path = None
        self.thread = None
        self.rows = []

    def _nvml_handle(self):
        import pynvml
        pynvml.nvmlInit()
        if self.pci:
            try:
                return pynvml, pynvml.nvmlDeviceGetHandleByPciBusId(self.pci)
            except pynvml.NVMLError:
                pass
        return pynvml, pynvml.nvmlDeviceGetHandleByIndex(self.gpu)

    def start(self):
        import threading
        try:
            nv, h = self._nvml_handle()
            reasons_fn = getattr(nv, "nvmlDeviceGetCurrentClocksEventReasons", None) or \
                nv.nvmlDeviceGetCurrentClocksThrottleReasons
            max_sm = nv.nvmlDeviceGetMaxClockInfo(h, nv.NVML_CLOCK_SM)
            self.stop_flag = threading.Event()

            def run():
                while not self.stop_flag.is_set():
                    try:
                        self.rows.append((nv.nvmlDeviceGetClockInfo(h, nv.NVML_CLOCK_SM), max_sm,
                                          nv.nvmlDeviceGetPowerUsage(h) / 1000.0, int(reasons_fn(h))))
                    except nv.NVMLError:
                        pass
                    self.stop_flag.wait(0.002)

            self.thread = threading.Thread(target=run, daemon=True)
            self.thread.start()
            while not self.rows and self.thread.is_alive():  # the first sample precedes the timed region
                time.sleep(0.001)
            self.rows.clear()
            return
        except Exception:
            self.thread = None
        import tempfile
        fd, self.path = tempfile.mkstemp(prefix="clocks_", suffix=".csv")
        os.close(fd)
        try:
            self.proc = subprocess.Popen(["nvidia-smi", "-i", str(self.gpu), "--query-gpu=" + self.Q,
                                          "--format=csv,noheader,nounits", "-lms", "10", "-f", self.path],
                                         stderr=subprocess.DEVNULL)
            time.sleep(0.5)
        except OSError:
            self.proc = None

    def stop(self):
        if self.thread is not None:
            self.stop_flag.set()
            self.thread.join(timeout=5)
            rows = list(self.rows)
            if not rows:
                return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"], "source": "nvml"}
            reasons = sorted({name for r in rows for bit, name in self.REASONS.items() if r[3] & bit})
            return {"sm_mhz": statistics.median(r[0] for r in rows), "sm_max_mhz": max(r[1] for r in rows),
                    "reasons": reasons, "samples": len(rows), "power_w_max": max(r[2] for r in rows),
                    "source": "nvml, every 2 ms"}
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        rows = []
        with open(self.path) as f:
            for line in f:
                parts = [x.strip() for x in line.split(",")]
                if len(parts) >= 9:
                    rows.append(parts)
        os.unlink(self.path)
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"]}
        sm = [float(r[1]) for r in rows if r[1].replace(".", "").isdigit()]
        mx = [float(r[2]) for r in rows if r[2].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i in range(4) if r[5 + i].lower() == "active"})
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(mx) if mx else None,
                "reasons": reasons, "samples": len(rows), "source": "nvidia-smi, every 10 ms"}


# ---------------------------------------------------------------- oracle leg

class OracleSample:
    """The CPU oracle (fp64 router GEMM + Top-K + gates + counts, then SMEBU)
    on a bounded sample of the workload's rows."""

    def __init__(self, cfg):
        import numpy as np
        import oracle
        import synth
        self.np, self.oracle, self.synth = np, oracle, synth
        self.cfg = cfg
        oracle.build()
        d, Nr = cfg["d"], cfg["Nr"]
        self.W = synth.router_weight(Nr, d, seed=synth.BASE_SEED + d)
        self.bias = synth.dead_start_bias(Nr).numpy()
        self.threads = int(os.environ.get("OMP_NUM_THREADS", os.cpu_count() or 1))

    def run(self, rows, seed):
        """Seconds the oracle takes for `rows` tokens (inputs made outside the timing)."""
        h = self.synth.hidden_normal(rows, self.cfg["d"], seed=seed, quant8=True)
        b = self.bias.copy()
        m = self.np.zeros(self.cfg["Nr"], self.np.float32)
        t0 = time.perf_counter()
        r = self.oracle.router_gemm(h, self.W, b, self.cfg["K"])
        self.oracle.smebu(r.counts, b, m)
        return time.perf_counter() - t0

    def rows_for(self, seconds):
        # a 64-row probe overstates the time per row (thread start-up), so a
        # second probe of about a tenth of the target refines the estimate
        t = self.run(64, seed=1)
        rows = int(max(64, min(self.cfg["T"], 64 * seconds / 10 / max(t, 1e-4))))
        t = self.run(rows, seed=2)
        return int(max(16, min(self.cfg["T"], rows * seconds / max(t, 1e-4))))


def oracle_sample(cfg, seconds, seed=0):
    """Time the oracle on a sample sized for about `seconds` of CPU work;
    returns (tokens_per_s, rows, threads, seconds)."""
    o = OracleSample(cfg)
    rows = o.rows_for(seconds)
    t = o.run(rows, seed)
    return rows / t, rows, o.threads, t


# ------------------------------------------------ oracle on every workload

def cpu_model():
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    return line.split(":", 1)[1].strip()
    except OSError:
        pass
    return "unknown"


# (workload, mode, timed on one thread, timed on all cores)
SUITE_ENTRIES = [
    ("tiny", "gemm", True, True), ("mid", "gemm", True, True), ("drift", "gemm", True, True),
    ("dispatch", "gemm", False, True), ("ties", "logits", False, True), ("dispatch", "dispatch", False, True),
]


def suite_cpu(seconds, threads_label):
    """CPU half of the suite, run in a child process whose OMP_NUM_THREADS
    fixes the oracle's threads: per entry, the rows timed and the seconds.
    Each sample is sized for about `seconds`; a sample smaller than the
    workload is extrapolated linearly (tokens/s)."""
    import numpy as np
    import oracle
    import synth
    oracle.build()
    out = []
    for name, mode, one, allc in SUITE_ENTRIES:
        if not (one if threads_label == "one_thread" else allc):
            continue
        c = synth.WORKLOADS[name]
        T, d, Nr, K = c["T"], c["d"], c["Nr"], c["K"]
        cap = T
        if mode == "gemm":
            W = synth.router_weight(Nr, d, seed=synth.BASE_SEED + d)

            def run(rows, seed):
                h = synth.hidden_normal(rows, d, seed=seed)
                b = np.zeros(Nr, np.float32)
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
    if threads_label == "one_thread":
        # the bias updates alone, per step, at N_r = 256 on loads of the tie workload's size
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


def cpu_baseline_suite(seconds, dev):
    """The oracle on every workload (one thread on tiny, mid and drift; all
    host cores on those, on the dispatch workload's router, on the tie
    workload in logits mode and on dispatch + combine), each beside the GPU
    path's tokens/s on the same configuration with inputs resident."""
    import torch
    import expert_bias_load_b200 as ebl
    import synth
    cpu = {}
    for label, threads in (("one_thread", 1), ("all_cores", os.cpu_count() or 1)):
        env = dict(os.environ, OMP_NUM_THREADS=str(threads))
        r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--suite-cpu-only",
                            "1" if label == "one_thread" else "2", "--suite-seconds", str(seconds)],
                           env=env, cwd=ROOT, capture_output=True, text=True, check=True)
        cpu[label] = (threads, json.loads(r.stdout.strip().splitlines()[-1]))
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
    # the bias updates alone: one CTA per step, 1000 back-to-back launches per CUDA-event pair
    counts = torch.bincount(torch.randint(0, 256, (4 * 1048576,), generator=torch.Generator().manual_seed(5)),
                            minlength=256).to(torch.int32).to(dev)
    b = synth.dead_start_bias(256, device=dev)
    m = torch.zeros(256, device=dev)
    upd = {"workload": "ties", "step": "bias update alone (N_r = 256), per step",
           "gpu_smebu_us": gpu_ms(lambda: ebl.smebu_step(counts, b, m), reps=1000) * 1e3,
           "gpu_sign_us": gpu_ms(lambda: ebl.sign_update_step(counts, b, 1e-3), reps=1000) * 1e3,
           "note": "GPU: per launch from Python, which the host's launch rate bounds; oracle: one thread, "
                   "per call through ctypes"}
    for r in cpu["one_thread"][1]:
        if r.get("mode") == "updates":
            upd["oracle_smebu_us"] = r["smebu_us"]
            upd["oracle_sign_us"] = r["sign_us"]
    for name, mode, _, _ in SUITE_ENTRIES:
        c = synth.WORKLOADS[name]
        T, d, Nr, K = c["T"], c["d"], c["Nr"], c["K"]
        bias = synth.dead_start_bias(Nr, device=dev) if name == "ties" else torch.zeros(Nr, device=dev)
        m = torch.zeros(Nr, device=dev)
        counts = torch.zeros(Nr, dtype=torch.int32, device=dev)
        idx = torch.empty(T, K, dtype=torch.int32, device=dev)
        g = torch.empty(T, K, device=dev)
        if mode == "gemm":
            h = synth.hidden_normal(T, d, seed=synth.step_seed(name, 0), device=dev)
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
            for r in res:
                if r["workload"] == name and r["mode"] == mode:
                    e["oracle_" + label] = {"threads": threads, "rows": r["rows"], "seconds": r["seconds"],
                                            "tokens_per_s": r["tokens_per_s"], "extrapolated": r["extrapolated"]}
                    e["gpu_over_oracle_" + label] = gpu_tps / r["tokens_per_s"]
        entries.append(e)
        del fn
        torch.cuda.empty_cache()
    entries.append(upd)
    return {"entries": entries, "cpu_model": cpu_model(), "nproc": os.cpu_count(),
            "note": "oracle samples sized for about %.0f s each; a sample smaller than T is extrapolated "
                    "linearly; GPU inputs resident" % seconds}


# ------------------------------------------------------------------- GPU leg

def main():
    args = parse()
    if args.suite_cpu_only:
        print(json.dumps(suite_cpu(args.suite_seconds, "one_thread" if args.suite_cpu_only == 1 else "all_cores")),
              flush=True)
        return
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    import synth
    cfg = dict(synth.WORKLOADS[WORKLOAD])
    if args.tokens > 0:
        cfg["T"] = args.tokens
    T, d, Nr, K = cfg["T"], cfg["d"], cfg["Nr"], cfg["K"]
    config = {"workload": "tie workload: T=%d tokens/GPU, d=%d, N_r=%d, K=%d, hidden on a 1/8 grid, "
                          "8 experts at bias -1.0, GEMM mode" % (T, d, Nr, K),
              "tokens_per_gpu": T, "d": d, "N_r": Nr, "K": K, "smebu": [5e-4, 0.5, 2.0],
              "l2": "inputs larger than L2 (hidden %.1f GB per GPU)" % (T * d * 2 / 1e9),
              "parallelism": "dp%d (per-expert loads all-reduced)" % world}

    if args.impl == "reference":
        if rank != 0:
            return
        # each step routes a bounded sample of the workload on the host cores,
        # sized so that the whole run takes about two minutes
        o = OracleSample(cfg)
        per_step = min(3.0, max(0.05, 120.0 / (args.warmup + args.steps)))
        rows = o.rows_for(per_step)
        threads = o.threads
        vals = []
        for s in range(args.warmup + args.steps):
            t = o.run(rows, seed=s)
            if s >= args.warmup:
                vals.append(rows / t)
        v = statistics.median(vals)
        line = {"impl": "reference", "metric": METRIC, "value": v, "unit": "tokens/s", "n_gpus": args.gpus,
                "steps": args.steps, "warmup": args.warmup, "ms_per_step": rows / v * 1e3,
                "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
                "data": "synthetic", "config": config,
                "cpu_baseline": {"value": v, "unit": "tokens/s", "cores": threads, "kind": "oracle",
                                 "sample": "%d rows of the tie workload per step (fp64 router + SMEBU)" % rows},
                "e2e": {"value": v, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
        print(json.dumps(line), flush=True)
        return

    import torch
    import torch.distributed as dist
    import expert_bias_load_b200 as ebl
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=dev)
    ebl.lib()

    # inputs resident in HBM: a fresh seeded batch per rank
    h = synth.hidden_normal(T, d, seed=synth.step_seed(WORKLOAD, 0) + 1000 * rank, device=dev, quant8=True)
    W = synth.router_weight(Nr, d, seed=synth.BASE_SEED + d).to(dev)
    bias = synth.dead_start_bias(Nr, device=dev)
    mom = torch.zeros(Nr, device=dev)
    counts = torch.zeros(Nr, dtype=torch.int32, device=dev)
    idx = torch.empty(T, K, dtype=torch.int32, device=dev)
    gates = torch.empty(T, K, dtype=torch.float32, device=dev)
    maxvio = torch.zeros(1, device=dev)
    status = torch.zeros(1, dtype=torch.int32, device=dev)
    stream = torch.cuda.current_stream()

    from expert_bias_load_b200.dp import DataParallelRouterStep, global_loads
    rec = [None, None]  # CUDA events around the router kernel of the current step

    def route(hidden, b, c):
        if rec[0] is not None:
            rec[0].record(stream)
        ebl.router_forward(hidden, W, b, K, c, topk_idx=idx, gates=gates, status=status, stream=stream)
        if rec[1] is not None:
            rec[1].record(stream)

    def update(c, b, m, mv):
        ebl.smebu_step(c, b, m, reset_counts=True, maxvio=mv, status=status, stream=stream)

    dp_step = DataParallelRouterStep(route, update)  # all-reduces the loads when world > 1

    def max_over_ranks(vals):
        """Element-wise max of per-rank timings (every rank calls this at the same point)."""
        if world == 1:
            return list(vals)
        t = torch.tensor(vals, device=dev, dtype=torch.float64)
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        return [float(x) for x in t]

    def step(ev0=None, ev1=None):
        rec[0], rec[1] = ev0, ev1
        dp_step(h, bias, mom, counts, maxvio)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    maxvio_first = float(maxvio.item())

    evr = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    props = torch.cuda.get_device_properties(dev)
    pci = None
    if hasattr(props, "pci_bus_id"):
        pci = "%08x:%02x:%02x.0" % (getattr(props, "pci_domain_id", 0), props.pci_bus_id, props.pci_device_id)
    clocks = ClockSampler(local, pci)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    clocks.start()
    e0.record(stream)
    for s in range(args.steps):
        step(*evr[s])
    e1.record(stream)
    torch.cuda.synchronize()
    clk = clocks.stop()
    if world > 1:
        dist.barrier()
    total_ms = e0.elapsed_time(e1)
    router_ms = statistics.mean(a.elapsed_time(b) for a, b in evr)
    if world > 1:
        t = torch.tensor([total_ms, router_ms], device=dev, dtype=torch.float64)
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        total_ms, router_ms = float(t[0]), float(t[1])
    st = int(status.item())
    ms_step = total_ms / args.steps
    value = T * world / (ms_step / 1e3)

    peaks = measured_peaks()
    flops = 2.0 * T * d * Nr
    alg_bytes = 2.0 * T * d + 8.0 * T * K + 2.0 * Nr * d + 8.0 * Nr
    achieved = flops / (router_ms / 1e3) / 1e12
    # The router is timed back to back for total_ms; a loop of a second or more
    # runs under the power cap like the sustained GEMM measurement, a shorter
    # one like the burst measurement.
    sustained = peaks.get("bf16_tflops_sustained")
    long_loop = total_ms >= 1000.0 and sustained
    peak = sustained if long_loop else peaks["bf16_tflops"]
    roofline = {"bound": "tensor", "achieved": achieved, "peak": peak, "unit": "TFLOP/s",
                "frac": achieved / peak, "traffic": profiled_traffic("ties_full"),
                "kernel": "router_gemm_kernel<4>", "kernel_ms": router_ms,
                "peak_source": "%s %s bf16 (%s); timed loop %.2f s" % (
                    peaks["source"], "sustained" if long_loop else "burst",
                    "MEASURED_PEAKS.json" if peaks["source"] == "measured" else "no MEASURED_PEAKS.json: the pool's earlier figures",
                    total_ms / 1e3),
                "frac_of_burst": achieved / peaks["bf16_tflops"],
                "frac_of_sustained": achieved / sustained if sustained else None,
                "hbm_view": {"alg_bytes": alg_bytes, "achieved_gbs": alg_bytes / (router_ms / 1e3) / 1e9,
                             "peak_gbs": peaks["hbm_gbs"],
                             "frac": alg_bytes / (router_ms / 1e3) / 1e9 / peaks["hbm_gbs"]},
                "roofline_time_ms": max(flops / peak / 1e12, alg_bytes / peaks["hbm_gbs"] / 1e9) * 1e3}
    roofline["frac_of_roofline_step"] = roofline["roofline_time_ms"] / ms_step

    # ---- end to end through the public API with host buffers
    e2e = None
    if args.e2e_steps > 0:
        h_host = torch.empty((T, d), dtype=torch.bfloat16, pin_memory=True)
        h_host.copy_(h)
        idx_host = torch.empty((T, K), dtype=torch.int32, pin_memory=True)
        gates_host = torch.empty((T, K), dtype=torch.float32, pin_memory=True)
        state_host = torch.empty((2 * Nr + 1,), dtype=torch.float32, pin_memory=True)
        state_dev = torch.empty((2 * Nr + 1,), dtype=torch.float32, device=dev)

        def e2e_step():
            h.copy_(h_host, non_blocking=True)
            step()
            state_dev[:Nr].copy_(bias)
            state_dev[Nr:2 * Nr].copy_(mom)
            state_dev[2 * Nr:].copy_(maxvio)
            idx_host.copy_(idx, non_blocking=True)
            gates_host.copy_(gates, non_blocking=True)
            state_host.copy_(state_dev, non_blocking=True)

        e2e_step()
        torch.cuda.synchronize()
        if world > 1:
            dist.barrier()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        for _ in range(args.e2e_steps):
            e2e_step()
        b.record(stream)
        torch.cuda.synchronize()
        e_ms = a.elapsed_time(b) / args.e2e_steps
        if world > 1:
            t = torch.tensor([e_ms], device=dev, dtype=torch.float64)
            dist.all_reduce(t, op=dist.ReduceOp.MAX)
            e_ms = float(t[0])
        e2e = {"value": T * world / (e_ms / 1e3), "unit": "tokens/s", "h2d_bytes_per_step": T * d * 2,
               "d2h_bytes_per_step": T * K * 8 + (2 * Nr + 1) * 4, "ms_per_step": e_ms}
        del h_host

    # ---- the rest of the hot path: dispatch, identity expert, combine (same workload)
    full = None
    if not args.no_full_step:
        tiles = torch.empty(((T + 127) // 128, Nr), dtype=torch.int32, device=dev)
        offsets = torch.empty(Nr + 1, dtype=torch.int32, device=dev)
        perm = torch.empty(T * K, dtype=torch.int32, device=dev)
        dest = torch.empty(T * K, dtype=torch.int32, device=dev)
        X = torch.empty((T * K, d), dtype=torch.bfloat16, device=dev)
        out = torch.empty((T, d), dtype=torch.float32, device=dev)
        ws = torch.empty(ebl.dispatch_workspace_bytes(T, Nr), dtype=torch.uint8, device=dev)
        ev = [torch.cuda.Event(enable_timing=True) for _ in range(4)]

        def fstep(rec):
            if rec:
                ev[0].record(stream)
            ebl.router_forward(h, W, bias, K, counts, topk_idx=idx, gates=gates, tile_counts=tiles,
                               status=status, stream=stream)
            global_loads(counts)
            ebl.smebu_step(counts, bias, mom, reset_counts=True, maxvio=maxvio, status=status, stream=stream)
            if rec:
                ev[1].record(stream)
            ebl.moe_dispatch(h, idx, Nr, tile_counts=tiles, offsets=offsets, perm=perm, dest=dest, dispatched=X,
                             workspace=ws, status=status, stream=stream)
            if rec:
                ev[2].record(stream)
            ebl.moe_combine(X, gates, dest, out=out, status=status, stream=stream)
            if rec:
                ev[3].record(stream)

        for _ in range(2):
            fstep(False)
        torch.cuda.synchronize()
        reps = max(3, min(10, args.steps // 50))
        tr = td = tc = 0.0
        for _ in range(reps):
            fstep(True)
            torch.cuda.synchronize()
            tr += ev[0].elapsed_time(ev[1])
            td += ev[1].elapsed_time(ev[2])
            tc += ev[2].elapsed_time(ev[3])
        tr, td, tc = max_over_ranks([tr / reps, td / reps, tc / reps])
        disp_bytes = T * d * 2 + T * K * d * 2
        comb_bytes = T * K * d * 2 + T * d * 4
        full = {"metric": "tokens/s through router+SMEBU+dispatch+identity expert+combine",
                "value": T * world / ((tr + td + tc) / 1e3), "ms_per_step": tr + td + tc,
                "router_smebu_ms": tr, "dispatch_ms": td, "combine_ms": tc,
                "dispatch_gbs": disp_bytes / (td / 1e3) / 1e9, "combine_gbs": comb_bytes / (tc / 1e3) / 1e9,
                "dispatch_frac_hbm": disp_bytes / (td / 1e3) / 1e9 / peaks["hbm_gbs"],
                "combine_frac_hbm": comb_bytes / (tc / 1e3) / 1e9 / peaks["hbm_gbs"]}
        del X, out

    # ---- logits mode (the bit-exact path) and the fused z-loss on the same workload shape
    extra = {}
    if not args.no_full_step:
        reps = max(3, min(20, args.steps // 50))
        zl = torch.zeros(1, dtype=torch.float64, device=dev)
        ev = [torch.cuda.Event(enable_timing=True) for _ in range(2)]
        for _ in range(2):
            ebl.router_forward_zloss(h, W, bias, K, counts, zl, topk_idx=idx, gates=gates, stream=stream)
        counts.zero_()
        ev[0].record(stream)
        for _ in range(reps):
            ebl.router_forward_zloss(h, W, bias, K, counts, zl, topk_idx=idx, gates=gates, stream=stream)
        ev[1].record(stream)
        torch.cuda.synchronize()
        extra["zloss_router_ms"] = max_over_ranks([ev[0].elapsed_time(ev[1]) / reps])[0]
        del zl
        # the balance option (per-tile statistics of the sequence-wise balance
        # loss) and the loss itself, sequences of 4096 tokens
        seq_len = 4096 if T % 4096 == 0 else 128 * (T // 128) if T % 128 == 0 else 0
        if seq_len:
            tcb = torch.empty((T + 127) // 128, Nr, dtype=torch.int32, device=dev)
            tpb = torch.empty((T + 127) // 128, Nr, dtype=torch.float32, device=dev)
            lseq = torch.empty(T // seq_len, dtype=torch.float64, device=dev)
            lval = torch.empty(1, dtype=torch.float64, device=dev)

            def balance_step():
                ebl.router_forward_balance(h, W, bias, K, counts, tcb, tpb, topk_idx=idx, gates=gates, stream=stream)
                ebl.seq_balance_loss(tcb, tpb, T, K, seq_len, loss_seq=lseq, loss=lval, stream=stream)

            for _ in range(2):
                balance_step()
            counts.zero_()
            ev[0].record(stream)
            for _ in range(reps):
                balance_step()
            ev[1].record(stream)
            torch.cuda.synchronize()
            bm = max_over_ranks([ev[0].elapsed_time(ev[1]) / reps])[0]
            extra["seq_balance"] = {"seq_len": seq_len, "router_balance_and_loss_ms": bm,
                                    "tokens_per_s": T * world / (bm / 1e3)}
            counts.zero_()
            del tcb, tpb, lseq, lval
        x = synth.logits_normal(T, Nr, seed=synth.step_seed(WORKLOAD, 1) + 1000 * rank, device=dev, quant8=True)
        # The logits kernels are issue-bound, so their time follows the SM
        # clock.  The GEMM-heavy measurements above leave the GPU near its
        # power limit (after the default loop of about 2 s, at the cap), so
        # the GPU idles a moment first and these launches start at the clock a
        # short run gets; the clock seen during the logits timing is reported.
        torch.cuda.synchronize()
        time.sleep(1.5)
        lreps = max(20, reps)
        for _ in range(2):
            ebl.router_forward_logits(x, bias, K, counts, topk_idx=idx, gates=gates, stream=stream)
        counts.zero_()
        torch.cuda.synchronize()
        lclocks = ClockSampler(local, pci)
        lclocks.start()
        ev[0].record(stream)
        for _ in range(lreps):
            ebl.router_forward_logits(x, bias, K, counts, topk_idx=idx, gates=gates, stream=stream)
        ev[1].record(stream)
        torch.cuda.synchronize()
        lclk = lclocks.stop()
        lm = max_over_ranks([ev[0].elapsed_time(ev[1]) / lreps])[0]
        lbytes = T * Nr * 4 + T * K * 8
        extra["logits_mode"] = {"tokens_per_s": T * world / (lm / 1e3), "ms": lm,
                                "achieved_gbs": lbytes / (lm / 1e3) / 1e9,
                                "frac_hbm": lbytes / (lm / 1e3) / 1e9 / peaks["hbm_gbs"],
                                "reps": lreps, "sm_mhz": lclk.get("sm_mhz"), "clock_reasons": lclk.get("reasons")}
        # the balance statistics fused into the routing pass (one read of the
        # logits), and as the separate fp64 pass
        tpl = torch.empty((T + 127) // 128, Nr, dtype=torch.float32, device=dev)
        tcl = torch.empty((T + 127) // 128, Nr, dtype=torch.int32, device=dev)
        for _ in range(2):
            ebl.router_forward_logits_balance(x, bias, K, counts, tcl, tpl, topk_idx=idx, gates=gates, stream=stream)
        counts.zero_()
        ev[0].record(stream)
        for _ in range(lreps):
            ebl.router_forward_logits_balance(x, bias, K, counts, tcl, tpl, topk_idx=idx, gates=gates, stream=stream)
        ev[1].record(stream)
        torch.cuda.synchronize()
        fm = max_over_ranks([ev[0].elapsed_time(ev[1]) / lreps])[0]
        extra["logits_mode"]["fused_balance_ms"] = fm
        extra["logits_mode"]["balance_stats_ms"] = fm - lm
        ebl.balance_stats_logits(x, tile_psum=tpl, stream=stream)
        ev[0].record(stream)
        for _ in range(reps):
            ebl.balance_stats_logits(x, tile_psum=tpl, stream=stream)
        ev[1].record(stream)
        torch.cuda.synchronize()
        extra["logits_mode"]["balance_stats_separate_fp64_ms"] = max_over_ranks([ev[0].elapsed_time(ev[1]) / reps])[0]
        del tpl, tcl
        counts.zero_()
        del x

    cpu = None
    suite = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        v, rows, threads, secs = oracle_sample(cfg, args.cpu_seconds)
        cpu = {"value": v, "unit": "tokens/s", "cores": threads, "kind": "oracle",
               "sample": "%d rows of the tie workload (fp64 router GEMM + top-K + gates + counts, then SMEBU), "
                         "%.1f s" % (rows, secs), "cpu_model": cpu_model(), "nproc": os.cpu_count()}
        if args.suite_seconds > 0 and args.tokens == 0:
            del h
            torch.cuda.empty_cache()
            suite = cpu_baseline_suite(args.suite_seconds, dev)

    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    if rank != 0:
        return
    line = {"metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms_step, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "bf16", "data": "synthetic", "config": config,
            "roofline": roofline, "cpu_baseline": cpu, "e2e": e2e, "gpu_launches": 2 * args.steps,
            "clocks": clk, "status": st, "maxvio_after_warmup": maxvio_first, "full_step": full, **extra,
            "cpu_baseline_suite": suite}
    print(json.dumps(line), flush=True)


if __name__ == "__main__":
    main()
