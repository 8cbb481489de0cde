"""The router step written as a plain PyTorch pipeline, timed beside the
library on the same GPU (a measurement tool, not a test; it needs a GPU):

    python -m tests.torch_baseline [--tokens 1048576] [--reps 20]

The PyTorch version is the unfused reading of the same step on the same
inputs: a cuBLAS bf16 matmul for the logits, then sigmoid, + bias, topk,
gates, bincount and the SMEBU update in separate kernels, with the logits
going through HBM.  Its results are not compared with the library's (the
logits are rounded to bf16 by the matmul); only the time is.  One JSON line.
"""
from __future__ import annotations

import argparse
import json
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)


def main(argv=None):
    import torch

    import expert_bias_load_b200 as ebl
    import synth

    ap = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    ap.add_argument("--tokens", type=int, default=synth.WORKLOADS["ties"]["T"])
    ap.add_argument("--reps", type=int, default=20)
    a = ap.parse_args(argv)
    dev = torch.device("cuda:0")
    c = synth.WORKLOADS["ties"]
    T, d, Nr, K = a.tokens, c["d"], c["Nr"], c["K"]
    h = synth.hidden_normal(T, d, seed=synth.step_seed("ties", 0), device=dev, quant8=True)
    W = synth.router_weight(Nr, d, seed=synth.BASE_SEED + d).to(dev)
    lam, beta, kappa = 5e-4, 0.5, 2.0

    def torch_step(b, m):
        x = torch.matmul(h, W.t()).float()                    # cuBLAS bf16 GEMM, logits through HBM
        s = torch.sigmoid(x)
        idx = torch.topk(s + b, K, dim=1).indices
        g = torch.gather(s, 1, idx)
        g = g / g.sum(1, keepdim=True)
        n = torch.bincount(idx.reshape(-1), minlength=Nr).double()
        nbar = n.mean()
        db = lam * torch.tanh(kappa * (nbar - n) / nbar)
        db = db - db.mean()
        m.mul_(beta).add_((1.0 - beta) * db.float())
        b.add_(m)
        return idx, g

    counts = torch.zeros(Nr, dtype=torch.int32, device=dev)
    idx_l = torch.empty(T, K, dtype=torch.int32, device=dev)
    g_l = torch.empty(T, K, device=dev)

    def lib_step(b, m):
        ebl.router_forward(h, W, b, K, counts, topk_idx=idx_l, gates=g_l)
        ebl.smebu_step(counts, b, m, reset_counts=True)

    ev = [torch.cuda.Event(enable_timing=True) for _ in range(2)]

    def timed(fn):
        b = synth.dead_start_bias(Nr, device=dev)
        m = torch.zeros(Nr, device=dev)
        for _ in range(3):
            fn(b, m)
        torch.cuda.synchronize()
        ev[0].record()
        for _ in range(a.reps):
            fn(b, m)
        ev[1].record()
        torch.cuda.synchronize()
        return ev[0].elapsed_time(ev[1]) / a.reps

    # alternate so that both see the same clock state
    t_torch = [timed(torch_step), timed(torch_step)]
    t_lib = [timed(lib_step), timed(lib_step)]
    t_torch.append(timed(torch_step))
    t_lib.append(timed(lib_step))
    ms_t, ms_l = min(t_torch), min(t_lib)
    print(json.dumps({"tokens": T, "d": d, "N_r": Nr, "K": K, "reps": a.reps,
                      "pytorch_ms_per_step": ms_t, "library_ms_per_step": ms_l,
                      "pytorch_tokens_per_s": T / (ms_t / 1e3), "library_tokens_per_s": T / (ms_l / 1e3),
                      "speedup": ms_t / ms_l}), flush=True)


if __name__ == "__main__":
    main()
