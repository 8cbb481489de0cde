"""Time one entry point of the library on one GPU.

    python -m expert_bias_load_b200.microbench logits --tokens 262144 --experts 256 --topk 4 --reps 3

Each invocation builds seeded synthetic inputs (the generators in `synth`), makes
`--warmup` calls and then `--reps` timed calls of one entry point on the current
stream, and prints one line: milliseconds per call (CUDA events), tokens per
second, and the bytes or flops per call over that time.  It runs nothing but the
public binding, so it is also the command to put under a profiler: with
`--warmup W` the timed calls are launches W+1 ... W+reps of that kernel.

Entry points: router (GEMM mode), zloss (GEMM mode with the z-loss), balance
(GEMM mode with the sequence-wise balance statistics, then the loss over
sequences of 4096 tokens, or of T tokens when T is smaller), logits (logits
mode), logits_balance (logits mode with the balance statistics in the same
pass), balance_logits (the logits-mode balance statistics as a separate fp64
pass), smebu, sign,
dispatch, combine.  For the one-CTA update kernels
(smebu, sign) the time per call is the host's launch rate, not the kernel's.
"""
from __future__ import annotations

import argparse

import torch

import expert_bias_load_b200 as ebl
import synth


def _time(fn, warmup, reps):
    for _ in range(warmup):
        fn()
    torch.cuda.synchronize()
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(2)]
    ev[0].record()
    for _ in range(reps):
        fn()
    ev[1].record()
    torch.cuda.synchronize()
    return ev[0].elapsed_time(ev[1]) / max(1, reps)


def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    ap.add_argument("op", choices=["router", "zloss", "balance", "logits", "logits_balance", "balance_logits", "smebu",
                                   "sign", "dispatch", "combine"])
    ap.add_argument("--tokens", type=int, default=1 << 20)
    ap.add_argument("--hidden", type=int, default=4096)
    ap.add_argument("--experts", type=int, default=256)
    ap.add_argument("--topk", type=int, default=4)
    ap.add_argument("--warmup", type=int, default=2)
    ap.add_argument("--reps", type=int, default=10)
    ap.add_argument("--seed", type=int, default=123)
    a = ap.parse_args(argv)
    if not torch.cuda.is_available():
        raise SystemExit("microbench needs a CUDA device")
    dev = torch.device("cuda:0")
    T, d, Nr, K = a.tokens, a.hidden, a.experts, a.topk
    bias = synth.dead_start_bias(Nr, device=dev)
    counts = torch.zeros(Nr, dtype=torch.int32, device=dev)
    work = ""
    if a.op in ("router", "zloss", "balance"):
        h = synth.hidden_normal(T, d, seed=a.seed, device=dev, quant8=True)
        W = synth.router_weight(Nr, d, seed=a.seed + 1).to(dev)
        idx = torch.empty(T, K, dtype=torch.int32, device=dev)
        g = torch.empty(T, K, device=dev)
        if a.op == "router":
            fn = lambda: ebl.router_forward(h, W, bias, K, counts, topk_idx=idx, gates=g)
        elif a.op == "balance":
            S = 4096 if T % 4096 == 0 else T
            if T % 128:
                raise SystemExit("balance needs --tokens a multiple of 128")
            tc = torch.empty(T // 128, Nr, dtype=torch.int32, device=dev)
            tp = torch.empty(T // 128, Nr, device=dev)

            def fn():
                ebl.router_forward_balance(h, W, bias, K, counts, tc, tp, topk_idx=idx, gates=g)
                ebl.seq_balance_loss(tc, tp, T, K, S)
        else:
            zl = torch.zeros(1, dtype=torch.float64, device=dev)
            fn = lambda: ebl.router_forward_zloss(h, W, bias, K, counts, zl, topk_idx=idx, gates=g)
        flops = 2.0 * T * d * Nr
        ms = _time(fn, a.warmup, a.reps)
        work = "%.1f TFLOP/s" % (flops / ms / 1e9)
    elif a.op == "logits":
        x = synth.logits_normal(T, Nr, seed=a.seed, device=dev, quant8=True)
        idx = torch.empty(T, K, dtype=torch.int32, device=dev)
        g = torch.empty(T, K, device=dev)
        fn = lambda: ebl.router_forward_logits(x, bias, K, counts, topk_idx=idx, gates=g)
        ms = _time(fn, a.warmup, a.reps)
        work = "%.1f GB/s" % ((T * Nr * 4 + T * K * 8) / ms / 1e6)
    elif a.op == "logits_balance":
        x = synth.logits_normal(T, Nr, seed=a.seed, device=dev, quant8=True)
        idx = torch.empty(T, K, dtype=torch.int32, device=dev)
        g = torch.empty(T, K, device=dev)
        tc = torch.empty((T + 127) // 128, Nr, dtype=torch.int32, device=dev)
        tp = torch.empty((T + 127) // 128, Nr, device=dev)
        fn = lambda: ebl.router_forward_logits_balance(x, bias, K, counts, tc, tp, topk_idx=idx, gates=g)
        ms = _time(fn, a.warmup, a.reps)
        work = "%.1f GB/s" % ((T * Nr * 4 + T * K * 8) / ms / 1e6)
    elif a.op == "balance_logits":
        x = synth.logits_normal(T, Nr, seed=a.seed, device=dev, quant8=True)
        tp = torch.empty((T + 127) // 128, Nr, device=dev)
        fn = lambda: ebl.balance_stats_logits(x, tile_psum=tp)
        ms = _time(fn, a.warmup, a.reps)
        work = "%.1f G scores/s" % (T * Nr / ms / 1e6)
    elif a.op in ("smebu", "sign"):
        counts.copy_(torch.randint(0, 2 * T * K // Nr + 1, (Nr,), generator=torch.Generator().manual_seed(a.seed),
                                   dtype=torch.int32).to(dev))
        m = torch.zeros(Nr, device=dev)
        if a.op == "smebu":
            fn = lambda: ebl.smebu_step(counts, bias, m)
        else:
            fn = lambda: ebl.sign_update_step(counts, bias, 1e-3)
        ms = _time(fn, a.warmup, a.reps)
        work = "%.1f us" % (ms * 1e3)
    else:
        h = synth.hidden_normal(T, d, seed=a.seed, device=dev)
        x = synth.logits_normal(T, Nr, seed=a.seed + 2, device=dev)
        tiles = torch.empty((T + ebl.tile_tokens() - 1) // ebl.tile_tokens(), Nr, dtype=torch.int32, device=dev)
        idx, g = ebl.router_forward_logits(x, bias, K, counts, tile_counts=tiles)
        del x
        offsets, perm, dest, X = ebl.moe_dispatch(h, idx, Nr, tile_counts=tiles)
        ws = torch.empty(max(16, ebl.dispatch_workspace_bytes(T, Nr)), dtype=torch.uint8, device=dev)
        if a.op == "dispatch":
            fn = lambda: ebl.moe_dispatch(h, idx, Nr, tile_counts=tiles, offsets=offsets, perm=perm, dest=dest,
                                          dispatched=X, workspace=ws)
            nbytes = T * d * 2 + T * K * d * 2
        else:
            out = torch.empty(T, d, device=dev)
            fn = lambda: ebl.moe_combine(X, g, dest, out=out)
            nbytes = T * K * d * 2 + T * d * 4
        ms = _time(fn, a.warmup, a.reps)
        work = "%.1f GB/s" % (nbytes / ms / 1e6)
    print("%s T=%d d=%d N_r=%d K=%d: %.4f ms, %.3e tokens/s, %s" % (a.op, T, d, Nr, K, ms, T / (ms / 1e3), work))


if __name__ == "__main__":
    main()
