"""Seeded synthetic inputs for the router step: hidden states, router weights,
fp32 logits and bias starting points.

This module draws random numbers and shapes them into the workloads; it holds
none of the router's, the balancer's or the dispatcher's arithmetic.  Both the
tests (which hand the same tensors to the CUDA library and to the CPU oracle)
and the benchmark use it.

Determinism: every generator takes an integer seed and a device.  The same
seed on the same device gives the same tensor; torch's CPU and CUDA generators
are different streams, so the CPU and GPU tensors of one seed differ.  A test
that compares two implementations generates once and gives both the same data.

Workload recipes (shapes, distributions) follow the five router workloads:
  tiny      T=2048,    d=256,  Nr=64,  K=4   hidden N(0,1)
  mid       T=65536,   d=2048, Nr=128, K=8   hidden N(0,1)
  drift     T=131072,  d=3072, Nr=256, K=4   N(0,1) + rank-8 drift on 16 router rows
  dispatch  T=262144,  d=4096, Nr=256, K=4   hidden N(0,1)
  ties      T=1048576, d=4096, Nr=256, K=4   values quantised to multiples of 1/8,
                                             8 experts starting at bias -1.0
W_router is truncated-normal with std 0.5/sqrt(d), clipped at +-2 std by
resampling, rounded to bf16 (round to nearest even).
"""
from __future__ import annotations

import math

import torch

BASE_SEED = 0xEB1

WORKLOADS = {
    "tiny": dict(T=2048, d=256, Nr=64, K=4, steps=10),
    "mid": dict(T=65536, d=2048, Nr=128, K=8, steps=50),
    "drift": dict(T=131072, d=3072, Nr=256, K=4, steps=200),
    "dispatch": dict(T=262144, d=4096, Nr=256, K=4, steps=1),
    "ties": dict(T=1048576, d=4096, Nr=256, K=4, steps=100),
}

# rows drawn per chunk when generating big tensors (keeps fp32 temporaries small)
_CHUNK_ELEMS = 1 << 28


def _gen(seed: int, device) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(int(seed) & ((1 << 63) - 1))
    return g


def _normal_rows(rows: int, cols: int, seed: int, device, quant8: bool, out_dtype) -> torch.Tensor:
    out = torch.empty((rows, cols), dtype=out_dtype, device=device)
    step = max(1, _CHUNK_ELEMS // max(cols, 1))
    for c, r0 in enumerate(range(0, rows, step)):
        r1 = min(rows, r0 + step)
        g = _gen(seed * 1000003 + c, device)
        x = torch.randn((r1 - r0, cols), generator=g, device=device, dtype=torch.float32)
        if quant8:
            x = torch.round(x * 8.0) / 8.0
        out[r0:r1] = x.to(out_dtype)
    return out


def hidden_normal(T: int, d: int, seed: int, device="cpu", quant8: bool = False) -> torch.Tensor:
    """bf16 [T,d], i.i.d. N(0,1); with quant8 the samples are rounded to
    multiples of 1/8 first (exact in bf16 for |x| < 32)."""
    return _normal_rows(T, d, seed, device, quant8, torch.bfloat16)


def logits_normal(T: int, Nr: int, seed: int, device="cpu", quant8: bool = False) -> torch.Tensor:
    """fp32 [T,Nr] precomputed router logits, i.i.d. N(0,1) (optionally
    quantised to multiples of 1/8 so that equal scores are common)."""
    return _normal_rows(T, Nr, seed, device, quant8, torch.float32)


def router_weight(Nr: int, d: int, seed: int, device="cpu") -> torch.Tensor:
    """bf16 [Nr,d]: truncated normal, std 0.5/sqrt(d), samples outside +-2 std
    redrawn until none remain."""
    std = 0.5 / math.sqrt(d)
    g = _gen(seed, "cpu")
    w = torch.randn((Nr, d), generator=g, dtype=torch.float64) * std
    bad = w.abs() > 2.0 * std
    while bool(bad.any()):
        n = int(bad.sum())
        w[bad] = torch.randn(n, generator=g, dtype=torch.float64) * std
        bad = w.abs() > 2.0 * std
    return w.to(torch.bfloat16).to(device)


def hidden_drift(T: int, d: int, W: torch.Tensor, seed: int, mu: float, device="cpu") -> torch.Tensor:
    """bf16 [T,d] = z + sum_{j<8} a_{t,j} u_j with z ~ N(0,1),
    u_j = unit(W[r_{2j}] + W[r_{2j+1}]) over 16 seeded distinct router rows r,
    and a_{t,j} ~ N(mu, 1).  The drift concentrates routing on those 16 experts."""
    Nr = W.shape[0]
    g = _gen(seed ^ 0x5A5A, "cpu")
    rows = torch.randperm(Nr, generator=g)[:16]
    Wf = W.to(torch.float32).cpu()
    u = torch.stack([Wf[rows[2 * j]] + Wf[rows[2 * j + 1]] for j in range(8)])
    u = u / u.norm(dim=1, keepdim=True)
    u = u.to(device)
    out = torch.empty((T, d), dtype=torch.bfloat16, device=device)
    step = max(1, _CHUNK_ELEMS // d)
    for c, r0 in enumerate(range(0, T, step)):
        r1 = min(T, r0 + step)
        gz = _gen(seed * 1000003 + c, device)
        z = torch.randn((r1 - r0, d), generator=gz, device=device, dtype=torch.float32)
        a = torch.randn((r1 - r0, 8), generator=gz, device=device, dtype=torch.float32) + mu
        out[r0:r1] = (z + a @ u).to(torch.bfloat16)
    return out


def drift_rows(Nr: int, seed: int) -> torch.Tensor:
    """The 16 router rows hidden_drift aligns with (same seed, same draw)."""
    g = _gen(seed ^ 0x5A5A, "cpu")
    return torch.randperm(Nr, generator=g)[:16]


def dead_start_bias(Nr: int, n_dead: int = 8, value: float = -1.0, device="cpu") -> torch.Tensor:
    """fp32 [Nr] zeros with the lowest n_dead experts set to `value`."""
    b = torch.zeros(Nr, dtype=torch.float32, device=device)
    b[:n_dead] = value
    return b


def step_seed(workload: str, step: int) -> int:
    """Seed of the fresh batch of step `step` of a workload."""
    index = list(WORKLOADS).index(workload) + 1
    return BASE_SEED + index + 7919 * step
