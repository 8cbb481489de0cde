"""The data-parallel step's exchange on two `gloo` ranks (CPU, no GPU).

Each rank routes its own shard of tokens with the CPU oracle standing in for
the CUDA router, the loads are all-reduced, and the oracle's SMEBU update is
applied.  After several steps both ranks must hold bit-identical bias and
momentum, equal to a single process that routed the concatenated batch.
"""
import os
import socket

import numpy as np
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import oracle
from expert_bias_load_b200.dp import DataParallelRouterStep, global_loads

T_PER_RANK, D, NR, K, STEPS = 96, 32, 16, 2, 6


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _inputs(step, rank):
    g = torch.Generator().manual_seed(1000 * step + rank)
    h = torch.randn(T_PER_RANK, D, generator=g).to(torch.bfloat16)
    return h


def _weight():
    g = torch.Generator().manual_seed(7)
    return (torch.randn(NR, D, generator=g) * 0.3).to(torch.bfloat16)


def _route(W):
    def route(hidden, bias, counts):
        r = oracle.router_gemm(hidden, W, bias.numpy(), K)
        counts += torch.from_numpy(r.counts.astype(np.int32))
        return r.idx
    return route


def _update(counts, bias, momentum, maxvio):
    b, m = bias.numpy(), momentum.numpy()
    oracle.smebu(counts.numpy().astype(np.int64), b, m)
    counts.zero_()


def _worker(rank, world, port, out):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        W = _weight()
        step = DataParallelRouterStep(_route(W), _update)
        bias = torch.zeros(NR)
        mom = torch.zeros(NR)
        counts = torch.zeros(NR, dtype=torch.int32)
        for s in range(STEPS):
            step(_inputs(s, rank), bias, mom, counts)
        out[rank] = (bias.clone(), mom.clone())
        # the exchange itself: loads of both ranks are summed
        c = torch.full((NR,), rank + 1, dtype=torch.int32)
        global_loads(c)
        assert torch.equal(c, torch.full((NR,), 3, dtype=torch.int32))
    finally:
        dist.destroy_process_group()


def test_two_rank_smebu_matches_single_process():
    world = 2
    manager = mp.Manager()
    out = manager.dict()
    mp.spawn(_worker, args=(world, _free_port(), out), nprocs=world, join=True)
    b0, m0 = out[0]
    b1, m1 = out[1]
    assert torch.equal(b0, b1) and torch.equal(m0, m1)          # replicas agree bit for bit
    # single process over the concatenated batch
    W = _weight()
    bias = np.zeros(NR, np.float32)
    mom = np.zeros(NR, np.float32)
    for s in range(STEPS):
        h = torch.cat([_inputs(s, r) for r in range(world)])
        r = oracle.router_gemm(h, W, bias, K)
        oracle.smebu(r.counts, bias, mom)
    assert np.array_equal(b0.numpy(), bias) and np.array_equal(m0.numpy(), mom)
    assert float(np.abs(bias).max()) > 0


def test_global_loads_is_identity_without_process_group():
    c = torch.arange(5, dtype=torch.int32)
    assert torch.equal(global_loads(c.clone()), c)
