"""The data-parallel router step with the CUDA kernels on two ranks.

"SMEBU Load Balancing", "How it works" defines n_i as the tokens routed to
expert i in the optimizer step; with the batch split over ranks that is the
sum of the ranks' loads, so each rank runs the library's router on its shard,
the int32 loads are all-reduced, and every rank applies the library's SMEBU
update to the global loads.

Two `gloo` ranks run as processes on the one GPU (cuda:0).  No kernel of one
rank waits on the other's: the exchange is a host-side all-reduce between the
router and the update, so the two processes only share the device.  Checks:
  - each step the all-reduced loads are the sum of the two ranks' local loads;
  - both ranks hold bit-identical bias and momentum after every step;
  - logits mode (bit-exact loads): the loads, bias and momentum equal those of
    the oracle routing the concatenated batch with its own bias, in closed
    loop;
  - GEMM mode: each rank's routing matches the oracle's fp64 router on its
    shard under the near-tie rule, and the oracle's update fed the global
    loads (open loop) leaves the ranks' state within 1e-6 relative.
"""
import datetime
import os
import socket

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

import oracle
import synth
from tests.parity import STATE_RTOL, assert_gemm_parity, rel_err

pytestmark = pytest.mark.gpu

WORLD = 2
STEPS = 20
T_RANK, D, NR, K = 4096 + 37, 512, 256, 4


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _shard(mode, step, rank):
    seed = 9000 + 101 * step + rank
    if mode == "logits":
        return synth.logits_normal(T_RANK, NR, seed=seed, quant8=True)
    return synth.hidden_normal(T_RANK, D, seed=seed)


def _weight():
    return synth.router_weight(NR, D, seed=8999)


def _worker(rank, world, port, mode, out_dir):
    import torch.distributed as dist

    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    torch.cuda.set_device(0)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=120))
    try:
        from expert_bias_load_b200 import dp

        dev = torch.device("cuda:0")
        step = dp.cuda_logits_step(K) if mode == "logits" else dp.cuda_step(_weight().to(dev), K)
        inner_route, inner_update = step.route, step.update
        rec = {"local": [], "glob": [], "b": [], "m": [], "idx": [], "gates": [], "b_in": []}

        def route(x, b, c):
            rec["b_in"].append(b.cpu().numpy().copy())
            idx, g = inner_route(x, b, c)
            rec["local"].append(c.cpu().numpy().copy())
            rec["idx"].append(idx.cpu().numpy())
            rec["gates"].append(g.cpu().numpy())
            return idx, g

        def update(c, b, m, mv):
            rec["glob"].append(c.cpu().numpy().copy())
            inner_update(c, b, m, mv)
            rec["b"].append(b.cpu().numpy().copy())
            rec["m"].append(m.cpu().numpy().copy())

        step.route, step.update = route, update
        bias = synth.dead_start_bias(NR, device=dev)
        mom = torch.zeros(NR, device=dev)
        counts = torch.zeros(NR, dtype=torch.int32, device=dev)
        for s in range(STEPS):
            step(_shard(mode, s, rank).to(dev), bias, mom, counts)
        torch.cuda.synchronize()
        np.savez(os.path.join(out_dir, "rank%d.npz" % rank), **{k: np.stack(v) for k, v in rec.items()})
        dist.barrier()
    finally:
        dist.destroy_process_group()


def _spawn(mode, tmp_path):
    mp.spawn(_worker, args=(WORLD, _free_port(), mode, str(tmp_path)), nprocs=WORLD, join=True)
    return [dict(np.load(os.path.join(tmp_path, "rank%d.npz" % r))) for r in range(WORLD)]


def _common_checks(r):
    r0, r1 = r
    assert np.array_equal(r0["glob"], r0["local"] + r1["local"])      # the exchange sums the loads
    assert np.array_equal(r0["glob"], r1["glob"])
    assert np.array_equal(r0["b"], r1["b"]) and np.array_equal(r0["m"], r1["m"])   # replicas agree bit for bit
    assert np.all(r0["glob"].sum(1) == K * T_RANK * WORLD)


def test_two_rank_logits_step_matches_oracle_on_concatenated_batch(cuda_device, tmp_path):
    r = _spawn("logits", tmp_path)
    _common_checks(r)
    b_o = synth.dead_start_bias(NR).numpy()
    m_o = np.zeros(NR, np.float32)
    for s in range(STEPS):
        x = torch.cat([_shard("logits", s, rank) for rank in range(WORLD)]).numpy()
        ref = oracle.router_logits(x, b_o, K)
        assert np.array_equal(r[0]["glob"][s].astype(np.int64), ref.counts), s
        for rank in range(WORLD):
            assert np.array_equal(r[rank]["idx"][s], ref.idx[rank * T_RANK:(rank + 1) * T_RANK]), (s, rank)
        oracle.smebu(ref.counts, b_o, m_o)
        assert rel_err(r[0]["b"][s], b_o).max() <= STATE_RTOL, s
        assert rel_err(r[0]["m"][s], m_o).max() <= STATE_RTOL, s
    assert float(np.abs(b_o[8:]).max()) > 0


def test_two_rank_gemm_step_matches_oracle_open_loop(cuda_device, tmp_path):
    r = _spawn("gemm", tmp_path)
    _common_checks(r)
    W = _weight()
    b_o = synth.dead_start_bias(NR).numpy()
    m_o = np.zeros(NR, np.float32)
    for s in range(STEPS):
        for rank in range(WORLD):
            b_in = r[rank]["b_in"][s]
            ref = oracle.router_gemm(_shard("gemm", s, rank), W, b_in, K, want_scores=True)
            assert_gemm_parity(r[rank]["idx"][s], r[rank]["gates"][s], ref, NR, b_in,
                               gpu_counts=r[rank]["local"][s])
        oracle.smebu(r[0]["glob"][s].astype(np.int64), b_o, m_o)
        assert rel_err(r[0]["b"][s], b_o).max() <= STATE_RTOL, s
        assert rel_err(r[0]["m"][s], m_o).max() <= STATE_RTOL, s
