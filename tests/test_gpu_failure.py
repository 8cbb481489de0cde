"""Failure detection and state handling on a B200, without faulting a GPU."""
import io
import time

import numpy as np
import pytest
import torch

import expert_bias_load_b200 as ebl
import synth

pytestmark = pytest.mark.gpu


def test_bounded_wait_times_out_and_context_survives(cuda_device):
    dev = cuda_device
    st = torch.zeros(1, dtype=torch.int32, device=dev)
    torch.cuda.synchronize()
    t0 = time.perf_counter()
    ebl.selftest_wait_timeout(st, limit_us=20000)
    torch.cuda.synchronize()
    dt = time.perf_counter() - t0
    assert int(st.item()) == ebl.EBL_ST_TIMEOUT
    assert 0.015 <= dt < 5.0
    # the context is still usable: a normal router call succeeds afterwards
    T, d, Nr, K = 256, 128, 64, 4
    h = synth.hidden_normal(T, d, seed=1, device=dev)
    W = synth.router_weight(Nr, d, seed=2).to(dev)
    counts = torch.zeros(Nr, dtype=torch.int32, device=dev)
    st.zero_()
    idx, g = ebl.router_forward(h, W, torch.zeros(Nr, device=dev), K, counts, status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0 and int(counts.sum().item()) == T * K


def _run_steps(h_steps, W, b, m, K):
    counts = torch.zeros(W.shape[0], dtype=torch.int32, device=W.device)
    for h in h_steps:
        ebl.router_forward(h, W, b, K, counts)
        ebl.smebu_step(counts, b, m, reset_counts=True)
    torch.cuda.synchronize()


def test_checkpoint_resume_is_bit_identical(cuda_device):
    """Stop after 15 of 30 steps, save bias and momentum, restore, finish: the
    final state equals an uninterrupted run bit for bit."""
    dev = cuda_device
    T, d, Nr, K = 2048, 256, 64, 4
    W = synth.router_weight(Nr, d, seed=3).to(dev)
    hs = [synth.hidden_normal(T, d, seed=100 + s, device=dev) for s in range(30)]
    b = torch.zeros(Nr, device=dev)
    m = torch.zeros(Nr, device=dev)
    _run_steps(hs, W, b, m, K)
    b2 = torch.zeros(Nr, device=dev)
    m2 = torch.zeros(Nr, device=dev)
    _run_steps(hs[:15], W, b2, m2, K)
    buf = io.BytesIO()
    torch.save({"expert_bias": b2.cpu(), "momentum": m2.cpu()}, buf)
    buf.seek(0)
    state = torch.load(buf)
    b3 = state["expert_bias"].to(dev)
    m3 = state["momentum"].to(dev)
    _run_steps(hs[15:], W, b3, m3, K)
    assert torch.equal(b, b3) and torch.equal(m, m3)
    assert float(b.abs().max()) > 0
