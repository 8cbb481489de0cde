"""SMEBU, the sign update and MaxVio on a B200 against the oracle."""
import math

import numpy as np
import pytest
import torch

import expert_bias_load_b200 as ebl
import oracle
import synth
from tests.parity import STATE_RTOL, rel_err, to_np

pytestmark = pytest.mark.gpu


def _random_counts(rng, Nr, total, skew):
    p = rng.dirichlet(np.full(Nr, skew))
    n = rng.multinomial(total, p)
    return n.astype(np.int64)


@pytest.mark.parametrize("Nr", [1, 7, 64, 128, 256])
def test_smebu_open_loop_200_steps(cuda_device, Nr):
    rng = np.random.default_rng(Nr)
    dev = cuda_device
    b_o = np.zeros(Nr, np.float32)
    m_o = np.zeros(Nr, np.float32)
    b_o[: min(8, Nr)] = -1.0
    b_g = torch.from_numpy(b_o.copy()).to(dev)
    m_g = torch.zeros(Nr, device=dev)
    mv = torch.zeros(1, device=dev)
    exact = 0
    for step in range(200):
        n = _random_counts(rng, Nr, 4 * 4096, 0.3 if step < 50 else 5.0)
        if step % 37 == 5:
            n[:] = 100                       # exact balance: step is 0
        c = torch.from_numpy(n.astype(np.int32)).to(dev)
        ebl.smebu_step(c, b_g, m_g, maxvio=mv)
        _, mvo = oracle.smebu(n, b_o, m_o)
        gb, gm = to_np(b_g), to_np(m_g)
        assert rel_err(gb, b_o).max() <= STATE_RTOL, step
        assert rel_err(gm, m_o).max() <= STATE_RTOL, step
        exact += int(np.array_equal(gb, b_o) and np.array_equal(gm, m_o))
        g = float(mv.item())
        assert (g == mvo) or (math.isinf(g) and math.isinf(mvo))
    assert exact >= 198      # fp64 tanh of two libraries may differ in the last bit, rarely


def test_smebu_reset_and_empty_load(cuda_device):
    dev = cuda_device
    Nr = 32
    b = torch.randn(Nr, device=dev) * 1e-3
    m = torch.randn(Nr, device=dev) * 1e-4
    b0, m0 = b.clone(), m.clone()
    c = torch.zeros(Nr, dtype=torch.int32, device=dev)
    st = torch.zeros(1, dtype=torch.int32, device=dev)
    mv = torch.zeros(1, device=dev)
    ebl.smebu_step(c, b, m, maxvio=mv, status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == ebl.EBL_ST_EMPTY_LOAD
    assert torch.equal(b, b0) and torch.equal(m, m0)
    c = torch.arange(1, Nr + 1, dtype=torch.int32, device=dev)
    st.zero_()
    ebl.smebu_step(c, b, m, reset_counts=True, maxvio=mv, status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0 and int(c.abs().sum().item()) == 0
    assert float(mv.item()) == np.float32(32.0)


@pytest.mark.parametrize("linear", [False, True])
def test_smebu_layers(cuda_device, linear):
    rng = np.random.default_rng(7 + linear)
    dev = cuda_device
    L, Nr = 5, 96
    b_o = np.zeros((L, Nr), np.float32)
    m_o = np.zeros((L, Nr), np.float32)
    b_g = torch.zeros(L, Nr, device=dev)
    m_g = torch.zeros(L, Nr, device=dev)
    mv = torch.zeros(L, device=dev)
    for step in range(30):
        n = np.stack([_random_counts(rng, Nr, 8192, 0.5 + l) for l in range(L)])
        c = torch.from_numpy(n.astype(np.int32)).to(dev)
        ebl.smebu_step_layers(c, b_g, m_g, linear=linear, maxvio=mv)
        for l in range(L):
            bl, ml = b_o[l].copy(), m_o[l].copy()
            if linear:
                oracle.smebu_linear(n[l], bl, ml)
            else:
                oracle.smebu(n[l], bl, ml)
            b_o[l], m_o[l] = bl, ml
        assert rel_err(to_np(b_g), b_o).max() <= STATE_RTOL
        assert rel_err(to_np(m_g), m_o).max() <= STATE_RTOL
    mvo = [oracle.maxvio(n[l])[0] for l in range(L)]
    assert np.allclose(to_np(mv), np.array(mvo, np.float32))


@pytest.mark.parametrize("Nr", [8, 128, 256])
def test_sign_update_open_loop(cuda_device, Nr):
    rng = np.random.default_rng(100 + Nr)
    dev = cuda_device
    b_o = (rng.standard_normal(Nr) * 1e-3).astype(np.float32)
    b_g = torch.from_numpy(b_o.copy()).to(dev)
    mv = torch.zeros(1, device=dev)
    for step in range(50):
        n = _random_counts(rng, Nr, 8 * 65536, 2.0)
        c = torch.from_numpy(n.astype(np.int32)).to(dev)
        ebl.sign_update_step(c, b_g, 1e-3, maxvio=mv)
        _, mvo = oracle.sign_update(n, b_o, 1e-3)
        assert np.array_equal(to_np(b_g), b_o), step
        assert float(mv.item()) == mvo or (math.isinf(mvo) and math.isinf(float(mv.item())))
    assert abs(to_np(b_g).astype(np.float64).sum()) < Nr * 1e-9


@pytest.mark.parametrize("update", ["smebu", "sign"])
def test_closed_loop_logits_mode(cuda_device, update):
    """Router (logits mode) -> bias update -> router ... for 100 steps: the
    counts are bit-exact every step, so the trajectories must agree."""
    dev = cuda_device
    T, Nr, K = 16384 + 3, 256, 4
    b_o = synth.dead_start_bias(Nr).numpy()
    m_o = np.zeros(Nr, np.float32)
    b_g = torch.from_numpy(b_o.copy()).to(dev)
    m_g = torch.zeros(Nr, device=dev)
    counts = torch.zeros(Nr, dtype=torch.int32, device=dev)
    mvs = []
    for step in range(100):
        x = synth.logits_normal(T, Nr, seed=synth.step_seed("ties", step), quant8=True)
        ebl.router_forward_logits(x.to(dev), b_g, K, counts)
        ref = oracle.router_logits(x.numpy(), b_o, K)
        n_g = to_np(counts).astype(np.int64)
        assert np.array_equal(n_g, ref.counts), step
        mv = torch.zeros(1, device=dev)
        if update == "smebu":
            ebl.smebu_step(counts, b_g, m_g, reset_counts=True, maxvio=mv)
            oracle.smebu(ref.counts, b_o, m_o)
        else:
            ebl.sign_update_step(counts, b_g, 1e-3, reset_counts=True, maxvio=mv)
            oracle.sign_update(ref.counts, b_o, 1e-3)
        assert rel_err(to_np(b_g), b_o).max() <= STATE_RTOL, step
        assert rel_err(to_np(m_g), m_o).max() <= STATE_RTOL, step
        mvs.append(float(mv.item()))
    assert math.isinf(mvs[0])            # the dead-start experts get no load at step 0
