"""Seeded random shapes through every mode against the oracle (small sizes):
logits mode bit-exact (both kernels: aligned and misaligned logits), GEMM mode
under the near-tie rule, dispatch and combine bit-exact, the bias updates
(SMEBU clamped and linear over several layers, the sign update), and the
sequence-wise balance statistics (GEMM mode, and logits mode fused into the
routing pass).  Each case
draws its sizes, the bias pattern and the value distribution from its own seed."""
import numpy as np
import pytest
import torch

import expert_bias_load_b200 as ebl
import oracle
import synth
from tests.parity import assert_gemm_parity, tile_hist, to_np

pytestmark = pytest.mark.gpu

CASES = list(range(24))


def _bias(rng, Nr):
    kind = rng.integers(0, 4)
    if kind == 0:
        return np.zeros(Nr, np.float32)
    if kind == 1:
        return (rng.standard_normal(Nr) * 0.02).astype(np.float32)
    if kind == 2:
        return (rng.integers(-2, 3, Nr) * 0.125).astype(np.float32)      # ties on a 1/8 grid
    b = np.zeros(Nr, np.float32)
    b[rng.choice(Nr, min(8, Nr - 1), replace=False)] = -1.0                # dead-start
    return b


@pytest.mark.parametrize("case", CASES)
def test_logits_mode_random_shapes(cuda_device, case):
    rng = np.random.default_rng(1000 + case)
    T = int(rng.integers(1, 3000))
    Nr = int(rng.choice([int(rng.integers(1, 257)), 4 * int(rng.integers(1, 65))]))
    K = int(rng.integers(1, min(8, Nr) + 1))
    scale = float(rng.choice([1.0, 4.0, 0.125]))
    x = (rng.standard_normal((T, Nr)) * scale).astype(np.float32)
    if rng.integers(0, 2):
        x = np.round(x * 8) / 8                                            # exact ties are common
    b = _bias(rng, Nr)
    dev = cuda_device
    misalign = bool(rng.integers(0, 2))
    if misalign:
        buf = torch.empty(T * Nr + 1, dtype=torch.float32, device=dev)
        buf[1:] = torch.from_numpy(x.reshape(-1)).to(dev)
        xd = buf[1:].view(T, Nr)
    else:
        xd = torch.from_numpy(x).to(dev)
    counts = torch.zeros(Nr, dtype=torch.int32, device=dev)
    tiles = torch.full(((T + 127) // 128, Nr), -1, dtype=torch.int32, device=dev)
    idx, g = ebl.router_forward_logits(xd, torch.from_numpy(b).to(dev), K, counts, tile_counts=tiles)
    torch.cuda.synchronize()
    ref = oracle.router_logits(x, b, K, tile_tokens=128)
    assert np.array_equal(to_np(idx), ref.idx), (T, Nr, K, misalign)
    assert np.array_equal(to_np(g).view(np.uint32), ref.gates.view(np.uint32))
    assert np.array_equal(to_np(counts), ref.counts)
    assert np.array_equal(to_np(tiles), ref.tile_counts)


@pytest.mark.parametrize("case", CASES[:12])
def test_gemm_mode_random_shapes(cuda_device, case):
    rng = np.random.default_rng(2000 + case)
    T = int(rng.integers(1, 2500))
    Nr = 32 * int(rng.integers(1, 9))
    K = int(rng.integers(1, min(8, Nr) + 1))
    d = 64 * int(rng.integers(1, 17))
    dev = cuda_device
    h = synth.hidden_normal(T, d, seed=3000 + case, quant8=bool(rng.integers(0, 2)))
    W = synth.router_weight(Nr, d, seed=4000 + case)
    b = _bias(rng, Nr)
    counts = torch.zeros(Nr, dtype=torch.int32, device=dev)
    tiles = torch.full(((T + 127) // 128, Nr), -1, dtype=torch.int32, device=dev)
    idx, g = ebl.router_forward(h.to(dev), W.to(dev), torch.from_numpy(b).to(dev), K, counts, tile_counts=tiles)
    torch.cuda.synchronize()
    ref = oracle.router_gemm(h, W, b, K, want_scores=True)
    gi = to_np(idx)
    assert_gemm_parity(gi, to_np(g), ref, Nr, b, gpu_counts=to_np(counts))
    assert np.array_equal(to_np(tiles), tile_hist(gi, Nr))


@pytest.mark.parametrize("case", CASES[:12])
def test_dispatch_combine_random_shapes(cuda_device, case):
    rng = np.random.default_rng(5000 + case)
    T = int(rng.integers(1, 4000))
    Nr = int(rng.integers(1, 257))
    K = int(rng.integers(1, min(8, Nr) + 1))
    d = 8 * int(rng.integers(1, 300))
    dev = cuda_device
    w = rng.random(Nr) ** 4 + 1e-3
    idx = np.stack([rng.choice(Nr, K, replace=False, p=w / w.sum()) for _ in range(T)]).astype(np.int32)
    h = synth.hidden_normal(T, d, seed=6000 + case)
    with_tiles = bool(rng.integers(0, 2))
    tiles = torch.from_numpy(tile_hist(idx, Nr)).to(dev) if with_tiles else None
    st = torch.zeros(1, dtype=torch.int32, device=dev)
    offsets, perm, dest, X = ebl.moe_dispatch(h.to(dev), torch.from_numpy(idx).to(dev), Nr, tile_counts=tiles,
                                              status=st)
    g = (rng.random((T, K)) * 2 - 0.5).astype(np.float32)
    Y = synth.hidden_normal(T * K, d, seed=7000 + case)                  # expert outputs differ per slot
    out = ebl.moe_combine(Y.to(dev), torch.from_numpy(g).to(dev), dest, status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    o_off, o_perm, o_dest = oracle.dispatch(idx, Nr)
    assert np.array_equal(to_np(offsets), o_off)
    assert np.array_equal(to_np(perm), o_perm)
    assert np.array_equal(to_np(dest), o_dest)
    hb = h.view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(to_np(X.view(torch.int16)).view(np.uint16), oracle.gather_rows(hb, o_perm))
    _, o32 = oracle.combine(Y.view(torch.int16).numpy().view(np.uint16), g, o_dest)
    assert np.array_equal(to_np(out).view(np.uint32), o32.view(np.uint32))


@pytest.mark.parametrize("case", range(16))
def test_bias_updates_random(cuda_device, case):
    """SMEBU (clamped and linear) for several layers and the sign update, on
    random loads (dead experts, skew, an empty layer), random starting state
    and random fp32 hyper-parameters: bias and momentum within 1e-6 relative
    of the oracle (bit-identical in practice), MaxVio exact, loads reset."""
    from tests.parity import STATE_RTOL, rel_err
    rng = np.random.default_rng(8000 + case)
    dev = cuda_device
    f32 = lambda v: float(np.float32(v))
    L, Nr = int(rng.integers(1, 9)), int(rng.integers(1, 257))
    lam, beta, kappa = f32(10 ** rng.uniform(-5, -2)), f32(rng.uniform(0, 0.99)), f32(rng.uniform(0.5, 4))
    gamma = f32(10 ** rng.uniform(-4, -2))
    linear = case % 3 == 0
    counts = (rng.pareto(1.5, (L, Nr)) * 50).astype(np.int64)
    counts[:, rng.choice(Nr, Nr // 10, replace=False)] = 0                 # dead experts
    if case % 5 == 1:
        counts[0] = 0                                                     # an empty layer
    b0 = (rng.standard_normal((L, Nr)) * 0.1).astype(np.float32)
    m0 = (rng.standard_normal((L, Nr)) * 1e-3).astype(np.float32)
    c_d = torch.from_numpy(counts.astype(np.int32)).to(dev)
    b_d, m_d = torch.from_numpy(b0.copy()).to(dev), torch.from_numpy(m0.copy()).to(dev)
    mv = torch.zeros(L, device=dev)
    st = torch.zeros(1, dtype=torch.int32, device=dev)
    ebl.smebu_step_layers(c_d, b_d, m_d, lam, beta, kappa, linear=linear, reset_counts=True, maxvio=mv, status=st)
    torch.cuda.synchronize()
    empty = False
    for l in range(L):
        b, m = b0[l].copy(), m0[l].copy()
        if linear:
            rc, mvo = oracle.smebu_linear(counts[l], b, m, lam, beta)
        else:
            rc, mvo = oracle.smebu(counts[l], b, m, lam, beta, kappa)
        empty |= rc != 0
        assert rel_err(to_np(b_d[l]), b).max() <= STATE_RTOL, l
        assert rel_err(to_np(m_d[l]), m).max() <= STATE_RTOL, l
        assert np.float32(mvo).tobytes() == to_np(mv[l:l + 1]).tobytes(), (l, mvo, float(mv[l]))
    assert bool(int(st.item()) & ebl.EBL_ST_EMPTY_LOAD) == empty
    assert int(c_d.abs().sum().item()) == 0
    # the sign update of the smaller models, on layer L-1's loads
    c1 = torch.from_numpy(counts[-1].astype(np.int32)).to(dev)
    b1 = torch.from_numpy(b0[-1].copy()).to(dev)
    mv1 = torch.zeros(1, device=dev)
    ebl.sign_update_step(c1, b1, gamma, maxvio=mv1)
    torch.cuda.synchronize()
    b = b0[-1].copy()
    rc, mvo = oracle.sign_update(counts[-1], b, gamma)
    assert rel_err(to_np(b1), b).max() <= STATE_RTOL
    assert np.float32(mvo).tobytes() == to_np(mv1).tobytes()


@pytest.mark.parametrize("case", range(8))
def test_balance_option_random_shapes(cuda_device, case):
    """GEMM mode with the balance option on random shapes: tile_psum against
    the oracle's per-tile sums, and the loss over random sequence lengths."""
    from tests.test_gpu_seq_balance import PSUM_ATOL, PSUM_RTOL
    rng = np.random.default_rng(9000 + case)
    S = 128 * int(rng.integers(1, 5))
    T = S * int(rng.integers(1, 6))
    Nr = 32 * int(rng.integers(1, 9))
    K = int(rng.integers(1, min(8, Nr) + 1))
    d = 64 * int(rng.integers(1, 17))
    dev = cuda_device
    h = synth.hidden_normal(T, d, seed=9100 + case, quant8=bool(rng.integers(0, 2)))
    W = synth.router_weight(Nr, d, seed=9200 + case)
    b = _bias(rng, Nr)
    counts = torch.zeros(Nr, dtype=torch.int32, device=dev)
    tc = torch.empty(T // 128, Nr, dtype=torch.int32, device=dev)
    tp = torch.empty(T // 128, Nr, device=dev)
    alpha = float(np.float32(10 ** rng.uniform(-5, -3)))
    ebl.router_forward_balance(h.to(dev), W.to(dev), torch.from_numpy(b).to(dev), K, counts, tc, tp)
    loss, loss_seq = ebl.seq_balance_loss(tc, tp, T, K, S, alpha)
    torch.cuda.synchronize()
    ref = oracle.router_gemm(h, W, b, K, want_scores=True)
    want = oracle.tile_psum(ref.scores, 128)
    assert np.all(np.abs(to_np(tp).astype(np.float64) - want) <= PSUM_RTOL * want + PSUM_ATOL)
    r = oracle.seq_balance(ref.scores, ref.idx, S, alpha)
    excused = (ref.gap < 1e-3).reshape(T // S, S).sum(1)
    assert np.all(np.abs(to_np(loss_seq) - r.loss_seq) <= 2e-5 * r.loss_seq + excused * alpha * Nr / S)


@pytest.mark.parametrize("case", list(range(12)))
def test_logits_mode_fused_balance_random_shapes(cuda_device, case):
    """router_forward_logits_balance on seeded random shapes: routing bit for
    bit that of router_forward_logits and the oracle's, the per-tile statistics
    within the fused tolerance (2^-16 relative + 2^-60) of the oracle's fp64
    sums of the rounded-once scores."""
    rng = np.random.default_rng(3000 + case)
    T = int(rng.integers(1, 3000))
    Nr = int(rng.choice([int(rng.integers(1, 257)), 4 * int(rng.integers(1, 65))]))
    K = int(rng.integers(1, min(8, Nr) + 1))
    scale = float(rng.choice([1.0, 4.0, 0.125]))
    x = (rng.standard_normal((T, Nr)) * scale).astype(np.float32)
    if rng.integers(0, 2):
        x = np.round(x * 8) / 8
    b = _bias(rng, Nr)
    dev = cuda_device
    misalign = bool(rng.integers(0, 2))
    if misalign:
        buf = torch.empty(T * Nr + 1, dtype=torch.float32, device=dev)
        buf[1:] = torch.from_numpy(x.reshape(-1)).to(dev)
        xd = buf[1:].view(T, Nr)
    else:
        xd = torch.from_numpy(x).to(dev)
    bd = torch.from_numpy(b).to(dev)
    tiles_n = (T + 127) // 128
    counts = torch.zeros(Nr, dtype=torch.int32, device=dev)
    tc = torch.full((tiles_n, Nr), -1, dtype=torch.int32, device=dev)
    tp = torch.full((tiles_n, Nr), -1.0, device=dev)
    idx, g = ebl.router_forward_logits_balance(xd, bd, K, counts, tc, tp)
    c2 = torch.zeros(Nr, dtype=torch.int32, device=dev)
    tc2 = torch.empty_like(tc)
    idx2, g2 = ebl.router_forward_logits(xd, bd, K, c2, tile_counts=tc2)
    torch.cuda.synchronize()
    assert torch.equal(idx, idx2) and torch.equal(g, g2) and torch.equal(counts, c2) and torch.equal(tc, tc2)
    ref = oracle.router_logits(x, b, K, tile_tokens=128, want_scores=True)
    assert np.array_equal(to_np(idx), ref.idx), (T, Nr, K, misalign)
    assert np.array_equal(to_np(tc), ref.tile_counts)
    want = oracle.tile_psum(ref.scores.astype(np.float64), 128)
    got = to_np(tp).astype(np.float64)
    assert np.all(np.abs(got - want) <= 2.0 ** -16 * want + 2.0 ** -60), (T, Nr, K, misalign)
