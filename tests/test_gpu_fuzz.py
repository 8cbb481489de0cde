"""Seeded random shapes through every mode against the oracle (small sizes):
logits mode bit-exact (both kernels: aligned and misaligned logits), GEMM mode
under the near-tie rule, dispatch and combine bit-exact.  Each case draws T,
N_r, K, d, the bias pattern and the value distribution from its own seed."""
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
