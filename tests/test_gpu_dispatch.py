"""Dispatch and combine on a B200 against the oracle."""
import numpy as np
import pytest
import torch

import expert_bias_load_b200 as ebl
import oracle
import synth
from tests.parity import to_np

pytestmark = pytest.mark.gpu


def _topk_ids(T, K, Nr, seed, skew=None):
    g = torch.Generator().manual_seed(seed)
    if skew is None:
        w = torch.ones(Nr)
    else:
        w = torch.rand(Nr, generator=g) ** skew + 1e-3
    return torch.multinomial(w.expand(T, Nr), K, replacement=False, generator=g).to(torch.int32)


CASES = [
    # T, d, Nr, K, use the router's tile counts
    (4096 + 33, 512, 256, 4, False),
    (4096 + 33, 512, 256, 4, True),
    (1, 64, 8, 8, False),
    (127, 24, 16, 3, False),
    (5000, 136, 64, 2, True),
    (3000, 1024, 128, 8, False),
    (700, 8256, 32, 2, False),           # rows of 16.5 KB: copied in 8 KB + 8 KB + 128 B pieces
]


@pytest.mark.parametrize("T,d,Nr,K,with_tiles", CASES)
def test_dispatch_combine_vs_oracle(cuda_device, T, d, Nr, K, with_tiles):
    dev = cuda_device
    idx = _topk_ids(T, K, Nr, seed=T + K, skew=4.0)
    h = synth.hidden_normal(T, d, seed=T + d)
    tiles = None
    if with_tiles:
        tc = np.zeros(((T + 127) // 128, Nr), np.int32)
        for j in range(tc.shape[0]):
            tc[j] = np.bincount(idx[j * 128:(j + 1) * 128].numpy().ravel(), minlength=Nr)
        tiles = torch.from_numpy(tc).to(dev)
    st = torch.zeros(1, dtype=torch.int32, device=dev)
    offsets, perm, dest, X = ebl.moe_dispatch(h.to(dev), idx.to(dev), Nr, tile_counts=tiles, status=st)
    torch.cuda.synchronize()
    o_off, o_perm, o_dest = oracle.dispatch(idx.numpy(), Nr)
    assert int(st.item()) == 0
    assert np.array_equal(to_np(offsets), o_off)
    assert np.array_equal(to_np(perm), o_perm)
    assert np.array_equal(to_np(dest), o_dest)
    hb = h.view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(to_np(X.view(torch.int16)).view(np.uint16), oracle.gather_rows(hb, o_perm))
    # combine with normalised gates: identity expert
    g = torch.rand(T, K, generator=torch.Generator().manual_seed(1)) + 0.05
    g = (g / g.sum(1, keepdim=True)).float()
    out = ebl.moe_combine(X, g.to(dev), dest, status=st)
    torch.cuda.synchronize()
    o64, o32 = oracle.combine(to_np(X.view(torch.int16)).view(np.uint16), g.numpy(), o_dest)
    assert int(st.item()) == 0
    assert np.array_equal(to_np(out).view(np.uint32), o32.view(np.uint32))   # same fma chain
    hd = h.float().numpy().astype(np.float64)
    assert np.allclose(to_np(out), hd, rtol=(2 * K + 1) * 2.0 ** -24, atol=0)
    assert np.allclose(o64, hd, rtol=(K + 1) * 2.0 ** -24, atol=0)


def test_dispatch_bad_expert_sets_status(cuda_device):
    dev = cuda_device
    T, d, Nr, K = 300, 64, 16, 2
    idx = _topk_ids(T, K, Nr, seed=9)
    idx[7, 1] = 16
    idx[200, 0] = -3
    h = synth.hidden_normal(T, d, seed=1)
    st = torch.zeros(1, dtype=torch.int32, device=dev)
    offsets, perm, dest, X = ebl.moe_dispatch(h.to(dev), idx.to(dev), Nr, status=st)
    torch.cuda.synchronize()
    assert int(st.item()) & ebl.EBL_ST_BAD_EXPERT
    d_np = to_np(dest)
    assert d_np[7 * K + 1] == -1 and d_np[200 * K + 0] == -1
    assert int(to_np(offsets)[-1]) == T * K - 2


def test_combine_bad_dest_sets_status(cuda_device):
    dev = cuda_device
    T, d, K = 64, 32, 2
    Y = synth.hidden_normal(T * K, d, seed=2).to(dev)
    dest = torch.arange(T * K, dtype=torch.int32, device=dev)
    dest[5] = T * K
    dest[6] = -1
    g = torch.full((T, K), 0.5, device=dev)
    st = torch.zeros(1, dtype=torch.int32, device=dev)
    out = ebl.moe_combine(Y, g, dest, status=st)
    torch.cuda.synchronize()
    assert int(st.item()) & ebl.EBL_ST_BAD_DEST
    assert torch.isfinite(out).all()


def test_router_then_dispatch_with_router_tiles(cuda_device):
    """router_forward's tile_counts feed moe_dispatch (the fused path)."""
    dev = cuda_device
    T, d, Nr, K = 2048 + 300, 256, 64, 4
    h = synth.hidden_normal(T, d, seed=11).to(dev)
    W = synth.router_weight(Nr, d, seed=12).to(dev)
    counts = torch.zeros(Nr, dtype=torch.int32, device=dev)
    tiles = torch.empty(((T + 127) // 128, Nr), dtype=torch.int32, device=dev)
    idx, gates = ebl.router_forward(h, W, torch.zeros(Nr, device=dev), K, counts, tile_counts=tiles)
    offsets, perm, dest, X = ebl.moe_dispatch(h, idx, Nr, tile_counts=tiles)
    torch.cuda.synchronize()
    o_off, o_perm, o_dest = oracle.dispatch(to_np(idx), Nr)
    assert np.array_equal(to_np(offsets), o_off)
    assert np.array_equal(to_np(perm), o_perm) and np.array_equal(to_np(dest), o_dest)
    assert np.array_equal(np.diff(o_off), to_np(counts))
    out = ebl.moe_combine(X, gates, dest)
    assert torch.allclose(out, h.float(), rtol=1e-6, atol=0)


def test_dispatch_inconsistent_tile_counts_sets_status(cuda_device):
    """Tile counts that do not belong to topk_idx (host-side fault injection):
    the call reports EBL_ST_BAD_COUNTS and writes nothing out of bounds."""
    dev = cuda_device
    T, d, Nr, K = 1000, 64, 32, 2
    idx = _topk_ids(T, K, Nr, seed=21).to(dev)
    h = synth.hidden_normal(T, d, seed=22).to(dev)
    tiles = torch.zeros(((T + 127) // 128, Nr), dtype=torch.int32, device=dev)
    tiles[:, 0] = 500                              # far too many pairs for expert 0
    X = torch.zeros((T * K, d), dtype=torch.bfloat16, device=dev)
    guard = torch.full((4096,), 7, dtype=torch.int16, device=dev)
    st = torch.zeros(1, dtype=torch.int32, device=dev)
    offsets, perm, dest, X = ebl.moe_dispatch(h, idx, Nr, tile_counts=tiles, dispatched=X, status=st)
    torch.cuda.synchronize()
    assert int(st.item()) & ebl.EBL_ST_BAD_COUNTS
    dn = to_np(dest)
    assert np.all((dn == -1) | ((dn >= 0) & (dn < T * K)))
    assert torch.all(guard == 7)


@pytest.mark.parametrize("T,d,K", [(1000, 1024, 4), (333, 136, 3), (64, 8, 8), (257, 4096, 1)])
def test_combine_distinct_expert_outputs_vs_oracle(cuda_device, T, d, K):
    """Every slot of a token reads a different expert-output row (random rows,
    a random permutation as dest, gates that do not sum to 1), so a slot read
    from the wrong row or a dropped slot changes the result; bit-exact against
    the oracle's fp32 fma chain in slot order."""
    dev = cuda_device
    g0 = torch.Generator().manual_seed(T + d + K)
    Y = synth.hidden_normal(T * K, d, seed=T * 3 + K)
    dest = torch.randperm(T * K, generator=g0).to(torch.int32)
    gates = (torch.rand(T, K, generator=g0) * 2.0 - 0.5).float()
    st = torch.zeros(1, dtype=torch.int32, device=dev)
    out = ebl.moe_combine(Y.to(dev), gates.to(dev), dest.to(dev), status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    yb = Y.view(torch.int16).numpy().view(np.uint16)
    _, o32 = oracle.combine(yb, gates.numpy(), dest.numpy())
    assert np.array_equal(to_np(out).view(np.uint32), o32.view(np.uint32))


def test_empty_batch_is_a_no_op(cuda_device):
    """T = 0 through the binding (empty tensors have no storage): the router
    modes and combine launch nothing and leave counts alone; dispatch zeroes
    the offsets."""
    dev = cuda_device
    Nr, K, d = 64, 4, 256
    counts = torch.arange(Nr, dtype=torch.int32, device=dev)
    before = counts.clone()
    W = synth.router_weight(Nr, d, seed=1).to(dev)
    bias = torch.zeros(Nr, device=dev)
    h = torch.empty(0, d, dtype=torch.bfloat16, device=dev)
    idx, g = ebl.router_forward(h, W, bias, K, counts)
    assert idx.shape == (0, K) and g.shape == (0, K)
    idx, g = ebl.router_forward_logits(torch.empty(0, Nr, device=dev), bias, K, counts)
    assert idx.shape == (0, K)
    offsets, perm, dest, X = ebl.moe_dispatch(h, idx, Nr, offsets=torch.full((Nr + 1,), 7, dtype=torch.int32,
                                                                             device=dev))
    out = ebl.moe_combine(X, g, dest)
    torch.cuda.synchronize()
    assert torch.equal(counts, before)
    assert int(offsets.abs().sum().item()) == 0
    assert perm.numel() == 0 and X.shape == (0, d) and out.shape == (0, d)
