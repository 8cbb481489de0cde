"""Full-size workloads in the launch configuration the benchmark times,
checked on sampled rows against the oracle and on properties that hold at any
size (the oracle cannot redo a billion-row GEMM in a test)."""
import numpy as np
import pytest
import torch

import expert_bias_load_b200 as ebl
import oracle
import synth
from tests.parity import assert_gemm_parity, to_np

pytestmark = pytest.mark.gpu

SAMPLE_ROWS = 8192


def _sampled_parity(h_dev, W, bias, K, idx, gates, seed):
    T = h_dev.shape[0]
    g = torch.Generator().manual_seed(seed)
    rows = torch.randperm(T, generator=g)[:SAMPLE_ROWS]
    rows = torch.cat([rows, torch.tensor([0, T - 1])]).sort().values
    hs = h_dev[rows.to(h_dev.device)].cpu()
    ref = oracle.router_gemm(hs, W.cpu(), bias.cpu().numpy(), K, want_scores=True)
    r = rows.numpy()
    return assert_gemm_parity(to_np(idx)[r], to_np(gates)[r], ref, W.shape[0], bias.cpu().numpy())


@pytest.mark.parametrize("name", ["mid", "drift", "ties"])
def test_router_full_size_sampled(cuda_device, name):
    cfg = synth.WORKLOADS[name]
    T, d, Nr, K = cfg["T"], cfg["d"], cfg["Nr"], cfg["K"]
    dev = cuda_device
    W = synth.router_weight(Nr, d, seed=synth.BASE_SEED + d).to(dev)
    seed = synth.step_seed(name, 0)
    if name == "drift":
        h = synth.hidden_drift(T, d, W, seed=seed, mu=2.0, device=dev)
    else:
        h = synth.hidden_normal(T, d, seed=seed, device=dev, quant8=(name == "ties"))
    bias = synth.dead_start_bias(Nr, device=dev) if name == "ties" else torch.zeros(Nr, device=dev)
    counts = torch.zeros(Nr, dtype=torch.int32, device=dev)
    st = torch.zeros(1, dtype=torch.int32, device=dev)
    idx, gates = ebl.router_forward(h, W, bias, K, counts, status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    _sampled_parity(h, W, bias, K, idx, gates, seed=T)
    # properties over all T rows
    hist = torch.bincount(idx.view(-1).long(), minlength=Nr)
    assert torch.equal(hist.to(torch.int32), counts)
    assert int(counts.sum().item()) == T * K
    srt = idx.sort(dim=1).values
    assert bool((srt[:, 1:] != srt[:, :-1]).all()) if K > 1 else True      # distinct experts per token
    gs = gates.double().sum(1)
    assert float((gs - 1).abs().max()) < K * 2e-7
    assert bool((gates > 0).all())
    if name == "ties":
        assert int(counts[:8].sum().item()) == 0     # bias -1 keeps the 8 dead-start experts out


def test_balance_option_full_tie_workload(cuda_device):
    """The balance option on the 1M-token tie workload (the benchmark's
    launch): routing bit-identical to router_forward; every tile's sums of
    s / total equal its 128 tokens; sampled tiles and one whole 4096-token
    sequence against the oracle (tolerances as in test_gpu_seq_balance)."""
    from tests.test_gpu_seq_balance import PSUM_ATOL, PSUM_RTOL
    cfg = synth.WORKLOADS["ties"]
    T, d, Nr, K, S = cfg["T"], cfg["d"], cfg["Nr"], cfg["K"], 4096
    dev = cuda_device
    W = synth.router_weight(Nr, d, seed=synth.BASE_SEED + d).to(dev)
    h = synth.hidden_normal(T, d, seed=synth.step_seed("ties", 0), device=dev, quant8=True)
    bias = synth.dead_start_bias(Nr, device=dev)
    tiles = T // 128
    c1 = torch.zeros(Nr, dtype=torch.int32, device=dev)
    c2 = torch.zeros(Nr, dtype=torch.int32, device=dev)
    tc = torch.empty(tiles, Nr, dtype=torch.int32, device=dev)
    tp = torch.empty(tiles, Nr, device=dev)
    idx, gates = ebl.router_forward_balance(h, W, bias, K, c1, tc, tp)
    loss, loss_seq = ebl.seq_balance_loss(tc, tp, T, K, S, ebl.SEQ_BALANCE_ALPHA)
    i2, g2 = ebl.router_forward(h, W, bias, K, c2)
    torch.cuda.synchronize()
    assert torch.equal(idx, i2) and torch.equal(gates, g2) and torch.equal(c1, c2)
    assert float((tp.double().sum(1) - 128).abs().max()) < 128 * 1e-5
    sample = sorted({0, tiles - 1} | set(np.random.default_rng(3).choice(tiles, 6, replace=False).tolist()))
    rows = torch.cat([torch.arange(j * 128, (j + 1) * 128) for j in sample])
    ref = oracle.router_gemm(h[rows.to(dev)].cpu(), W.cpu(), bias.cpu().numpy(), K, want_scores=True)
    want = oracle.tile_psum(ref.scores, 128)
    got = to_np(tp)[sample].astype(np.float64)
    assert np.all(np.abs(got - want) <= PSUM_RTOL * want + PSUM_ATOL)
    # the last sequence end to end
    b = T // S - 1
    hs = h[b * S:(b + 1) * S].cpu()
    ref = oracle.router_gemm(hs, W.cpu(), bias.cpu().numpy(), K, want_scores=True)
    r = oracle.seq_balance(ref.scores, ref.idx, S, ebl.SEQ_BALANCE_ALPHA)
    excused = int((ref.gap < 1e-3).sum())
    got = float(loss_seq[b].item())
    assert abs(got - r.loss) <= 2e-5 * r.loss + excused * ebl.SEQ_BALANCE_ALPHA * Nr / S, (got, r.loss, excused)
    assert abs(float(loss.item()) - float(loss_seq.mean().item())) <= 1e-15 * float(loss.item())


def test_logits_mode_full_tie_workload(cuda_device):
    """The tie workload in logits mode at full size: bit-exact against the
    oracle, and the sequence-wise balance loss within one fp32 rounding."""
    cfg = synth.WORKLOADS["ties"]
    T, Nr, K = cfg["T"], cfg["Nr"], cfg["K"]
    dev = cuda_device
    x = synth.logits_normal(T, Nr, seed=synth.step_seed("ties", 1), quant8=True, device=dev)
    bias = synth.dead_start_bias(Nr, device=dev)
    counts = torch.zeros(Nr, dtype=torch.int32, device=dev)
    tiles = torch.empty(((T + 127) // 128, Nr), dtype=torch.int32, device=dev)
    idx, gates = ebl.router_forward_logits(x, bias, K, counts, tile_counts=tiles)
    tp = ebl.balance_stats_logits(x)
    S = 4096
    loss, loss_seq = ebl.seq_balance_loss(tiles, tp, T, K, S, ebl.SEQ_BALANCE_ALPHA)
    torch.cuda.synchronize()
    ref = oracle.router_logits(to_np(x), to_np(bias), K, tile_tokens=128, want_scores=True)
    assert np.array_equal(to_np(idx), ref.idx)
    assert np.array_equal(to_np(gates), ref.gates)
    assert np.array_equal(to_np(counts), ref.counts)
    assert np.array_equal(to_np(tiles), ref.tile_counts)
    # the sequence-wise balance loss over 256 sequences of 4096 tokens (tolerances
    # as in test_gpu_seq_balance: one fp32 rounding per tile sum)
    scores = ref.scores.astype(np.float64)
    want = oracle.tile_psum(scores, 128)
    assert np.all(np.abs(to_np(tp).astype(np.float64) - want) <= 2.0 ** -23 * want)
    r = oracle.seq_balance(scores, ref.idx, S, ebl.SEQ_BALANCE_ALPHA)
    assert np.allclose(to_np(loss_seq), r.loss_seq, rtol=1.2e-7, atol=0)
    # the same statistics fused into the routing pass: routing bit for bit, the
    # statistics within the fused tolerance (test_gpu_seq_balance)
    from tests.test_gpu_seq_balance import FUSED_ATOL, FUSED_RTOL
    c2 = torch.zeros(Nr, dtype=torch.int32, device=dev)
    tc2 = torch.empty_like(tiles)
    tp2 = torch.empty_like(tp)
    idx2, gates2 = ebl.router_forward_logits_balance(x, bias, K, c2, tc2, tp2)
    loss2, loss_seq2 = ebl.seq_balance_loss(tc2, tp2, T, K, S, ebl.SEQ_BALANCE_ALPHA)
    torch.cuda.synchronize()
    assert torch.equal(idx2, idx) and torch.equal(gates2, gates) and torch.equal(c2, counts)
    assert torch.equal(tc2, tiles)
    assert np.all(np.abs(to_np(tp2).astype(np.float64) - want) <= FUSED_RTOL * want + FUSED_ATOL)
    assert np.allclose(to_np(loss_seq2), r.loss_seq, rtol=FUSED_RTOL, atol=0)


def test_dispatch_combine_full_size(cuda_device):
    """The dispatch workload: router, dispatch, identity expert, combine."""
    cfg = synth.WORKLOADS["dispatch"]
    T, d, Nr, K = cfg["T"], cfg["d"], cfg["Nr"], cfg["K"]
    dev = cuda_device
    h = synth.hidden_normal(T, d, seed=synth.step_seed("dispatch", 0), device=dev)
    W = synth.router_weight(Nr, d, seed=synth.BASE_SEED + d).to(dev)
    counts = torch.zeros(Nr, dtype=torch.int32, device=dev)
    tiles = torch.empty(((T + 127) // 128, Nr), dtype=torch.int32, device=dev)
    idx, gates = ebl.router_forward(h, W, torch.zeros(Nr, device=dev), K, counts, tile_counts=tiles)
    st = torch.zeros(1, dtype=torch.int32, device=dev)
    offsets, perm, dest, X = ebl.moe_dispatch(h, idx, Nr, tile_counts=tiles, status=st)
    torch.cuda.synchronize()
    o_off, o_perm, o_dest = oracle.dispatch(to_np(idx), Nr)
    assert int(st.item()) == 0
    assert np.array_equal(to_np(offsets), o_off)
    assert np.array_equal(to_np(perm), o_perm)
    assert np.array_equal(to_np(dest), o_dest)
    assert torch.equal(X, h[perm.long()])                       # every row, bit for bit
    out = ebl.moe_combine(X, gates, dest, status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    # sampled rows against the oracle's fp32 chain, all rows against the identity
    rows = torch.randperm(T, generator=torch.Generator().manual_seed(3))[:256].sort().values
    pr = (rows[:, None] * K + torch.arange(K)[None, :]).reshape(-1)
    Xs = to_np(X[dest[pr.to(dev)].long()].view(torch.int16)).view(np.uint16)
    _, o32 = oracle.combine(Xs, to_np(gates[rows.to(dev)]), np.arange(pr.numel(), dtype=np.int32))
    assert np.array_equal(to_np(out[rows.to(dev)]), o32)
    rel = ((out - h.float()).abs() / h.float().abs().clamp_min(1e-30)).max()
    assert float(rel) <= (2 * K + 1) * 2.0 ** -24
