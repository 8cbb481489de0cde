"""The sequence-wise balance loss on the GPU against the oracle.

router_forward_balance writes per-tile sums of the normalised scores
s / sum_j s (tile_psum) beside the per-tile loads; seq_balance_loss turns them
into the per-sequence and batch values.  Tolerances:
  - tile_psum: the epilogue's scores are fp32 sigmoids (fast exp and
    reciprocal, a few ulp) of fp32-accumulated logits; s / total and the
    fixed-order fp32 sums over 128 rows add a few ulp more.  Each entry is
    within 2e-5 relative (+1e-6 absolute per token of the tile) of the fp64 oracle; the
    measured error is printed.
  - seq_balance_loss on given statistics: fp64 sums in another order than the
    oracle's, 1e-12 relative.
  - End to end in GEMM mode: the tile_psum error, plus the selections of
    tokens the near-tie rule excuses: moving one selection of a sequence from
    expert i to j changes its loss by alpha N_r / (K S^2) (q_j - q_i), at most
    alpha N_r / (K S) per moved selection.
  - Logits mode: the scores have one defined rounding and the selections are
    bit-exact, and balance_stats_logits sums in fp64 and rounds once, so each
    tile_psum entry is within one fp32 rounding (2^-24 relative, taken as
    2^-23 for the fp64 summation order) of the oracle, and the loss, a sum of
    positive terms each off by at most that much, within 1.2e-7 relative.
  - Logits mode, statistics fused into the routing pass
    (router_forward_logits_balance): the routing outputs are
    router_forward_logits' bit for bit; the statistics use the fast fp32
    score.  Its relative error is at most (1 - s)(2 + 1.173 |x|) ulp from the
    fast exp, 0.5 ulp from 1 + e and 2 ulp from the fast reciprocal: 52 ulp
    (6.2e-6) at |x| = 40 and 10 ulp (1.2e-6) at |x| <= 6.  The row total
    (32 terms per lane, 3 shuffle adds) adds at most 35 ulp relative, 1/total
    and the product 1.5 ulp, the fixed-order sum over the tile's rows (8 per
    lane, 2 shuffle adds, 3 warp adds) 13 ulp: at most 2^-16 relative in
    all (8.4e-6 at |x| = 40); scores below 2^-126 and above exp overflow are
    covered by an absolute 2^-60.  The loss, a positive combination of the
    entries, within 2^-16 relative too.
"""
import numpy as np
import pytest
import torch

import expert_bias_load_b200 as ebl
import oracle
import synth
from tests.parity import assert_gemm_parity, tile_hist, to_np

pytestmark = pytest.mark.gpu

PSUM_RTOL = 2e-5
PSUM_ATOL = 1e-6 * 128
FUSED_RTOL = 2.0 ** -16
FUSED_ATOL = 2.0 ** -60

# T, d, N_r, K, seq_len: ragged last tiles, both epilogue layouts (N_r % 64 == 0
# splits the experts over two warp groups, else one), K from 1 to 8
CASES = [
    (1000, 256, 64, 4, None),
    (2048, 512, 256, 4, 512),
    (1536, 128, 96, 2, 256),
    (777, 192, 32, 1, None),
    (4096, 1024, 128, 8, 1024),
    (1280, 64, 224, 6, 128),
    (300, 4096, 256, 4, None),
]


def _route(T, d, Nr, K, seed, zloss=False):
    dev = torch.device("cuda:0")
    h = synth.hidden_normal(T, d, seed=seed, device=dev)
    W = synth.router_weight(Nr, d, seed=seed + 1).to(dev)
    bias = (torch.randn(Nr, generator=torch.Generator().manual_seed(seed)) * 0.02).to(dev)
    tiles = (T + 127) // 128
    counts = torch.zeros(Nr, dtype=torch.int32, device=dev)
    tc = torch.full((tiles, Nr), -1, dtype=torch.int32, device=dev)
    tp = torch.full((tiles, Nr), -1.0, device=dev)
    z = torch.zeros(1, dtype=torch.float64, device=dev) if zloss else None
    idx, g = ebl.router_forward_balance(h, W, bias, K, counts, tc, tp, zloss_sum=z)
    return h, W, bias, counts, tc, tp, z, idx, g


@pytest.mark.parametrize("T,d,Nr,K,S", CASES)
def test_tile_psum_vs_oracle(cuda_device, T, d, Nr, K, S):
    h, W, bias, counts, tc, tp, _, idx, g = _route(T, d, Nr, K, seed=T + Nr)
    # the routing outputs are those of router_forward, bit for bit
    c2 = torch.zeros(Nr, dtype=torch.int32, device=cuda_device)
    t2 = torch.empty_like(tc)
    i2, g2 = ebl.router_forward(h, W, bias, K, c2, tile_counts=t2)
    torch.cuda.synchronize()
    assert torch.equal(idx, i2) and torch.equal(g, g2) and torch.equal(counts, c2) and torch.equal(tc, t2)
    ref = oracle.router_gemm(h.cpu(), W.cpu(), bias.cpu().numpy(), K, want_scores=True)
    gi = to_np(idx)
    assert_gemm_parity(gi, to_np(g), ref, Nr, bias.cpu().numpy(), gpu_counts=to_np(counts))
    assert np.array_equal(to_np(tc), tile_hist(gi, Nr))
    want = oracle.tile_psum(ref.scores, 128)
    got = to_np(tp).astype(np.float64)
    err = np.abs(got - want)
    assert np.all(err <= PSUM_RTOL * np.abs(want) + PSUM_ATOL), err.max()
    # one unit of s / total per token: rows of a tile sum to its token count
    rows = np.minimum(128, T - 128 * np.arange(want.shape[0]))
    assert np.allclose(got.sum(1), rows, rtol=1e-5, atol=0)
    print("tile_psum max abs err %.3e, max rel err %.3e" % (err.max(), (err / np.maximum(want, 1e-30)).max()))


def test_balance_with_zloss_matches_zloss_call(cuda_device):
    """Both options in one launch: the z-loss statistic equals router_forward_zloss's
    up to the order of its fp64 atomics, tile_psum equals the balance-only launch
    bit for bit."""
    T, d, Nr, K = 2000, 512, 128, 4
    h, W, bias, counts, tc, tp, z, idx, g = _route(T, d, Nr, K, seed=91, zloss=True)
    _, _, _, _, tc2, tp2, _, i2, g2 = _route(T, d, Nr, K, seed=91)
    c3 = torch.zeros(Nr, dtype=torch.int32, device=cuda_device)
    z3 = torch.zeros(1, dtype=torch.float64, device=cuda_device)
    ebl.router_forward_zloss(h, W, bias, K, c3, z3)
    torch.cuda.synchronize()
    assert torch.equal(tp, tp2) and torch.equal(tc, tc2) and torch.equal(idx, i2) and torch.equal(g, g2)
    assert abs(float(z.item()) - float(z3.item())) <= 1e-12 * float(z3.item())


@pytest.mark.parametrize("Nr,K,S,B", [(256, 4, 4096, 3), (64, 8, 128, 40), (96, 1, 384, 5), (7, 3, 256, 2),
                                      (1, 1, 128, 1)])
def test_seq_balance_loss_kernel(cuda_device, Nr, K, S, B):
    """The loss kernels on seeded per-tile statistics (not produced by the
    router): per-sequence and batch values against the oracle's regrouping."""
    rng = np.random.default_rng(Nr * 1000 + S)
    T = S * B
    tiles = T // 128
    tc = rng.integers(0, 3 * K * 128 // max(Nr, 1) + 2, (tiles, Nr)).astype(np.int32)
    tp = (rng.random((tiles, Nr)) * 128 / Nr * 2).astype(np.float32)
    alpha = float(np.float32(5e-5))
    loss, loss_seq = ebl.seq_balance_loss(torch.from_numpy(tc).to(cuda_device), torch.from_numpy(tp).to(cuda_device),
                                          T, K, S, alpha)
    torch.cuda.synchronize()
    ref, ref_seq = oracle.seq_balance_tiles(tc, tp.astype(np.float64), T, K, S, alpha, 128)
    assert np.allclose(to_np(loss_seq), ref_seq, rtol=1e-12, atol=0)
    assert abs(float(loss.item()) - ref) <= 1e-12 * abs(ref)


@pytest.mark.parametrize("T,d,Nr,K,S", [c for c in CASES if c[4] is not None])
def test_seq_balance_end_to_end(cuda_device, T, d, Nr, K, S):
    alpha = ebl.SEQ_BALANCE_ALPHA
    h, W, bias, counts, tc, tp, _, idx, g = _route(T, d, Nr, K, seed=7 * T + d)
    loss, loss_seq = ebl.seq_balance_loss(tc, tp, T, K, S, alpha)
    torch.cuda.synchronize()
    ref = oracle.router_gemm(h.cpu(), W.cpu(), bias.cpu().numpy(), K, want_scores=True)
    r = oracle.seq_balance(ref.scores, ref.idx, S, alpha)
    excused = (ref.gap < 1e-3).reshape(T // S, S).sum(1)
    allow = 2e-5 * np.abs(r.loss_seq) + excused * K * alpha * Nr / (K * S)
    got = to_np(loss_seq)
    assert np.all(np.abs(got - r.loss_seq) <= allow), (got, r.loss_seq, excused)
    assert abs(float(loss.item()) - got.mean()) <= 1e-15 * abs(got.mean())
    print("seq balance loss %.9e oracle %.9e (excused tokens %d)" % (float(loss.item()), r.loss, excused.sum()))


def test_equal_scores_give_alpha(cuda_device):
    """W = 0: every logit is 0 and every score 1/2, so s / total = 1/N_r for
    every expert and the loss is alpha exactly, whatever the selection."""
    T, d, Nr, K, S = 1024, 128, 256, 4, 256
    dev = cuda_device
    h = synth.hidden_normal(T, d, seed=5, device=dev)
    W = torch.zeros(Nr, d, dtype=torch.bfloat16, device=dev)
    counts = torch.zeros(Nr, dtype=torch.int32, device=dev)
    tc = torch.empty(T // 128, Nr, dtype=torch.int32, device=dev)
    tp = torch.empty(T // 128, Nr, device=dev)
    ebl.router_forward_balance(h, W, torch.zeros(Nr, device=dev), K, counts, tc, tp)
    loss, loss_seq = ebl.seq_balance_loss(tc, tp, T, K, S, 0.25)
    torch.cuda.synchronize()
    assert torch.all(tp == 128.0 / Nr)
    assert float(loss.item()) == 0.25 and torch.all(loss_seq == 0.25)


def test_empty_batch_is_a_noop(cuda_device):
    dev = cuda_device
    Nr, d = 64, 128
    e16 = torch.empty(0, d, dtype=torch.bfloat16, device=dev)
    W = synth.router_weight(Nr, d, seed=1).to(dev)
    counts = torch.zeros(Nr, dtype=torch.int32, device=dev)
    tc = torch.empty(0, Nr, dtype=torch.int32, device=dev)
    tp = torch.empty(0, Nr, device=dev)
    idx, g = ebl.router_forward_balance(e16, W, torch.zeros(Nr, device=dev), 4, counts, tc, tp)
    loss, loss_seq = ebl.seq_balance_loss(tc, tp, 0, 4, 128)
    torch.cuda.synchronize()
    assert idx.numel() == 0 and loss_seq.numel() == 0 and int(counts.sum().item()) == 0


LOGITS_CASES = [(1000, 256, 4), (300, 7, 3), (129, 1, 1), (4096, 64, 8), (2000, 255, 2), (256, 33, 5)]


@pytest.mark.parametrize("T,Nr,K", LOGITS_CASES)
def test_logits_mode_tile_psum(cuda_device, T, Nr, K):
    rng = np.random.default_rng(T + Nr)
    x = (rng.standard_normal((T, Nr)) * 3).astype(np.float32)
    x[: T // 3] = np.round(x[: T // 3] * 8) / 8                          # ties and repeated values
    x[T // 2, : min(Nr, 6)] = [88.7, -88.7, -103.0, -104.0, 700.0, -3e38][: min(Nr, 6)]   # saturated, subnormal
    xd = torch.from_numpy(x).to(cuda_device)
    tp = ebl.balance_stats_logits(xd)
    torch.cuda.synchronize()
    ref = oracle.router_logits(x, np.zeros(Nr, np.float32), K, want_scores=True)
    want = oracle.tile_psum(ref.scores.astype(np.float64), 128)
    got = to_np(tp).astype(np.float64)
    err = np.abs(got - want)
    assert np.all(err <= 2.0 ** -23 * want), (err / want).max()
    print("logits-mode tile_psum max rel err %.3e (2^-24 = %.3e)" % ((err / want).max(), 2.0 ** -24))


@pytest.mark.parametrize("T,Nr,K,S", [(4096, 256, 4, 1024), (1536, 64, 8, 512), (1280, 13, 2, 128)])
def test_logits_mode_loss_end_to_end(cuda_device, T, Nr, K, S):
    """Logits mode: exact selections and loads, so the loss has no excused tokens."""
    rng = np.random.default_rng(3 * T + Nr)
    x = np.round(rng.standard_normal((T, Nr)).astype(np.float32) * 8) / 8
    b = (rng.integers(-2, 3, Nr) * 0.01).astype(np.float32)
    dev = cuda_device
    xd = torch.from_numpy(x).to(dev)
    counts = torch.zeros(Nr, dtype=torch.int32, device=dev)
    tc = torch.empty(T // 128, Nr, dtype=torch.int32, device=dev)
    ebl.router_forward_logits(xd, torch.from_numpy(b).to(dev), K, counts, tile_counts=tc)
    tp = ebl.balance_stats_logits(xd)
    alpha = ebl.SEQ_BALANCE_ALPHA
    loss, loss_seq = ebl.seq_balance_loss(tc, tp, T, K, S, alpha)
    torch.cuda.synchronize()
    ref = oracle.router_logits(x, b, K, want_scores=True, tile_tokens=128)
    assert np.array_equal(to_np(tc), ref.tile_counts)
    r = oracle.seq_balance(ref.scores.astype(np.float64), ref.idx, S, alpha)
    assert np.allclose(to_np(loss_seq), r.loss_seq, rtol=1.2e-7, atol=0), (to_np(loss_seq), r.loss_seq)
    assert abs(float(loss.item()) - r.loss) <= 1.2e-7 * r.loss


def _fused(xd, bias, K):
    T, Nr = xd.shape
    dev = xd.device
    tiles = (T + 127) // 128
    counts = torch.zeros(Nr, dtype=torch.int32, device=dev)
    tc = torch.full((tiles, Nr), -1, dtype=torch.int32, device=dev)
    tp = torch.full((tiles, Nr), -1.0, device=dev)
    idx, g = ebl.router_forward_logits_balance(xd, bias, K, counts, tc, tp)
    return idx, g, counts, tc, tp


# vector-kernel shapes with padding columns (N_r % 4 == 0 but below the lanes' column blocks)
FUSED_EXTRA = [(3000, 256, 4), (1100, 128, 8), (777, 4, 2), (500, 68, 6), (500, 132, 3), (600, 252, 8)]


@pytest.mark.parametrize("misalign", [False, True])
@pytest.mark.parametrize("T,Nr,K", LOGITS_CASES + FUSED_EXTRA)
def test_logits_mode_fused_balance(cuda_device, T, Nr, K, misalign):
    """router_forward_logits_balance: routing identical to router_forward_logits
    (and to the oracle), tile_psum within the fused tolerance of the oracle's
    fp64 sums of the rounded-once scores.  misalign: the logits 4 bytes past a
    16-byte boundary (the row kernel plus the separate statistics pass)."""
    rng = np.random.default_rng(7 * T + Nr)
    x = (rng.standard_normal((T, Nr)) * 3).astype(np.float32)
    x[: T // 3] = np.round(x[: T // 3] * 8) / 8
    x[T // 2, : min(Nr, 6)] = [88.7, -88.7, -103.0, -104.0, 700.0, -3e38][: min(Nr, 6)]
    b = (rng.integers(-3, 4, Nr) * 0.01).astype(np.float32)
    dev = cuda_device
    if misalign:
        buf = torch.empty(T * Nr + 1, device=dev)
        buf[1:] = torch.from_numpy(x).reshape(-1).to(dev)
        xd = buf[1:].view(T, Nr)
    else:
        xd = torch.from_numpy(x).to(dev)
    bd = torch.from_numpy(b).to(dev)
    idx, g, counts, tc, tp = _fused(xd, bd, K)
    c2 = torch.zeros(Nr, dtype=torch.int32, device=dev)
    tc2 = torch.empty_like(tc)
    idx2, g2 = ebl.router_forward_logits(xd, bd, K, c2, tile_counts=tc2)
    torch.cuda.synchronize()
    assert torch.equal(idx, idx2) and torch.equal(g, g2) and torch.equal(counts, c2) and torch.equal(tc, tc2)
    ref = oracle.router_logits(x, b, K, want_scores=True, tile_tokens=128)
    assert np.array_equal(to_np(idx), ref.idx) and np.array_equal(to_np(g), ref.gates)
    assert np.array_equal(to_np(tc), ref.tile_counts)
    want = oracle.tile_psum(ref.scores.astype(np.float64), 128)
    got = to_np(tp).astype(np.float64)
    err = np.abs(got - want)
    assert np.all(err <= FUSED_RTOL * want + FUSED_ATOL), (err / np.maximum(want, 1e-300)).max()
    rows = np.minimum(128, T - 128 * np.arange(want.shape[0]))
    assert np.allclose(got.sum(1), rows, rtol=1e-5, atol=0)          # each row's normalised scores sum to 1
    print("fused logits-mode tile_psum max rel err %.3e (tolerance %.3e)"
          % ((err / np.maximum(want, 1e-30)).max(), FUSED_RTOL))


@pytest.mark.parametrize("T,Nr,K,S", [(4096, 256, 4, 1024), (1536, 64, 8, 512), (2560, 128, 2, 256)])
def test_logits_mode_fused_loss_end_to_end(cuda_device, T, Nr, K, S):
    rng = np.random.default_rng(5 * T + Nr)
    x = np.round(rng.standard_normal((T, Nr)).astype(np.float32) * 8) / 8
    b = (rng.integers(-2, 3, Nr) * 0.01).astype(np.float32)
    dev = cuda_device
    idx, g, counts, tc, tp = _fused(torch.from_numpy(x).to(dev), torch.from_numpy(b).to(dev), K)
    alpha = ebl.SEQ_BALANCE_ALPHA
    loss, loss_seq = ebl.seq_balance_loss(tc, tp, T, K, S, alpha)
    torch.cuda.synchronize()
    ref = oracle.router_logits(x, b, K, want_scores=True, tile_tokens=128)
    assert np.array_equal(to_np(tc), ref.tile_counts)
    r = oracle.seq_balance(ref.scores.astype(np.float64), ref.idx, S, alpha)
    assert np.allclose(to_np(loss_seq), r.loss_seq, rtol=FUSED_RTOL, atol=0), (to_np(loss_seq), r.loss_seq)
    assert abs(float(loss.item()) - r.loss) <= FUSED_RTOL * r.loss


def test_logits_mode_fused_balance_empty_and_checks(cuda_device):
    dev = cuda_device
    Nr = 64
    x = torch.empty(0, Nr, device=dev)
    counts = torch.zeros(Nr, dtype=torch.int32, device=dev)
    tc = torch.empty(0, Nr, dtype=torch.int32, device=dev)
    tp = torch.empty(0, Nr, device=dev)
    idx, g = ebl.router_forward_logits_balance(x, torch.zeros(Nr, device=dev), 4, counts, tc, tp)
    torch.cuda.synchronize()
    assert idx.numel() == 0 and int(counts.sum().item()) == 0
    rc = ebl.lib().router_forward_logits_balance(ebl._ptr(torch.zeros(256, Nr, device=dev)),
                                                 ebl._ptr(torch.zeros(Nr, device=dev)), 256, Nr, 4,
                                                 ebl._ptr(torch.zeros(256, 4, dtype=torch.int32, device=dev)),
                                                 ebl._ptr(torch.zeros(256, 4, device=dev)), ebl._ptr(counts),
                                                 None, ebl._ptr(torch.zeros(2, Nr, device=dev)), None, None)
    assert rc == ebl.EBL_EINVAL                                         # tile_counts is required
