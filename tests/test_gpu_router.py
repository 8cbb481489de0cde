"""Router kernels against the oracle on a B200 (GEMM mode and logits mode)."""
import numpy as np
import pytest
import torch

import expert_bias_load_b200 as ebl
import oracle
import synth
from tests.parity import STATE_RTOL, assert_gemm_parity, rel_err, tile_hist, to_np

pytestmark = pytest.mark.gpu


def _run_logits(logits, bias, K, want_tiles=True, misalign=False):
    """misalign: place the logits 4 bytes past a 16-byte boundary, which sends
    them through the row kernel instead of the vector kernel."""
    dev = torch.device("cuda:0")
    T, Nr = logits.shape
    if misalign:
        buf = torch.empty(T * Nr + 1, dtype=torch.float32, device=dev)
        buf[1:] = logits.reshape(-1).to(dev)
        x = buf[1:].view(T, Nr)
        assert x.data_ptr() % 16 == 4
    else:
        x = logits.to(dev)
    b = bias.to(dev)
    counts = torch.zeros(Nr, dtype=torch.int32, device=dev)
    tiles = torch.full(((T + 127) // 128, Nr), -7, dtype=torch.int32, device=dev) if want_tiles else None
    idx, gates = ebl.router_forward_logits(x, b, K, counts, tile_counts=tiles)
    torch.cuda.synchronize()
    return to_np(idx), to_np(gates), to_np(counts), (to_np(tiles) if want_tiles else None)


LOGITS_CASES = [
    # T, Nr, K, quantised, bias kind
    (2048 + 77, 64, 4, False, "small"),
    (1000, 8, 8, True, "ties"),
    (1000, 8, 3, True, "ties"),
    (513, 16, 1, False, "small"),
    (3000, 256, 4, True, "dead"),
    (4096, 128, 8, False, "small"),
    (129, 200, 5, True, "ties"),
    (1, 33, 2, False, "small"),
    (127, 256, 7, False, "dead"),
    (777, 4, 2, True, "ties"),           # the smallest row the vector kernel takes (one float4)
    (500, 68, 6, False, "small"),        # just past 64 experts: 4 float4 per lane, 3 of them partly padding
    (500, 132, 3, True, "dead"),         # just past 128: 8 float4 per lane
    (600, 252, 8, True, "ties"),         # ragged last column block
    (100, 1, 1, False, "small"),         # a single expert
    (257, 2, 2, True, "ties"),           # K = N_r with ties
    (300, 3, 2, True, "ties"),
]


@pytest.mark.parametrize("misalign", [False, True])
@pytest.mark.parametrize("T,Nr,K,quant,bk", LOGITS_CASES)
def test_logits_mode_bit_exact(cuda_device, T, Nr, K, quant, bk, misalign):
    logits = synth.logits_normal(T, Nr, seed=100 + T + Nr + K, quant8=quant)
    if bk == "small":
        bias = torch.randn(Nr, generator=torch.Generator().manual_seed(K)) * 0.01
    elif bk == "ties":
        bias = (torch.randint(-2, 3, (Nr,), generator=torch.Generator().manual_seed(K)) * 0.125).float()
    else:
        bias = synth.dead_start_bias(Nr, n_dead=min(8, Nr - K))
    idx, gates, counts, tiles = _run_logits(logits, bias, K, misalign=misalign)
    ref = oracle.router_logits(logits.numpy(), bias.numpy(), K, tile_tokens=128)
    assert np.array_equal(idx, ref.idx)
    assert np.array_equal(gates.view(np.uint32), ref.gates.view(np.uint32))
    assert np.array_equal(counts, ref.counts)
    assert np.array_equal(tiles, ref.tile_counts)


def test_logits_mode_tie_workload_slice(cuda_device):
    """The tie workload (values on a 1/8 grid, 8 experts starting at -1) on a
    65536-token slice: exact ties between scores are everywhere."""
    T, Nr, K = 65536 + 5, 256, 4
    logits = synth.logits_normal(T, Nr, seed=synth.step_seed("ties", 0), quant8=True)
    bias = synth.dead_start_bias(Nr)
    idx, gates, counts, tiles = _run_logits(logits, bias, K)
    ref = oracle.router_logits(logits.numpy(), bias.numpy(), K, tile_tokens=128)
    assert np.array_equal(idx, ref.idx)
    assert np.array_equal(gates, ref.gates)
    assert np.array_equal(counts, ref.counts)
    assert np.array_equal(tiles, ref.tile_counts)
    assert counts[:8].sum() == 0          # the dead-start experts are never picked at step 0


def test_logits_mode_bias_forces_expert(cuda_device):
    T, Nr, K = 999, 64, 4
    logits = synth.logits_normal(T, Nr, seed=5)
    bias = torch.zeros(Nr)
    bias[17] = 10.0
    idx, gates, counts, _ = _run_logits(logits, bias, K, want_tiles=False)
    assert np.all(idx[:, 0] == 17) and counts[17] == T


GEMM_CASES = [
    # T, d, Nr, K
    (2048, 256, 64, 4),          # the tiny workload
    (2048 + 77, 256, 64, 4),     # ragged tail
    (3000, 512, 256, 4),
    (1000, 2048, 128, 8),        # the mid workload's shape, fewer tokens
    (777, 128, 32, 1),
    (777, 128, 32, 8),
    (129, 64, 96, 3),
    (1, 64, 32, 2),
    (5000, 3072, 256, 4),        # the drift workload's shape, fewer tokens
    (300, 4096, 256, 8),
    (1000, 192, 160, 5),         # one epilogue group (N_r % 64 != 0), 5 slots
    (600, 320, 192, 6),          # two groups of 96 experts
    (513, 64, 224, 7),           # one group of 224 experts, a single K stage
    (2 * 128 * 148 + 5, 128, 64, 2),  # more pair tiles than the persistent grid holds at once
]


@pytest.mark.parametrize("T,d,Nr,K", GEMM_CASES)
def test_gemm_mode_vs_oracle(cuda_device, T, d, Nr, K):
    dev = cuda_device
    h = synth.hidden_normal(T, d, seed=T * 7 + d)
    W = synth.router_weight(Nr, d, seed=d + Nr)
    bias = torch.randn(Nr, generator=torch.Generator().manual_seed(3)) * 0.02
    counts = torch.zeros(Nr, dtype=torch.int32, device=dev)
    tiles = torch.full(((T + 127) // 128, Nr), -7, dtype=torch.int32, device=dev)
    status = torch.zeros(1, dtype=torch.int32, device=dev)
    idx, gates = ebl.router_forward(h.to(dev), W.to(dev), bias.to(dev), K, counts, tile_counts=tiles,
                                    status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    ref = oracle.router_gemm(h, W, bias.numpy(), K, want_scores=True)
    gi = to_np(idx)
    assert_gemm_parity(gi, to_np(gates), ref, Nr, bias.numpy(), gpu_counts=to_np(counts))
    assert np.array_equal(to_np(tiles), tile_hist(gi, Nr))
    g = to_np(gates).astype(np.float64)
    assert np.allclose(g.sum(1), 1.0, atol=K * 2e-7)


def test_gemm_mode_tiny_workload_smebu_steps(cuda_device):
    """The tiny workload end to end: 10 steps of fresh hidden, router, SMEBU."""
    dev = cuda_device
    cfg = synth.WORKLOADS["tiny"]
    T, d, Nr, K = cfg["T"], cfg["d"], cfg["Nr"], cfg["K"]
    W = synth.router_weight(Nr, d, seed=synth.BASE_SEED)
    b_g = torch.zeros(Nr, device=dev)
    m_g = torch.zeros(Nr, device=dev)
    b_o = np.zeros(Nr, np.float32)
    m_o = np.zeros(Nr, np.float32)
    counts = torch.zeros(Nr, dtype=torch.int32, device=dev)
    maxvio = torch.zeros(1, device=dev)
    for step in range(cfg["steps"]):
        h = synth.hidden_normal(T, d, seed=synth.step_seed("tiny", step))
        ref = oracle.router_gemm(h, W, b_o, K, want_scores=True)
        idx, gates = ebl.router_forward(h.to(dev), W.to(dev), b_g, K, counts)
        torch.cuda.synchronize()
        n_gpu = to_np(counts).astype(np.int64)
        assert_gemm_parity(to_np(idx), to_np(gates), ref, Nr, b_o, gpu_counts=n_gpu)
        ebl.smebu_step(counts, b_g, m_g, reset_counts=True, maxvio=maxvio)
        # open loop: the oracle's SMEBU is fed the GPU's counts
        oracle.smebu(n_gpu, b_o, m_o)
        torch.cuda.synchronize()
        assert rel_err(to_np(b_g), b_o).max() <= STATE_RTOL
        assert rel_err(to_np(m_g), m_o).max() <= STATE_RTOL
        assert float(maxvio.item()) == np.float32(oracle.maxvio(n_gpu)[0])
        assert int(counts.sum().item()) == 0


ZLOSS_CASES = [(2048 + 77, 256, 64, 4), (3000, 512, 256, 4), (1000, 2048, 128, 8), (129, 64, 96, 3)]


@pytest.mark.parametrize("T,d,Nr,K", ZLOSS_CASES)
def test_router_zloss_vs_oracle(cuda_device, T, d, Nr, K):
    """Fused z-loss statistic: sum_t logsumexp(x_t)^2 within 1e-4 relative of the
    fp64 oracle (fp32 logits and exp/log: per-token error ~1e-5 relative), and
    the routing outputs bit-identical to router_forward."""
    dev = cuda_device
    h = synth.hidden_normal(T, d, seed=T + 3 * d, device=dev)
    W = synth.router_weight(Nr, d, seed=Nr + d).to(dev)
    bias = (torch.randn(Nr, generator=torch.Generator().manual_seed(5)) * 0.02).to(dev)
    c1 = torch.zeros(Nr, dtype=torch.int32, device=dev)
    c2 = torch.zeros(Nr, dtype=torch.int32, device=dev)
    z = torch.zeros(1, dtype=torch.float64, device=dev)
    i1, g1 = ebl.router_forward(h, W, bias, K, c1)
    i2, g2 = ebl.router_forward_zloss(h, W, bias, K, c2, z)
    torch.cuda.synchronize()
    assert torch.equal(i1, i2) and torch.equal(g1, g2) and torch.equal(c1, c2)
    ref = oracle.router_zloss(h.cpu(), W.cpu())
    assert abs(float(z.item()) - ref) <= 1e-4 * ref, (float(z.item()), ref)
    # accumulates: a second call adds the same amount again
    ebl.router_forward_zloss(h, W, bias, K, c2, z)
    torch.cuda.synchronize()
    assert abs(float(z.item()) - 2 * ref) <= 2e-4 * ref


def test_alternating_shapes_share_one_kernel(cuda_device):
    """Shapes that need different shared-memory sizes on the same kernel
    instantiation, in both orders (the larger one first, then a smaller one,
    then the larger one again), all launch."""
    dev = cuda_device
    for Nr in (64, 256, 64, 128, 256, 64):
        T, d, K = 300, 256, 4
        h = synth.hidden_normal(T, d, seed=Nr, device=dev)
        W = synth.router_weight(Nr, d, seed=Nr + 1).to(dev)
        counts = torch.zeros(Nr, dtype=torch.int32, device=dev)
        idx, g = ebl.router_forward(h, W, torch.zeros(Nr, device=dev), K, counts)
        torch.cuda.synchronize()
        assert int(counts.sum().item()) == T * K


def test_logits_mode_all_equal_keys(cuda_device):
    """Every expert has the same key (logits 0, bias 0), and rows where 40
    experts share the top key: the candidate buffer overflows and is scored in
    several rounds, and the lowest indices still win."""
    T, Nr, K = 200, 256, 4
    x = torch.zeros(T, Nr)
    bias = torch.zeros(Nr)
    x[100:, 60:100] = 1.0                          # rows 100.. : experts 60..99 tie at the top
    idx, gates, counts, tiles = _run_logits(x, bias, K)
    assert np.array_equal(idx[:100], np.tile(np.arange(K, dtype=np.int32), (100, 1)))
    assert np.array_equal(idx[100:], np.tile(np.arange(60, 60 + K, dtype=np.int32), (100, 1)))
    assert np.all(gates == np.float32(0.25))
    ref = oracle.router_logits(x.numpy(), bias.numpy(), K, tile_tokens=128)
    assert np.array_equal(idx, ref.idx) and np.array_equal(counts, ref.counts)


@pytest.mark.parametrize("misalign", [False, True])
@pytest.mark.parametrize("Nr,K", [(256, 4), (128, 8), (64, 3), (256, 1)])
def test_logits_mode_many_tied_candidates(cuda_device, Nr, K, misalign):
    """Rows where 1..90 experts tie at the top key (logits on a 1/8 grid, bias
    on a 1/8 grid for half of the rows): the candidates of a row are scored in
    one to four rounds of 24 and merged, and equal keys go to the lower
    index."""
    T = 3000
    g = torch.Generator().manual_seed(Nr * 10 + K)
    x = torch.round(torch.randn(T, Nr, generator=g) * 8) / 8 - 4.0
    ties = torch.randint(1, min(90, Nr) + 1, (T,), generator=g)
    for t in range(T):
        cols = torch.randperm(Nr, generator=g)[: int(ties[t])]
        x[t, cols] = 1.5
    bias = torch.zeros(Nr)
    bias[torch.randperm(Nr, generator=g)[: Nr // 4]] = -0.125
    idx, gates, counts, tiles = _run_logits(x, bias, K, misalign=misalign)
    ref = oracle.router_logits(x.numpy(), bias.numpy(), K, tile_tokens=128)
    assert np.array_equal(idx, ref.idx)
    assert np.array_equal(gates.view(np.uint32), ref.gates.view(np.uint32))
    assert np.array_equal(counts, ref.counts)
    assert np.array_equal(tiles, ref.tile_counts)


@pytest.mark.parametrize("layout", ["spread", "clustered"])
@pytest.mark.parametrize("Nr,K", [(256, 4), (128, 8), (64, 2), (256, 1)])
def test_logits_mode_wide_fast_path(cuda_device, Nr, K, layout):
    """Every row has 5 to 16 experts tied at the top key, spread over the row
    or packed into runs of consecutive experts (up to 8 in one lane's block
    of the vector kernel): the loop-free candidate stage then scores two
    candidates per lane and takes up to 8 from one lane.  Equal keys go to the
    lower index, bit for bit as the oracle."""
    T = 4096
    g = torch.Generator().manual_seed(Nr * 100 + K + (7 if layout == "clustered" else 0))
    x = torch.round(torch.randn(T, Nr, generator=g) * 8) / 8 - 4.0
    ties = torch.randint(5, 17, (T,), generator=g)
    for t in range(T):
        n = int(ties[t])
        if layout == "spread":
            cols = torch.randperm(Nr, generator=g)[:n]
        else:
            start = int(torch.randint(0, Nr - n + 1, (1,), generator=g))
            cols = torch.arange(start, start + n)
        x[t, cols] = 1.5
    bias = torch.zeros(Nr)
    idx, gates, counts, tiles = _run_logits(x, bias, K)
    ref = oracle.router_logits(x.numpy(), bias.numpy(), K, tile_tokens=128)
    assert np.array_equal(idx, ref.idx)
    assert np.array_equal(gates.view(np.uint32), ref.gates.view(np.uint32))
    assert np.array_equal(counts, ref.counts)
    assert np.array_equal(tiles, ref.tile_counts)


def test_logits_score_error_within_bound(cuda_device):
    """The approximate score logits mode ranks with stays well inside the
    error bound its candidate limit assumes, over a dense sweep of [-40, 40],
    the values near 0, and random finite fp32 bit patterns."""
    dev = cuda_device
    sweep = torch.linspace(-40.0, 40.0, 1 << 24, device=dev)
    tiny = torch.linspace(-1e-3, 1e-3, 1 << 20, device=dev)
    bits = torch.randint(0, 1 << 31, (1 << 22,), generator=torch.Generator().manual_seed(3), dtype=torch.int64)
    bits = bits.to(torch.int32).view(torch.float32)
    rnd = bits[torch.isfinite(bits)].to(dev)
    rnd = torch.cat([rnd, -rnd])
    for x in (sweep, tiny, rnd):
        err, bound = ebl.selftest_score_error(x.contiguous())
        assert 0.0 < bound <= 2.0 ** -8
        assert err * 4.0 <= bound, (err, bound)
    err, _ = ebl.selftest_score_error(torch.tensor([0.0, 1.0, -1.0], device=dev))
    assert err < 2.0 ** -11


@pytest.mark.parametrize("misalign", [False, True])
def test_logits_mode_saturated_scores(cuda_device, misalign):
    """Logits of scale 60: most sigmoids round to exactly 0.0 or 1.0 in fp32,
    so dozens of experts per row share the top key and the lowest indices
    must win; a small bias on a 1/64 grid splits some of them."""
    T, Nr, K = 2000, 256, 4
    g = torch.Generator().manual_seed(77)
    x = torch.randn(T, Nr, generator=g) * 60.0
    bias = (torch.randint(-1, 2, (Nr,), generator=g) / 64.0).float()
    idx, gates, counts, tiles = _run_logits(x, bias, K, misalign=misalign)
    ref = oracle.router_logits(x.numpy(), bias.numpy(), K, tile_tokens=128)
    assert np.array_equal(idx, ref.idx)
    assert np.array_equal(gates.view(np.uint32), ref.gates.view(np.uint32))
    assert np.array_equal(counts, ref.counts)
    assert np.array_equal(tiles, ref.tile_counts)


def test_microbench_runs_every_entry_point(cuda_device, capsys):
    from expert_bias_load_b200 import microbench
    for op in ("router", "zloss", "balance", "logits", "balance_logits", "smebu", "sign", "dispatch", "combine"):
        microbench.main([op, "--tokens", "4096", "--hidden", "256", "--experts", "64", "--topk", "4",
                         "--warmup", "1", "--reps", "2"])
    lines = [l for l in capsys.readouterr().out.splitlines() if " ms, " in l]
    assert len(lines) == 9
