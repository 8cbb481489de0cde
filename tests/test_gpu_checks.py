"""Input validation and the exact-score cross-check on a B200.

ebl_check_finite_* must flag a NaN or an infinity wherever it sits (the
unaligned head, the 16-byte body, the tail) and must not flag the largest
finite values.  The exact logits-mode score the library computes in fp64 is
compared, value by value, with the oracle's (the host's fp64 exp): the
contract of logits mode is that both round to the same fp32.
"""
import numpy as np
import pytest
import torch

import expert_bias_load_b200 as ebl
import oracle
import synth
from tests.parity import to_np

pytestmark = pytest.mark.gpu


def _flag(x):
    st = torch.zeros(1, dtype=torch.int32, device=x.device)
    ebl.check_finite(x, st)
    torch.cuda.synchronize()
    return int(st.item())


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
def test_check_finite_flags_every_position(cuda_device, dtype):
    base = torch.randn(5003, device=cuda_device).to(dtype)
    big = torch.tensor([3.0e38 if dtype == torch.float32 else 3.0e38], device=cuda_device).to(dtype)
    assert torch.isfinite(big).all()
    for off in range(0, 9):                       # every alignment of the view's start
        for n in (1, 7, 8, 9, 64, 4000):
            x = base[off:off + n]
            assert _flag(x) == 0
            y = x.clone()
            y[-1] = big[0]
            assert _flag(y) == 0                   # the largest finite values pass
            for pos in sorted({0, n // 2, n - 1}):
                for bad in (float("nan"), float("inf"), float("-inf")):
                    buf = base.clone()
                    z = buf[off:off + n]
                    z[pos] = bad
                    assert _flag(z) == ebl.EBL_ST_NONFINITE, (dtype, off, n, pos, bad)
    assert _flag(base[:0]) == 0


def test_exact_scores_match_the_oracle(cuda_device):
    """Every exact score of a 4.2 M-value sweep (the 1/8 grid of the tie
    workload, N(0,1) and N(0,4) samples, and values near 0 and near the
    saturation ends) rounds to the same fp32 as the oracle's."""
    g = torch.Generator().manual_seed(11)
    parts = [
        torch.arange(-320, 321, dtype=torch.float32) / 8,
        torch.randn(1 << 21, generator=g),
        torch.randn(1 << 21, generator=g) * 4,
        torch.linspace(-1e-3, 1e-3, 4096),
        torch.linspace(15.0, 20.0, 4096), torch.linspace(-104.0, -85.0, 4096),
    ]
    x = torch.cat(parts)
    x = torch.cat([x, torch.zeros((-x.numel()) % 256)])
    exact = torch.empty_like(x, device=cuda_device)
    err, bound = ebl.selftest_score_error(x.to(cuda_device), exact_out=exact)
    torch.cuda.synchronize()
    ref = oracle.router_logits(x.numpy().reshape(-1, 256), np.zeros(256, np.float32), 1, want_scores=True)
    gpu = exact.cpu().numpy()
    mismatches = int(np.count_nonzero(gpu.view(np.uint32) != ref.scores.reshape(-1).view(np.uint32)))
    print("\nexact-score mismatches: %d of %d values; approximation error %.3e (bound %.3e)"
          % (mismatches, x.numel(), err, bound))
    assert mismatches == 0
    assert err * 4 <= bound


@pytest.mark.parametrize("mode", ["gemm", "logits_vec", "logits_row"])
def test_unfilled_slots_are_reported(cuda_device, mode):
    """A bias of -inf on all but two experts leaves K = 4 slots with only two
    keys above -inf: those two fill slots 0 and 1 (as the oracle orders them),
    slots 2 and 3 get id 0x7fffffff and gate 0 (GEMM mode: gate 0 too), add no
    load, and EBL_ST_NONFINITE is raised.  A finite bias raises nothing."""
    dev = cuda_device
    T, Nr, K, d = 300, 64, 4, 128
    live = [5, 40]
    bias = torch.full((Nr,), float("-inf"))
    bias[live] = 0.0
    counts = torch.zeros(Nr, dtype=torch.int32, device=dev)
    st = torch.zeros(1, dtype=torch.int32, device=dev)
    if mode == "gemm":
        h = synth.hidden_normal(T, d, seed=61)
        W = synth.router_weight(Nr, d, seed=62)
        idx, g = ebl.router_forward(h.to(dev), W.to(dev), bias.to(dev), K, counts, status=st)
        ref = oracle.router_gemm(h, W, np.zeros(Nr, np.float32), K, want_scores=True)
        scores = ref.scores
    else:
        x = synth.logits_normal(T, Nr, seed=63)
        if mode == "logits_row":               # 4 bytes past a 16-byte boundary: the row kernel
            buf = torch.empty(T * Nr + 1, device=dev)
            buf[1:] = x.reshape(-1).to(dev)
            xd = buf[1:].view(T, Nr)
        else:
            xd = x.to(dev)
        idx, g = ebl.router_forward_logits(xd, bias.to(dev), K, counts, status=st)
        scores = oracle.router_logits(x.numpy(), np.zeros(Nr, np.float32), 1, want_scores=True).scores
    torch.cuda.synchronize()
    assert int(st.item()) == ebl.EBL_ST_NONFINITE
    gi, gg = to_np(idx), to_np(g)
    s = scores[:, live]
    first = np.where(s[:, 0] >= s[:, 1], live[0], live[1])   # equal scores: the lower index first
    second = np.where(first == live[0], live[1], live[0])
    # GEMM mode orders the two the oracle's way except where fp32 and fp64
    # scores may disagree (keys closer than the near-tie margin)
    rows = np.abs(s[:, 0] - s[:, 1]) >= (1e-3 if mode == "gemm" else 0.0)
    assert rows.sum() > T // 2
    assert np.array_equal(gi[rows, 0], first[rows]) and np.array_equal(gi[rows, 1], second[rows])
    assert np.all(np.sort(gi[:, :2], 1) == np.array(live))
    assert np.all(gi[:, 2:] == 0x7fffffff)
    assert np.all(gg[:, 2:] == 0.0)
    assert np.allclose(gg[:, :2].sum(1), 1.0, atol=1e-6)
    c = to_np(counts)
    assert c[live].sum() == 2 * T and c.sum() == 2 * T

    # finite bias: nothing raised
    st.zero_()
    counts.zero_()
    if mode == "gemm":
        ebl.router_forward(h.to(dev), W.to(dev), torch.zeros(Nr, device=dev), K, counts, status=st)
    else:
        ebl.router_forward_logits(xd, torch.zeros(Nr, device=dev), K, counts, status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
