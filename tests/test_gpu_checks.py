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
