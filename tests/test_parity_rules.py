"""The GEMM-mode comparison rule itself (CPU): near-ties excuse exactly what
they should and nothing else."""
import numpy as np
import pytest

import oracle
from tests.parity import MARGIN, assert_gemm_parity


def _case():
    # 2 tokens, 6 experts, K = 3.  Token 0: slots 1 and 2 nearly tie (1e-7),
    # the K-th/(K+1)-th gap is wide.  Token 1: the K-th and (K+1)-th nearly tie.
    scores = np.array([[0.90, 0.80, 0.8000001, 0.10, 0.20, 0.30],
                       [0.90, 0.80, 0.70, 0.6999999, 0.20, 0.10]])
    bias = np.zeros(6, np.float32)
    keys = scores + bias
    idx = np.argsort(-keys, axis=1, kind="stable")[:, :3].astype(np.int32)
    srt = -np.sort(-keys, axis=1)
    gap = srt[:, 2] - srt[:, 3]
    sel = np.take_along_axis(scores, idx.astype(np.int64), 1)
    gates = sel / sel.sum(1, keepdims=True)
    counts = np.bincount(idx.ravel(), minlength=6).astype(np.int64)
    return oracle.RouterResult(idx=idx, gates=gates, counts=counts, scores=scores, gap=gap), bias


def test_identical_results_pass():
    orc, bias = _case()
    assert assert_gemm_parity(orc.idx.copy(), orc.gates.copy(), orc, 6, bias) == 1   # token 1 is excused


def test_swap_of_near_equal_selected_keys_passes():
    orc, bias = _case()
    gi = orc.idx.copy()
    gi[0, [1, 2]] = gi[0, [2, 1]]
    gg = orc.gates.copy()
    gg[0, [1, 2]] = gg[0, [2, 1]]
    assert_gemm_parity(gi, gg, orc, 6, bias)


def test_swap_of_distant_keys_fails():
    orc, bias = _case()
    gi = orc.idx.copy()
    gi[0, [0, 1]] = gi[0, [1, 0]]
    gg = orc.gates.copy()
    gg[0, [0, 1]] = gg[0, [1, 0]]
    with pytest.raises(AssertionError):
        assert_gemm_parity(gi, gg, orc, 6, bias)


def test_set_change_at_a_near_tie_is_excused_elsewhere_not():
    orc, bias = _case()
    gi = orc.idx.copy()
    gi[1, 2] = 3                                  # token 1: the near-tied (K+1)-th expert instead
    assert_gemm_parity(gi, orc.gates.copy(), orc, 6, bias, gpu_counts=np.bincount(gi.ravel(), minlength=6))
    gi = orc.idx.copy()
    gi[0, 2] = 5                                  # token 0: a set change across a wide gap
    with pytest.raises(AssertionError):
        assert_gemm_parity(gi, orc.gates.copy(), orc, 6, bias)


def test_margin_is_the_documented_one():
    assert MARGIN == 1e-3
