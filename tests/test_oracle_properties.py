"""Property checks of the CPU oracle on generated inputs (no GPU).

The pins in oracle_pins.py fix the oracle on hand-derived and closed-form
cases; these checks draw many small random problems (hypothesis, derandomised
so every run sees the same examples) and assert what the mathematics fixes for
any input:
  - Top-K (logits mode): selected experts are exactly those whose rank
    #{j : key_j > key_i or (key_j == key_i and j < i)} is below K, in rank
    order; gates sum to 1.
  - SMEBU ("SMEBU Load Balancing", eqs. (23)-(28)): the re-centred step sums to
    zero, so sum b changes only by rounding; |m| <= 2 lambda (1 - beta) after a
    step from m = 0; the step falls with the load: every expert above the mean
    load gets a smaller step than every expert below it.
  - Sign update (eqs. (20)-(22)): the bias has zero mean after a step.
  - Dispatch: perm is a permutation of the pairs' tokens, offsets are the
    exclusive scan of the loads, and each expert's pairs keep pair order.
  - Sequence-wise balance loss (the reading of eqs. (29)-(32)): sum_i P_i = 1,
    sum_i f_i = N_r per sequence, equal scores give alpha, and the per-tile
    pieces regroup to the same values.
"""
import numpy as np
from hypothesis import given, settings
from hypothesis import strategies as st

import oracle

PROFILE = settings(max_examples=40, deadline=None, derandomize=True)


def _keys_ranked(key):
    n = key.size
    rank = np.array([sum(1 for j in range(n) if key[j] > key[i] or (key[j] == key[i] and j < i)) for i in range(n)])
    return rank


@PROFILE
@given(Nr=st.integers(1, 12), K=st.integers(1, 8), T=st.integers(1, 20), seed=st.integers(0, 2**31 - 1),
       grid=st.booleans())
def test_topk_matches_rank_definition(Nr, K, T, seed, grid):
    K = min(K, Nr)
    rng = np.random.default_rng(seed)
    x = rng.standard_normal((T, Nr)).astype(np.float32)
    if grid:
        x = np.round(x * 2) / 2                                              # many exact ties
    b = (rng.integers(-1, 2, Nr) * 0.25).astype(np.float32)
    r = oracle.router_logits(x, b, K, want_scores=True)
    for t in range(T):
        key = (r.scores[t] + b).astype(np.float32)                           # one fp32 add, as the oracle's
        rank = _keys_ranked(key)
        want = [int(np.nonzero(rank == k)[0][0]) for k in range(K)]
        assert list(r.idx[t]) == want
        assert abs(float(r.gates[t].astype(np.float64).sum()) - 1.0) <= K * 2.0 ** -23


@PROFILE
@given(Nr=st.integers(2, 64), seed=st.integers(0, 2**31 - 1), lam=st.floats(1e-5, 1e-2),
       beta=st.floats(0.0, 0.95), kappa=st.floats(0.5, 4.0))
def test_smebu_step_properties(Nr, seed, lam, beta, kappa):
    rng = np.random.default_rng(seed)
    n = rng.integers(0, 1000, Nr).astype(np.int64)
    n[0] = max(n[0], 1)
    lam, beta, kappa = (float(np.float32(v)) for v in (lam, beta, kappa))
    b = (rng.standard_normal(Nr) * 0.1).astype(np.float32)
    b0 = b.astype(np.float64)
    m = np.zeros(Nr, np.float32)
    rc, _ = oracle.smebu(n, b, m, lam, beta, kappa)
    assert rc == 0
    step = b.astype(np.float64) - b0
    assert abs(step.sum()) <= Nr * 4 * 2.0 ** -24 * (np.abs(b0).max() + 2 * lam)   # re-centred step sums to 0
    assert np.all(np.abs(m) <= 2 * lam * (1 - beta) * (1 + 1e-6))                  # from m = 0: |m| <= (1-b) 2 lam
    nbar = n.mean()
    over = n > nbar * (1 + 1e-9)
    under = n < nbar * (1 - 1e-9)
    # above-mean experts get a smaller step than below-mean ones
    if over.any() and under.any():
        assert step[over].max() < step[under].min()


@PROFILE
@given(Nr=st.integers(1, 64), seed=st.integers(0, 2**31 - 1), gamma=st.floats(1e-5, 1e-2))
def test_sign_update_zero_mean(Nr, seed, gamma):
    rng = np.random.default_rng(seed)
    n = rng.integers(1, 100, Nr).astype(np.int64)
    b = (rng.standard_normal(Nr) * 0.1).astype(np.float32)
    rc, _ = oracle.sign_update(n, b, float(np.float32(gamma)))
    assert rc == 0
    assert abs(float(b.astype(np.float64).sum())) <= Nr * 2.0 ** -24 * (float(np.abs(b).max()) + gamma) * 2


@PROFILE
@given(Nr=st.integers(1, 40), K=st.integers(1, 8), T=st.integers(0, 60), seed=st.integers(0, 2**31 - 1))
def test_dispatch_is_a_stable_expert_sort(Nr, K, T, seed):
    K = min(K, Nr)
    rng = np.random.default_rng(seed)
    rows = [rng.choice(Nr, K, replace=False) for _ in range(T)]
    idx = (np.stack(rows) if rows else np.zeros((0, K))).astype(np.int32).reshape(T, K)
    offsets, perm, dest = oracle.dispatch(idx, Nr)
    loads = np.bincount(idx.reshape(-1), minlength=Nr)
    assert np.array_equal(offsets, np.concatenate([[0], np.cumsum(loads)]))
    assert np.array_equal(np.sort(dest), np.arange(T * K))                 # dest is a permutation of the slots
    p = np.arange(T * K)
    assert np.array_equal(perm[dest], p // K)                               # each slot's row is its token
    for e in range(Nr):
        mine = p[idx.reshape(-1) == e]
        assert np.array_equal(dest[mine], np.arange(offsets[e], offsets[e + 1]))   # pair order kept


@PROFILE
@given(Nr=st.integers(1, 24), K=st.integers(1, 6), S=st.sampled_from([128, 256]), B=st.integers(1, 3),
       seed=st.integers(0, 2**31 - 1))
def test_seq_balance_properties(Nr, K, S, B, seed):
    K = min(K, Nr)
    rng = np.random.default_rng(seed)
    T = S * B
    idx = np.stack([rng.choice(Nr, K, replace=False) for _ in range(T)]).astype(np.int32)
    scores = 1.0 / (1.0 + np.exp(-rng.standard_normal((T, Nr)) * 3))
    alpha = 5e-5
    r = oracle.seq_balance(scores, idx, S, alpha)
    assert np.allclose(r.P.sum(1), 1.0, rtol=1e-12, atol=0)
    assert np.allclose(r.f.sum(1), Nr, rtol=1e-12, atol=0)
    assert np.all(r.loss_seq > 0)
    eq = oracle.seq_balance(np.full((T, Nr), 0.7), idx, S, alpha)
    assert np.allclose(eq.loss_seq, alpha, rtol=1e-12, atol=0)
    counts = np.stack([np.bincount(idx[j * 128:(j + 1) * 128].reshape(-1), minlength=Nr)
                       for j in range(T // 128)]).astype(np.int32)
    loss, loss_seq = oracle.seq_balance_tiles(counts, oracle.tile_psum(scores, 128), T, K, S, alpha, 128)
    assert np.allclose(loss_seq, r.loss_seq, rtol=1e-12, atol=0) and abs(loss - r.loss) <= 1e-12 * r.loss
