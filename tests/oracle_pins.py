"""Pins for the CPU oracle: checks of `oracle` against what the pages and the
mathematics fix, independent of the oracle's own code.

Each pin is a function with no arguments that raises AssertionError on
failure.  test_oracle_pins.py runs them against the oracle;
test_oracle_mutants.py runs them against copies of the oracle with a planted
mistake and expects every copy to fail at least one pin.

What pins what:
  - Top-K and the bias/gate split: brute-force rank enumeration on tiny expert
    counts; hand-derived tie cases (golden/topk_ties.txt); the b = 0 special
    case equal to a library top-k of the logits; +10 bias forcing an expert;
    gates unchanged by the bias.
  - Router projection and sigmoid: numpy matmul of the widened bf16 inputs and
    scipy's expit (independent library routines).
  - SMEBU: hand-derived steps (golden/smebu_overload_2x.txt), scale invariance,
    oddness, zero-sum step, balance fixed point, closed-form trajectory under
    constant counts, step bounds.
  - Sign update: closed-form trajectory, zero-mean bias, sign(0) = 0.
  - MaxVio: hand examples (golden/maxvio.txt).
  - Per-tile loads (logits mode): numpy bincount of each 128-token tile's
    selections, summing to the per-expert counts.
  - The near-tie gap that GEMM-mode parity uses to excuse tokens: the K-th
    minus the (K+1)-th largest biased score, from a numpy sort of the scores.
  - Dispatch: numpy stable argsort; permutation and offset invariants.
  - Combine: numpy einsum in fp64; the identity-expert round trip; the fp32
    chain within its rounding bound.
  - Sequence-wise balance loss: two hand-derived examples
    (golden/seq_balance.txt); equal scores give exactly alpha; sum_i P_i = 1
    and sum_i f_i = N_r per sequence; f from a numpy histogram; invariance
    under a repeated batch and under shuffles inside a sequence; the per-tile
    pieces add up to the per-sequence values.
"""
from __future__ import annotations

import math
import os

import numpy as np
from scipy.special import expit

import oracle

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")
F32_EPS = 2.0 ** -24


# ----------------------------------------------------------------- helpers

def _bf16(a: np.ndarray) -> np.ndarray:
    """float -> bf16 bit patterns, round to nearest even (for test inputs)."""
    f = np.ascontiguousarray(a, dtype=np.float32).view(np.uint32).astype(np.uint64)
    rounded = (f + 0x7FFF + ((f >> 16) & 1)) >> 16
    return rounded.astype(np.uint16)


def _bf16_to_f64(h: np.ndarray) -> np.ndarray:
    return (h.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def _brute_ranks(key: np.ndarray) -> np.ndarray:
    """rank_i = #{j : key_j > key_i or (key_j == key_i and j < i)}."""
    n = key.shape[-1]
    j = np.arange(n)
    gt = key[..., None, :] > key[..., :, None]
    eq = (key[..., None, :] == key[..., :, None]) & (j[None, :] < j[:, None])
    return (gt | eq).sum(-1)


def _select_from_ranks(ranks: np.ndarray, K: int) -> np.ndarray:
    """slot k holds the expert whose rank is k."""
    T, n = ranks.shape
    out = np.full((T, K), -1, np.int32)
    for t in range(T):
        for i in range(n):
            if ranks[t, i] < K:
                out[t, ranks[t, i]] = i
    return out


def _read_kv(name):
    rows = {}
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            k, *v = line.split()
            rows[k] = v
    return rows


# -------------------------------------------------------------- Top-K pins

def pin_topk_bruteforce_logits_mode():
    rng = np.random.default_rng(11)
    for Nr in range(1, 11):
        for K in range(1, Nr + 1):
            T = 64
            x = rng.standard_normal((T, Nr)).astype(np.float32)
            x[: T // 2] = np.round(x[: T // 2] * 2) / 2          # forced score ties
            b = (rng.integers(-2, 3, Nr) * 0.25).astype(np.float32)  # forced key ties
            r = oracle.router_logits(x, b, K, want_scores=True)
            key = (r.scores + b[None, :]).astype(np.float32)   # binary32 add
            want = _select_from_ranks(_brute_ranks(key), K)
            assert np.array_equal(r.idx, want), (Nr, K)
            assert np.array_equal(r.counts, np.bincount(want.ravel(), minlength=Nr)), (Nr, K)


def pin_topk_golden_ties():
    g = _read_kv("topk_ties.txt")
    Nr = int(g["nr"][0])
    b = np.array([float(v) for v in g["bias"]], np.float32)
    x = np.zeros((3, Nr), np.float32)
    for K in range(1, Nr + 1):
        want = np.array([int(v) for v in g["k%d" % K]], np.int32)
        r = oracle.router_logits(x, b, K)
        assert np.array_equal(r.idx, np.tile(want, (3, 1))), K
        assert np.all(r.gates == np.float32(1.0 / K)), K
        h = np.zeros((3, 8), np.uint16)
        w = np.zeros((Nr, 8), np.uint16)
        rg = oracle.router_gemm(h, w, b, K)
        assert np.array_equal(rg.idx, np.tile(want, (3, 1))), K
        assert np.allclose(rg.gates, 1.0 / K, rtol=0, atol=1e-15), K


def pin_gemm_matches_library_and_bruteforce():
    rng = np.random.default_rng(12)
    for Nr in (1, 2, 3, 5, 8, 10):
        for K in sorted({1, (Nr + 1) // 2, Nr}):
            T, d = 40, 24
            h = _bf16(rng.standard_normal((T, d)))
            w = _bf16(rng.standard_normal((Nr, d)) * 0.3)
            b = (rng.standard_normal(Nr) * 0.05).astype(np.float32)
            r = oracle.router_gemm(h, w, b, K, want_logits=True, want_scores=True)
            x = _bf16_to_f64(h) @ _bf16_to_f64(w).T            # library matmul
            assert np.allclose(r.logits, x, rtol=1e-13, atol=1e-13), (Nr, K)
            s = expit(x)                                        # library sigmoid
            assert np.allclose(r.scores, s, rtol=1e-14, atol=0), (Nr, K)
            key = s + b.astype(np.float64)[None, :]
            want = _select_from_ranks(_brute_ranks(key), K)
            assert np.array_equal(r.idx, want), (Nr, K)
            sel = np.take_along_axis(s, want.astype(np.int64), 1)
            assert np.allclose(r.gates, sel / sel.sum(1, keepdims=True), rtol=1e-14, atol=0)


def pin_zero_bias_is_topk_of_logits():
    import torch
    rng = np.random.default_rng(13)
    T, d, Nr, K = 64, 64, 32, 6
    h = _bf16(rng.standard_normal((T, d)))
    w = _bf16(rng.standard_normal((Nr, d)) * 0.2)
    r = oracle.router_gemm(h, w, np.zeros(Nr, np.float32), K, want_logits=True)
    ref = torch.topk(torch.from_numpy(r.logits), K, dim=1, sorted=True).indices.numpy()
    assert np.array_equal(r.idx, ref.astype(np.int32))
    xl = rng.standard_normal((T, Nr)).astype(np.float32)
    rl = oracle.router_logits(xl, np.zeros(Nr, np.float32), K)
    refl = torch.topk(torch.from_numpy(xl.astype(np.float64)), K, dim=1, sorted=True).indices.numpy()
    assert np.array_equal(rl.idx, refl.astype(np.int32))


def pin_tile_counts_are_tile_histograms():
    rng = np.random.default_rng(29)
    T, Nr, K, tile = 1000, 16, 3, 128           # a ragged last tile
    x = rng.standard_normal((T, Nr)).astype(np.float32)
    b = (rng.standard_normal(Nr) * 0.1).astype(np.float32)
    r = oracle.router_logits(x, b, K, tile_tokens=tile)
    tiles = (T + tile - 1) // tile
    assert r.tile_counts.shape == (tiles, Nr)
    for j in range(tiles):
        want = np.bincount(r.idx[j * tile:(j + 1) * tile].ravel(), minlength=Nr)
        assert np.array_equal(r.tile_counts[j], want), j
    assert np.array_equal(r.tile_counts.sum(0), r.counts)


def pin_gap_is_kth_minus_next_biased_score():
    rng = np.random.default_rng(31)
    T, d, Nr, K = 200, 64, 24, 5
    h = _bf16(rng.standard_normal((T, d)))
    w = _bf16(rng.standard_normal((Nr, d)) * 0.2)
    b = (rng.standard_normal(Nr) * 0.05).astype(np.float32)
    r = oracle.router_gemm(h, w, b, K, want_scores=True)
    keys = np.sort(r.scores + b.astype(np.float64), axis=1)[:, ::-1]
    want = keys[:, K - 1] - keys[:, K]
    assert np.all(r.gap >= 0)
    assert np.allclose(r.gap, want, rtol=0, atol=1e-15)
    rk = oracle.router_gemm(h, w, b, Nr)        # K = N_r: nothing is left out
    assert np.all(np.isinf(rk.gap))


def pin_bias_forces_expert():
    rng = np.random.default_rng(14)
    T, d, Nr, K = 50, 32, 16, 3
    h = _bf16(rng.standard_normal((T, d)))
    w = _bf16(rng.standard_normal((Nr, d)) * 0.2)
    for j in (0, 7, 15):
        b = np.zeros(Nr, np.float32)
        b[j] = 10.0
        r = oracle.router_gemm(h, w, b, K)
        assert np.all(r.idx[:, 0] == j) and r.counts[j] == T
        rl = oracle.router_logits(rng.standard_normal((T, Nr)).astype(np.float32), b, K)
        assert np.all(rl.idx[:, 0] == j) and rl.counts[j] == T


def pin_bias_never_touches_gates():
    rng = np.random.default_rng(15)
    T, d, Nr, K = 200, 32, 16, 4
    h = _bf16(rng.standard_normal((T, d)))
    w = _bf16(rng.standard_normal((Nr, d)) * 0.3)
    b = (rng.standard_normal(Nr) * 0.02).astype(np.float32)
    r0 = oracle.router_gemm(h, w, np.zeros(Nr, np.float32), K, want_scores=True)
    r1 = oracle.router_gemm(h, w, b, K, want_scores=True)
    assert np.array_equal(r0.scores, r1.scores)
    same = np.all(np.sort(r0.idx, 1) == np.sort(r1.idx, 1), axis=1)
    assert same.sum() > 10 and (~same).sum() > 10
    for t in np.nonzero(same)[0]:
        g0 = dict(zip(r0.idx[t], r0.gates[t]))
        g1 = dict(zip(r1.idx[t], r1.gates[t]))
        for e in g0:
            assert abs(g0[e] - g1[e]) <= 1e-15
    # gates follow the unbiased scores of the selected experts
    sel = np.take_along_axis(r1.scores, r1.idx.astype(np.int64), 1)
    assert np.allclose(r1.gates, sel / sel.sum(1, keepdims=True), rtol=1e-14, atol=0)


def pin_gates_normalised():
    rng = np.random.default_rng(16)
    T, d, Nr = 100, 16, 12
    h = _bf16(rng.standard_normal((T, d)))
    w = _bf16(rng.standard_normal((Nr, d)) * 0.3)
    b = (rng.standard_normal(Nr) * 0.05).astype(np.float32)
    for K in (1, 2, 5, 12):
        r = oracle.router_gemm(h, w, b, K)
        assert np.allclose(r.gates.sum(1), 1.0, rtol=0, atol=4e-16), K
        if K == 1:
            assert np.all(r.gates == 1.0)
        else:
            assert np.all((r.gates > 0) & (r.gates < 1))
        rl = oracle.router_logits(rng.standard_normal((T, Nr)).astype(np.float32), b, K)
        assert np.allclose(rl.gates.astype(np.float64).sum(1), 1.0, rtol=0, atol=K * F32_EPS)


def pin_sigmoid_symmetry_and_rounding():
    rng = np.random.default_rng(17)
    T, d, Nr = 30, 16, 8
    h = _bf16(rng.standard_normal((T, d)))
    w = _bf16(rng.standard_normal((Nr, d)) * 0.3)
    neg = h ^ np.uint16(0x8000)                     # exact negation of bf16
    zero = np.zeros(Nr, np.float32)
    sp = oracle.router_gemm(h, w, zero, 1, want_scores=True).scores
    sn = oracle.router_gemm(neg, w, zero, 1, want_scores=True).scores
    assert np.allclose(sp + sn, 1.0, rtol=0, atol=5e-16)
    s0 = oracle.router_gemm(np.zeros((2, d), np.uint16), w, zero, 1, want_scores=True).scores
    assert np.all(s0 == 0.5)
    x = (rng.standard_normal((200, 64)) * 4).astype(np.float32)
    sl = oracle.router_logits(x, np.zeros(64, np.float32), 2, want_scores=True).scores
    ref = expit(x.astype(np.float64)).astype(np.float32)
    mism = sl != ref
    assert mism.sum() <= 1
    if mism.any():
        assert np.all(np.abs(sl[mism].view(np.int32) - ref[mism].view(np.int32)) <= 1)


# ------------------------------------------------------------- z-loss pins

def pin_zloss_library_and_closed_form():
    from scipy.special import logsumexp
    rng = np.random.default_rng(18)
    T, d, Nr = 50, 40, 24
    h = _bf16(rng.standard_normal((T, d)))
    w = _bf16(rng.standard_normal((Nr, d)) * 0.4)
    x = _bf16_to_f64(h) @ _bf16_to_f64(w).T
    ref = float(np.sum(logsumexp(x, axis=1) ** 2))                 # library logsumexp
    assert abs(oracle.router_zloss(h, w) - ref) <= 1e-12 * ref
    # all logits 0: every row is log(N_r), so the sum is T log^2 N_r
    z = oracle.router_zloss(np.zeros((7, 8), np.uint16), w[:, :8])
    assert abs(z - 7 * math.log(Nr) ** 2) <= 1e-12 * z
    # shifting every logit of a row by c shifts its log-sum-exp by c (large c: no overflow)
    hb = np.zeros((1, d), np.uint16)
    hb[0, 0] = _bf16(np.array([64.0]))[0]
    wb = np.zeros((Nr, d), np.uint16)
    wb[:, 0] = _bf16(np.array([16.0]))[0]                          # every logit = 1024
    z = oracle.router_zloss(hb, wb)
    assert abs(z - (1024.0 + math.log(Nr)) ** 2) <= 1e-9 * z


# -------------------------------------------------------------- SMEBU pins

def pin_smebu_golden_overload():
    g = _read_kv("smebu_overload_2x.txt")
    lam, beta, kappa = float(g["lambda"][0]), float(g["beta"][0]), float(g["kappa"][0])
    for key in ("counts", "counts_scaled"):
        n = np.array([int(v) for v in g[key]], np.int64)
        b = np.zeros(n.size, np.float32)
        m = np.zeros(n.size, np.float32)
        for step in (1, 2):
            rc, _ = oracle.smebu(n, b, m, lam, beta, kappa)
            assert rc == 0
            wm = np.array([float(v) for v in g["m%d" % step]])
            wb = np.array([float(v) for v in g["b%d" % step]])
            assert np.allclose(m, wm, rtol=3 * F32_EPS, atol=0), (key, step, m, wm)
            assert np.allclose(b, wb, rtol=3 * F32_EPS, atol=0), (key, step, b, wb)


def pin_smebu_dead_and_double_load():
    # dead expert: v = 1; 2x loaded: v = -1 (SMEBU note, eqs. (23)-(24))
    lam, kappa = 5e-4, 2.0
    n = np.array([0, 200, 100, 100, 100, 100, 100, 100], np.int64)   # nbar = 100
    b = np.zeros(8, np.float32)
    m = np.zeros(8, np.float32)
    oracle.smebu(n, b, m, lam, 0.0, kappa)   # beta = 0: m = db, b = db
    pre = lam * np.tanh(kappa * np.array([1, -1, 0, 0, 0, 0, 0, 0], np.float64))
    want = pre - pre.mean()
    assert np.allclose(b, want, rtol=3 * F32_EPS, atol=1e-12)
    assert b[0] > 0 and b[1] < 0           # under-used up, over-used down


def pin_smebu_scale_invariance_and_oddness():
    # v depends on n/nbar only (scale invariance), and tanh is odd, so the
    # mirrored loads n' = 2 nbar - n give exactly the negated step.
    rng = np.random.default_rng(21)
    Nr = 64
    half = rng.integers(-100, 101, Nr // 2)
    delta = np.concatenate([half, -rng.permutation(half)])
    base = (100 + delta).astype(np.int64)                  # nbar = 100, 0 <= n <= 200
    mirror = 200 - base
    outs = []
    for n in (base, base * 1000, mirror):
        b = np.zeros(Nr, np.float32)
        m = np.zeros(Nr, np.float32)
        oracle.smebu(n, b, m)
        outs.append((b.copy(), m.copy()))
    assert np.array_equal(outs[0][0], outs[1][0]) and np.array_equal(outs[0][1], outs[1][1])
    assert np.array_equal(outs[0][0], -outs[2][0]) and np.array_equal(outs[0][1], -outs[2][1])
    # mirrored pairs make the pre-centring mean 0: the sign of the step is the sign of v
    v = (100.0 - base) / 100.0
    nz = v != 0
    assert np.all(np.sign(outs[0][0][nz]) == np.sign(v[nz]))


def pin_smebu_zero_sum_and_balance():
    rng = np.random.default_rng(22)
    Nr = 256
    b = (rng.standard_normal(Nr) * 1e-3).astype(np.float32)
    m = np.zeros(Nr, np.float32)
    s0 = b.astype(np.float64).sum()
    bound = 0.0
    for t in range(50):
        n = rng.integers(0, 3000, Nr).astype(np.int64)
        n[0] = 0
        oracle.smebu(n, b, m)
        bound += F32_EPS * float(np.abs(b).astype(np.float64).sum()) + 1e-15
        assert abs(b.astype(np.float64).sum() - s0) <= bound, t
        assert np.all(np.abs(m) <= np.float32(2 * 5e-4))
    # exact balance: every step is 0, so m <- beta m and b <- b + beta m
    n = np.full(Nr, 77, np.int64)
    m0 = m.astype(np.float64).copy()
    b0 = b.astype(np.float64).copy()
    oracle.smebu(n, b, m, beta=0.5)
    assert np.array_equal(m, (0.5 * m0).astype(np.float32))
    assert np.array_equal(b, (b0 + 0.5 * m0).astype(np.float32))
    # sum n = 0: rejected, state untouched
    bb, mm = b.copy(), m.copy()
    rc, _ = oracle.smebu(np.zeros(Nr, np.int64), b, m)
    assert rc == oracle.ORC_EDATA and np.array_equal(b, bb) and np.array_equal(m, mm)


def pin_smebu_closed_form_trajectory():
    # constant counts: the step D is fixed, so m_t = (1 - beta^t) D and
    # b_t = b_0 + D (t - beta (1 - beta^t) / (1 - beta)).  beta = 0.8 so that
    # beta and 1 - beta cannot be confused.
    rng = np.random.default_rng(23)
    Nr, beta, lam, kappa = 32, 0.8, 5e-4, 2.0
    n = rng.integers(0, 500, Nr).astype(np.int64)
    b = np.zeros(Nr, np.float32)
    m = np.zeros(Nr, np.float32)
    oracle.smebu(n, b, m, lam, 0.0, kappa)           # beta = 0: b = m = D (fp32)
    D = b.astype(np.float64).copy()
    assert abs(D.sum()) <= Nr * F32_EPS * np.abs(D).max()
    assert np.all(np.abs(D) <= 2 * lam)
    b = np.zeros(Nr, np.float32)
    m = np.zeros(Nr, np.float32)
    eb = np.zeros(Nr)
    beta32 = float(np.float32(beta))
    for t in range(1, 41):
        oracle.smebu(n, b, m, lam, beta, kappa)
        wm = (1 - beta32 ** t) * D
        wb = D * (t - beta32 * (1 - beta32 ** t) / (1 - beta32))
        em = 4 * F32_EPS * np.abs(D)
        eb += F32_EPS * np.abs(b) + em
        assert np.all(np.abs(m - wm) <= em + 1e-18), t
        assert np.all(np.abs(b - wb) <= eb + t * F32_EPS * np.abs(D) + 1e-18), t


def pin_smebu_linear_variant():
    # linear, unclamped ablation: db = lambda * v
    n = np.array([0, 200, 100, 100], np.int64)
    b = np.zeros(4, np.float32)
    m = np.zeros(4, np.float32)
    oracle.smebu_linear(n, b, m, 5e-4, 0.0)
    pre = 5e-4 * np.array([1.0, -1.0, 0, 0])
    assert np.allclose(b, pre - pre.mean(), rtol=2 * F32_EPS, atol=1e-12)


# ---------------------------------------------------------- sign-update pins

def pin_sign_update_closed_form():
    # constant counts: b_t = (b_0 - mean b_0) + t (db - mean db), sum b_t = 0
    rng = np.random.default_rng(31)
    Nr, gamma = 128, 1e-3
    half = rng.integers(-100, 101, Nr // 2)
    half[:5] = 0                                             # balanced experts: sign(0) = 0
    symmetric = (200 + np.concatenate([half, -half[::-1]])).astype(np.int64)
    skewed = np.full(Nr, 100, np.int64)                      # one hot expert: mean(db) != 0
    skewed[7] = 100 + 50 * Nr
    for n in (symmetric, skewed):
        _sign_update_trajectory(rng, n, Nr, gamma)


def _sign_update_trajectory(rng, n, Nr, gamma):
    nbar = n.sum() / Nr
    b0 = (rng.standard_normal(Nr) * 1e-2).astype(np.float32)
    b = b0.copy()
    db = np.float32(gamma) * np.sign(nbar - n)
    eb = np.zeros(Nr)
    for t in range(1, 31):
        rc, _ = oracle.sign_update(n, b, gamma)
        assert rc == 0
        want = (b0.astype(np.float64) - b0.astype(np.float64).mean()) + t * (db - db.mean())
        # own rounding this step, plus the mean of the errors carried in b
        eb = eb + F32_EPS * np.abs(b) + eb.sum() / Nr + 1e-17
        assert np.all(np.abs(b - want) <= eb), t
        assert abs(b.astype(np.float64).sum()) <= eb.sum(), t


def pin_sign_update_balance():
    Nr = 16
    b = np.linspace(-1e-2, 2e-2, Nr).astype(np.float32)
    want = b.astype(np.float64) - b.astype(np.float64).mean()
    oracle.sign_update(np.full(Nr, 9, np.int64), b, 1e-3)   # sign(0) = 0
    assert np.allclose(b, want, rtol=0, atol=2 * F32_EPS * 0.02)
    n = np.array([10, 30] * (Nr // 2), np.int64)            # nbar = 20
    b = np.zeros(Nr, np.float32)
    oracle.sign_update(n, b, 1e-3)
    assert np.all(b[0::2] == np.float32(1e-3)) and np.all(b[1::2] == np.float32(-1e-3))


# -------------------------------------------------------------- MaxVio pins

def pin_maxvio_golden():
    with open(os.path.join(GOLDEN, "maxvio.txt")) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            val, counts = line.split(":")
            n = np.array([int(v) for v in counts.split()], np.int64)
            got, mx, mn = oracle.maxvio(n)
            want = float(val)
            assert (got == want) if math.isfinite(want) else math.isinf(got), (line, got)
            assert mx == n.max() and mn == n.min()
            b = np.zeros(n.size, np.float32)
            m = np.zeros(n.size, np.float32)
            _, mv = oracle.smebu(n, b, m)
            assert (mv == np.float32(want)) if math.isfinite(want) else math.isinf(mv)


# ------------------------------------------------------------ dispatch pins

def pin_dispatch_stable_sort():
    rng = np.random.default_rng(41)
    for (T, K, Nr) in ((1, 1, 1), (7, 3, 5), (300, 4, 16), (1000, 8, 64)):
        idx = np.stack([rng.choice(Nr, K, replace=False) for _ in range(T)]).astype(np.int32)
        offsets, perm, dest = oracle.dispatch(idx, Nr)
        order = np.argsort(idx.ravel(), kind="stable")      # library stable sort
        assert np.array_equal(perm, (order // K).astype(np.int32))
        inv = np.empty_like(order)
        inv[order] = np.arange(order.size)
        assert np.array_equal(dest, inv.astype(np.int32))
        cnt = np.bincount(idx.ravel(), minlength=Nr)
        assert offsets[0] == 0 and offsets[-1] == T * K
        assert np.array_equal(np.diff(offsets), cnt)
        assert np.array_equal(np.bincount(perm, minlength=T), np.full(T, K))
        h = _bf16(rng.standard_normal((T, 24)))
        X = oracle.gather_rows(h, perm)
        assert np.array_equal(X, h[perm])
    bad = np.array([[0, 5]], np.int32)
    try:
        oracle.dispatch(bad, 5)
    except ValueError:
        pass
    else:
        raise AssertionError("out-of-range expert id accepted")


def pin_combine_library_and_roundtrip():
    rng = np.random.default_rng(42)
    T, K, Nr, d = 200, 4, 16, 40
    idx = np.stack([rng.choice(Nr, K, replace=False) for _ in range(T)]).astype(np.int32)
    g = rng.random((T, K)).astype(np.float32)
    Y = _bf16(rng.standard_normal((T * K, d)))
    _, _, dest = oracle.dispatch(idx, Nr)
    o64, o32 = oracle.combine(Y, g, dest)
    Yd = _bf16_to_f64(Y)[dest.reshape(T, K)]                     # [T,K,d]
    ref = np.einsum("tk,tkd->td", g.astype(np.float64), Yd)      # library contraction
    assert np.allclose(o64, ref, rtol=1e-15, atol=1e-15)
    bound = K * F32_EPS * np.einsum("tk,tkd->td", np.abs(g.astype(np.float64)), np.abs(Yd))
    assert np.all(np.abs(o32.astype(np.float64) - ref) <= bound + 1e-30)
    # identity expert: dispatch the hidden rows, combine with normalised gates
    h = _bf16(rng.standard_normal((T, d)))
    offsets, perm, dest = oracle.dispatch(idx, Nr)
    X = oracle.gather_rows(h, perm)
    gn = (g / g.sum(1, keepdims=True)).astype(np.float32)
    r64, r32 = oracle.combine(X, gn, dest)
    hd = _bf16_to_f64(h)
    assert np.allclose(r64, hd, rtol=(K + 1) * F32_EPS, atol=0)
    assert np.allclose(r32, hd, rtol=(2 * K + 1) * F32_EPS, atol=0)



# ------------------------------------------------- sequence-wise balance pins

def _frac(v):
    from fractions import Fraction
    return float(Fraction(v))


def pin_seq_balance_golden():
    g = _read_kv("seq_balance.txt")
    for ex in ("A", "B"):
        T, Nr, K, S = (int(v) for v in g[ex + "_shape"])
        scores = np.array([_frac(v) for v in g[ex + "_scores"]]).reshape(T, Nr)
        idx = np.array([int(v) for v in g[ex + "_idx"]], np.int32).reshape(T, K)
        r = oracle.seq_balance(scores, idx, S, _frac(g[ex + "_alpha"][0]))
        for key, got in (("f", r.f), ("P", r.P), ("loss_seq", r.loss_seq)):
            want = np.array([_frac(v) for v in g[ex + "_" + key]])
            assert np.allclose(got.reshape(-1), want, rtol=1e-14, atol=1e-300), (ex, key, got, want)
        want = _frac(g[ex + "_loss"][0])
        assert abs(r.loss - want) <= 1e-14 * want, (ex, r.loss, want)


def pin_seq_balance_equal_scores_and_invariants():
    rng = np.random.default_rng(29)
    Nr, K, S, B = 16, 3, 64, 6
    T = B * S
    idx = np.stack([rng.choice(Nr, K, replace=False) for _ in range(T)]).astype(np.int32)
    alpha = 5e-5
    # every score equal: s' = 1/N_r, so P_i = 1/N_r and L = alpha * (sum_i f_i) / N_r = alpha
    r = oracle.seq_balance(np.full((T, Nr), 0.3), idx, S, alpha)
    assert np.allclose(r.loss_seq, alpha, rtol=1e-13, atol=0) and abs(r.loss - alpha) <= 1e-13 * alpha
    scores = expit(rng.standard_normal((T, Nr)) * 2)
    r = oracle.seq_balance(scores, idx, S, alpha)
    assert np.allclose(r.P.sum(1), 1.0, rtol=1e-13, atol=0)          # s' sums to 1 per token
    assert np.allclose(r.f.sum(1), Nr, rtol=1e-13, atol=0)           # K*S selections per sequence
    for b in range(B):                                               # f from a library histogram
        n = np.bincount(idx[b * S:(b + 1) * S].reshape(-1), minlength=Nr)
        assert np.allclose(r.f[b] * (K * S) / Nr, n, rtol=1e-14, atol=1e-14)
    assert abs(r.loss - r.loss_seq.mean()) <= 1e-15 * r.loss
    # a batch of the same sequences twice has the same value; a shuffle of the
    # tokens inside each sequence leaves every sequence's value unchanged
    r2 = oracle.seq_balance(np.concatenate([scores, scores]), np.concatenate([idx, idx]), S, alpha)
    assert abs(r2.loss - r.loss) <= 1e-14 * r.loss
    perm = np.concatenate([b * S + rng.permutation(S) for b in range(B)])
    r3 = oracle.seq_balance(scores[perm], idx[perm], S, alpha)
    assert np.allclose(r3.loss_seq, r.loss_seq, rtol=1e-13, atol=0)
    # all of a sequence on one expert with K = 1: f = N_r there, so L = alpha N_r P_e
    one = np.zeros((S, 1), np.int32) + 5
    r4 = oracle.seq_balance(scores[:S], one, S, alpha)
    assert abs(r4.loss - alpha * Nr * r4.P[0, 5]) <= 1e-14 * r4.loss


def pin_seq_balance_tiles_agree():
    rng = np.random.default_rng(31)
    Nr, K, S, B, tile = 24, 2, 256, 3, 128
    T = B * S
    idx = np.stack([rng.choice(Nr, K, replace=False) for _ in range(T)]).astype(np.int32)
    scores = expit(rng.standard_normal((T, Nr)))
    psum = oracle.tile_psum(scores, tile)
    assert np.allclose(psum.sum(1), tile, rtol=1e-13, atol=0)       # one unit of s' per token
    rag = oracle.tile_psum(scores[:T - 37], tile)
    assert rag.shape[0] == T // tile and abs(rag[-1].sum() - (tile - 37)) <= 1e-12
    counts = np.stack([np.bincount(idx[j * tile:(j + 1) * tile].reshape(-1), minlength=Nr)
                       for j in range(T // tile)]).astype(np.int32)
    ref = oracle.seq_balance(scores, idx, S, 5e-5)
    loss, loss_seq = oracle.seq_balance_tiles(counts, psum, T, K, S, 5e-5, tile)
    assert np.allclose(loss_seq, ref.loss_seq, rtol=1e-12, atol=0) and abs(loss - ref.loss) <= 1e-12 * ref.loss
    per = S // tile
    for b in range(B):
        assert np.allclose(psum[b * per:(b + 1) * per].sum(0), S * ref.P[b], rtol=1e-12, atol=0)

ALL_PINS = [v for k, v in sorted(globals().items()) if k.startswith("pin_")]
