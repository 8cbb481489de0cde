"""Comparison rules between the CUDA library and the CPU oracle.

Logits mode is bit-exact: indices, gates, counts and tile counts are compared
for equality.

GEMM mode: the library accumulates the router projection in fp32 on the
tensor cores, the oracle in fp64, so a token whose K-th and (K+1)-th biased
scores are closer than MARGIN (oracle's fp64 gap) is excused from the
selection comparison.  Every other token must select the same experts in the
same slot order; per-expert counts may differ by at most the number of
excused tokens whose selection (on either side) contains that expert; gates
agree within GATE_ATOL wherever the selected sets agree.
"""
from __future__ import annotations

import numpy as np
import torch

MARGIN = 1e-3
GATE_ATOL = 2e-3
REL_FLOOR = 1e-9      # relative error floor for bias/momentum (b crosses 0)
STATE_RTOL = 1e-6


def to_np(t: torch.Tensor) -> np.ndarray:
    return t.detach().cpu().numpy()


def assert_gemm_parity(gpu_idx, gpu_gates, orc, Nr, gpu_counts=None, margin=MARGIN):
    gi = np.asarray(gpu_idx)
    gg = np.asarray(gpu_gates, dtype=np.float64)
    oi = orc.idx
    excused = orc.gap < margin
    keep = ~excused
    bad = np.nonzero(np.any(gi[keep] != oi[keep], axis=1))[0]
    assert bad.size == 0, "non-excused tokens differ: %d (first row %s gpu %s orc %s)" % (
        bad.size, np.nonzero(keep)[0][bad[0]], gi[keep][bad[0]], oi[keep][bad[0]])
    same = np.all(np.sort(gi, 1) == np.sort(oi, 1), axis=1)
    # gates, aligned by expert id
    og = orc.gates
    for rows in (np.nonzero(same)[0],):
        if rows.size == 0:
            continue
        a = np.argsort(gi[rows], 1)
        b = np.argsort(oi[rows], 1)
        ga = np.take_along_axis(gg[rows], a, 1)
        gb = np.take_along_axis(og[rows], b, 1)
        err = np.abs(ga - gb).max()
        assert err <= GATE_ATOL, "gate error %g" % err
    if gpu_counts is not None:
        gc = np.asarray(gpu_counts, dtype=np.int64)
        assert np.array_equal(gc, np.bincount(gi.ravel(), minlength=Nr)), "counts != histogram of topk_idx"
        allow = np.zeros(Nr, np.int64)
        ex_rows = np.nonzero(excused)[0]
        for r in ex_rows:
            for e in set(gi[r].tolist()) | set(oi[r].tolist()):
                allow[e] += 1
        diff = np.abs(gc - orc.counts)
        assert np.all(diff <= allow), "count difference beyond excused tokens"
    return int(excused.sum())


def rel_err(x, ref):
    x = np.asarray(x, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    return np.abs(x - ref) / np.maximum(np.abs(ref), REL_FLOOR)


def tile_hist(idx: np.ndarray, Nr: int, tile: int = 128) -> np.ndarray:
    T = idx.shape[0]
    tiles = (T + tile - 1) // tile
    out = np.zeros((tiles, Nr), np.int32)
    for j in range(tiles):
        out[j] = np.bincount(idx[j * tile:(j + 1) * tile].ravel(), minlength=Nr)
    return out
