"""Comparison rules between the CUDA library and the CPU oracle.

Logits mode is bit-exact: indices, gates, counts and tile counts are compared
for equality.

GEMM mode: the library accumulates the router projection in fp32 on the
tensor cores, the oracle in fp64, so results are exact except where two keys
that decide the output are closer than MARGIN (in the oracle's fp64 keys):
  - the selected set must equal the oracle's unless the oracle's K-th and
    (K+1)-th biased scores are closer than MARGIN (the token is excused);
  - wherever the sets agree, the slot order must be the oracle's up to swaps
    of experts whose keys are closer than MARGIN: the oracle key of the
    library's slot-k expert is within MARGIN of the oracle's k-th key;
  - per-expert counts may differ by at most the number of excused tokens
    whose selection (on either side) contains that expert;
  - gates agree within GATE_ATOL wherever the selected sets agree.
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


def assert_gemm_parity(gpu_idx, gpu_gates, orc, Nr, bias, gpu_counts=None, margin=MARGIN):
    """orc: oracle.router_gemm(..., want_scores=True) on the same rows; bias:
    the fp32 bias both sides used."""
    gi = np.asarray(gpu_idx)
    gg = np.asarray(gpu_gates, dtype=np.float64)
    oi = orc.idx
    assert orc.scores is not None, "the oracle result needs want_scores=True"
    keys = orc.scores + np.asarray(bias, dtype=np.float32).astype(np.float64)[None, :]
    excused = orc.gap < margin
    same = np.all(np.sort(gi, 1) == np.sort(oi, 1), axis=1)
    bad = np.nonzero(~excused & ~same)[0]
    assert bad.size == 0, "non-excused tokens select different experts: %d (first row %d gpu %s orc %s)" % (
        bad.size, bad[0], gi[bad[0]], oi[bad[0]])
    rows = np.nonzero(same)[0]
    if rows.size:
        kg = np.take_along_axis(keys[rows], gi[rows].astype(np.int64), 1)
        ko = np.take_along_axis(keys[rows], oi[rows].astype(np.int64), 1)
        off = np.abs(kg - ko)
        worst = int(np.argmax(off.max(1)))
        assert off.max() < margin, "slot order differs beyond near-ties (row %d gpu %s orc %s, key gap %g)" % (
            rows[worst], gi[rows[worst]], oi[rows[worst]], off.max())
    # gates, aligned by expert id
    og = orc.gates
    if rows.size:
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
