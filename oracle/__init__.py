"""Test infrastructure: the fp64 CPU oracle for the MoE router step with SMEBU.

This package is NOT part of the product.  Only the test suite, the smoke check
and the benchmark's CPU-baseline leg may import it.  It wraps the plain C file
``ebl_oracle.c`` (built into ``libebl_oracle.so`` beside it) with numpy
marshalling and nothing else: every step of the arithmetic lives in the C file,
each function there citing the page, section and equation it restates.

The oracle shares no code with the CUDA library and never imports it.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from typing import NamedTuple

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "ebl_oracle.c")
_LIB_PATH = os.path.join(_HERE, "libebl_oracle.so")

ORC_OK = 0
ORC_EINVAL = -1
ORC_EDATA = -4

# Flags fix the floating-point semantics the oracle promises: no contraction of
# a*b+c into one rounding, no reassociation, binary64/binary32 as written.
CFLAGS = ["-O2", "-fPIC", "-shared", "-fopenmp", "-ffp-contract=off",
          "-fno-fast-math", "-fexcess-precision=standard", "-std=c11"]


def build(force: bool = False) -> str:
    """Compile ebl_oracle.c into libebl_oracle.so (gcc, OpenMP)."""
    if (not force and os.path.exists(_LIB_PATH)
            and os.path.getmtime(_LIB_PATH) >= os.path.getmtime(_SRC)):
        return _LIB_PATH
    tmp = _LIB_PATH + ".tmp.%d" % os.getpid()
    subprocess.check_call(["gcc", *CFLAGS, "-o", tmp, _SRC, "-lm"])
    os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


_libs = {}
_active = [None]


def _bind(path):
    lib = ctypes.CDLL(path)
    P = ctypes.c_void_p
    i64 = ctypes.c_int64
    i32 = ctypes.c_int
    f32 = ctypes.c_float
    lib.orc_router_gemm.argtypes = [P, P, P, i64, i32, i32, i32, P, P, P, P, P, P]
    lib.orc_router_gemm.restype = i32
    lib.orc_router_logits.argtypes = [P, P, i64, i32, i32, P, P, P, P, P, i32]
    lib.orc_router_logits.restype = i32
    lib.orc_router_zloss.argtypes = [P, P, i64, i32, i32]
    lib.orc_router_zloss.restype = ctypes.c_double
    lib.orc_maxvio.argtypes = [P, i32, P, P]
    lib.orc_maxvio.restype = ctypes.c_double
    lib.orc_smebu.argtypes = [P, P, P, i32, f32, f32, f32, P]
    lib.orc_smebu.restype = i32
    lib.orc_smebu_linear.argtypes = [P, P, P, i32, f32, f32, P]
    lib.orc_smebu_linear.restype = i32
    lib.orc_sign_update.argtypes = [P, P, i32, f32, P]
    lib.orc_sign_update.restype = i32
    lib.orc_dispatch.argtypes = [P, i64, i32, i32, P, P, P]
    lib.orc_dispatch.restype = i32
    lib.orc_gather_rows.argtypes = [P, P, i64, i32, P]
    lib.orc_gather_rows.restype = None
    lib.orc_combine.argtypes = [P, P, P, i64, i32, i32, i64, P, P]
    lib.orc_combine.restype = i32
    lib.orc_seq_balance.argtypes = [P, P, i64, i32, i32, i64, ctypes.c_double, P, P, P, P]
    lib.orc_seq_balance.restype = i32
    lib.orc_tile_psum.argtypes = [P, i64, i32, i32, P]
    lib.orc_tile_psum.restype = i32
    lib.orc_seq_balance_tiles.argtypes = [P, P, i64, i32, i32, i64, i32, ctypes.c_double, P, P]
    lib.orc_seq_balance_tiles.restype = i32
    return lib


def _load():
    if _active[0] is not None:
        return _active[0]
    if _LIB_PATH not in _libs:
        build()
        _libs[_LIB_PATH] = _bind(_LIB_PATH)
    return _libs[_LIB_PATH]


class use_library:
    """Context manager: route this module's calls to another build of the
    oracle (the planted-mistake tests compile altered copies of the C file)."""

    def __init__(self, path):
        self.path = path

    def __enter__(self):
        if self.path not in _libs:
            _libs[self.path] = _bind(self.path)
        self._prev = _active[0]
        _active[0] = _libs[self.path]
        return self

    def __exit__(self, *exc):
        _active[0] = self._prev
        return False


def compile_variant(src_text: str, out_path: str) -> str:
    """Compile C source text with the oracle's flags into out_path."""
    c_path = out_path + ".c"
    with open(c_path, "w") as f:
        f.write(src_text)
    subprocess.check_call(["gcc", *CFLAGS, "-o", out_path, c_path, "-lm"])
    return out_path


def source_text() -> str:
    with open(_SRC) as f:
        return f.read()


def _ptr(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def _c(a, dtype):
    return np.ascontiguousarray(a, dtype=dtype)


def _bf16_bits(a) -> np.ndarray:
    """Accept uint16 bit patterns (numpy) or a torch bfloat16 tensor."""
    if hasattr(a, "dtype") and str(a.dtype) == "torch.bfloat16":
        import torch
        return a.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16)
    a = np.asarray(a)
    if a.dtype != np.uint16:
        raise TypeError("bf16 input must be uint16 bit patterns or a torch.bfloat16 tensor")
    return np.ascontiguousarray(a)


class RouterResult:
    def __init__(self, **kw):
        self.__dict__.update(kw)


def router_gemm(hidden, W, bias, K, counts=None, want_logits=False, want_scores=False):
    """GEMM-mode router step in fp64.  hidden [T,d], W [Nr,d] as bf16 bits."""
    h = _bf16_bits(hidden)
    w = _bf16_bits(W)
    T, d = h.shape
    Nr = w.shape[0]
    b = _c(bias, np.float32)
    idx = np.empty((T, K), np.int32)
    gates = np.empty((T, K), np.float64)
    cnt = np.zeros(Nr, np.int64) if counts is None else counts
    logits = np.empty((T, Nr), np.float64) if want_logits else None
    scores = np.empty((T, Nr), np.float64) if want_scores else None
    gap = np.empty(T, np.float64)
    rc = _load().orc_router_gemm(_ptr(h), _ptr(w), _ptr(b), T, d, Nr, K, _ptr(idx), _ptr(gates),
                                 _ptr(cnt), _ptr(logits), _ptr(scores), _ptr(gap))
    if rc != ORC_OK:
        raise ValueError("orc_router_gemm returned %d" % rc)
    return RouterResult(idx=idx, gates=gates, counts=cnt, logits=logits, scores=scores, gap=gap)


def router_logits(logits, bias, K, counts=None, want_scores=False, tile_tokens=0):
    """Logits-mode router step (fp32 scores/keys, fp64-rounded sigmoid)."""
    x = _c(logits, np.float32)
    T, Nr = x.shape
    b = _c(bias, np.float32)
    idx = np.empty((T, K), np.int32)
    gates = np.empty((T, K), np.float32)
    cnt = np.zeros(Nr, np.int64) if counts is None else counts
    scores = np.empty((T, Nr), np.float32) if want_scores else None
    tiles = (T + tile_tokens - 1) // tile_tokens if tile_tokens else 0
    tc = np.empty((tiles, Nr), np.int32) if tile_tokens else None
    rc = _load().orc_router_logits(_ptr(x), _ptr(b), T, Nr, K, _ptr(idx), _ptr(gates), _ptr(cnt),
                                   _ptr(scores), _ptr(tc), int(tile_tokens))
    if rc != ORC_OK:
        raise ValueError("orc_router_logits returned %d" % rc)
    return RouterResult(idx=idx, gates=gates, counts=cnt, scores=scores, tile_counts=tc)


def router_zloss(hidden, W):
    """sum_t (logsumexp_i x_{t,i})^2 of the fp64 router logits."""
    h = _bf16_bits(hidden)
    w = _bf16_bits(W)
    return float(_load().orc_router_zloss(_ptr(h), _ptr(w), h.shape[0], h.shape[1], w.shape[0]))


def maxvio(counts):
    c = _c(counts, np.int64)
    mx = np.zeros(1, np.int64)
    mn = np.zeros(1, np.int64)
    v = _load().orc_maxvio(_ptr(c), c.size, _ptr(mx), _ptr(mn))
    return v, int(mx[0]), int(mn[0])


def smebu(counts, bias, momentum, lam=5e-4, beta=0.5, kappa=2.0):
    """One SMEBU step; bias and momentum (float32 arrays) are updated in place."""
    c = _c(counts, np.int64)
    assert bias.dtype == np.float32 and momentum.dtype == np.float32
    assert bias.flags.c_contiguous and momentum.flags.c_contiguous
    mv = np.zeros(1, np.float32)
    rc = _load().orc_smebu(_ptr(c), _ptr(bias), _ptr(momentum), c.size, lam, beta, kappa, _ptr(mv))
    return rc, float(mv[0])


def smebu_linear(counts, bias, momentum, lam=5e-4, beta=0.5):
    c = _c(counts, np.int64)
    assert bias.dtype == np.float32 and momentum.dtype == np.float32
    mv = np.zeros(1, np.float32)
    rc = _load().orc_smebu_linear(_ptr(c), _ptr(bias), _ptr(momentum), c.size, lam, beta, _ptr(mv))
    return rc, float(mv[0])


def sign_update(counts, bias, gamma=1e-3):
    """One aux-loss-free sign step; bias (float32) is updated in place."""
    c = _c(counts, np.int64)
    assert bias.dtype == np.float32 and bias.flags.c_contiguous
    mv = np.zeros(1, np.float32)
    rc = _load().orc_sign_update(_ptr(c), _ptr(bias), c.size, gamma, _ptr(mv))
    return rc, float(mv[0])


def dispatch(idx, Nr):
    """Stable expert-sorted dispatch of the (token, slot) pairs of idx [T,K]."""
    i = _c(idx, np.int32)
    T, K = i.shape
    offsets = np.empty(Nr + 1, np.int32)
    perm = np.empty(T * K, np.int32)
    dest = np.empty(T * K, np.int32)
    rc = _load().orc_dispatch(_ptr(i), T, K, Nr, _ptr(offsets), _ptr(perm), _ptr(dest))
    if rc != ORC_OK:
        raise ValueError("orc_dispatch returned %d" % rc)
    return offsets, perm, dest


def gather_rows(hidden, perm):
    h = _bf16_bits(hidden)
    p = _c(perm, np.int32)
    X = np.empty((p.size, h.shape[1]), np.uint16)
    _load().orc_gather_rows(_ptr(h), _ptr(p), p.size, h.shape[1], _ptr(X))
    return X


def combine(Y, gates, dest, want64=True, want32=True):
    """out[t] = sum_k g[t,k] * Y[dest[t*K+k]] in fp64 and as the fp32 fma chain."""
    y = _bf16_bits(Y)
    g = _c(gates, np.float32)
    T, K = g.shape
    d = y.shape[1]
    dst = _c(dest, np.int32).reshape(-1)
    o64 = np.empty((T, d), np.float64) if want64 else None
    o32 = np.empty((T, d), np.float32) if want32 else None
    rc = _load().orc_combine(_ptr(y), _ptr(g), _ptr(dst), T, d, K, y.shape[0], _ptr(o64), _ptr(o32))
    if rc != ORC_OK:
        raise ValueError("orc_combine returned %d" % rc)
    return o64, o32


class SeqBalance(NamedTuple):
    loss: float             # mean over the sequences of the batch
    loss_seq: np.ndarray    # fp64 [B]
    f: np.ndarray           # fp64 [B, N_r]
    P: np.ndarray           # fp64 [B, N_r]


def seq_balance(scores, idx, seq_len, alpha=5e-5):
    """Sequence-wise balance loss from the router's sigmoid scores [T,N_r]
    and selections [T,K] (sequences of seq_len consecutive tokens)."""
    s = _c(scores, np.float64)
    i = _c(idx, np.int32)
    T, Nr = s.shape
    K = i.shape[1]
    B = T // seq_len if seq_len > 0 else 0
    f = np.zeros((max(B, 1), Nr))
    P = np.zeros((max(B, 1), Nr))
    ls = np.zeros(max(B, 1))
    loss = np.zeros(1)
    rc = _load().orc_seq_balance(_ptr(s), _ptr(i), T, Nr, K, seq_len, alpha, _ptr(f), _ptr(P), _ptr(ls), _ptr(loss))
    if rc != 0:
        raise ValueError("orc_seq_balance returned %d" % rc)
    return SeqBalance(float(loss[0]), ls, f, P)


def tile_psum(scores, tile_tokens=128):
    """Per-tile sums of the normalised scores s / sum_j s: fp64 [ceil(T/tile), N_r]."""
    s = _c(scores, np.float64)
    T, Nr = s.shape
    out = np.zeros(((T + tile_tokens - 1) // tile_tokens, Nr))
    rc = _load().orc_tile_psum(_ptr(s), T, Nr, tile_tokens, _ptr(out))
    if rc != 0:
        raise ValueError("orc_tile_psum returned %d" % rc)
    return out


def seq_balance_tiles(tile_counts, psum, T, K, seq_len, alpha=5e-5, tile_tokens=128):
    """The same loss from per-tile loads and per-tile normalised-score sums.
    Returns (loss, loss_seq fp64 [B])."""
    c = _c(tile_counts, np.int32)
    q = _c(psum, np.float64)
    Nr = c.shape[1]
    B = T // seq_len if seq_len > 0 else 0
    ls = np.zeros(max(B, 1))
    loss = np.zeros(1)
    rc = _load().orc_seq_balance_tiles(_ptr(c), _ptr(q), T, Nr, K, seq_len, tile_tokens, alpha, _ptr(ls), _ptr(loss))
    if rc != 0:
        raise ValueError("orc_seq_balance_tiles returned %d" % rc)
    return float(loss[0]), ls
