"""expert_bias_load_b200 -- MoE router step with aux-loss-free expert-bias
balancing (SMEBU) on B200.

A thin Python binding of libebl.so (C ABI declared in include/ebl.h).  Every
step of the router, the bias updates, dispatch and combine runs in the CUDA
kernels of that library; this module only checks tensor dtypes, devices and
shapes, allocates outputs with torch, and passes pointers and sizes.  There is
no CPU fallback: if libebl.so is missing or cannot be loaded, every call
raises.

Sources of the method: "Arcee Trinity Large Technical Report" section 2.3
("Mixture-of-Experts"); "SMEBU Load Balancing" (study note), eqs. (17),
(20)-(28); "Arcee Halts 400B Blackwell Model Collapse With Dynamic Router
Biases", "The MaxVio Metric and the Day-4 Crisis".
"""
from __future__ import annotations

import ctypes
import os

import torch

__all__ = [
    "EblError", "lib", "lib_path", "tile_tokens", "router_forward", "router_forward_zloss", "router_forward_balance",
    "seq_balance_loss", "balance_stats_logits", "router_forward_logits", "router_forward_logits_balance",
    "smebu_step",
    "smebu_step_layers", "sign_update_step", "moe_dispatch", "moe_combine", "dispatch_workspace_bytes",
    "read_internal_status", "check_finite", "EBL_ST_BAD_EXPERT", "EBL_ST_BAD_DEST", "EBL_ST_EMPTY_LOAD",
    "EBL_ST_TIMEOUT", "EBL_ST_BAD_COUNTS", "EBL_ST_NONFINITE",
    "SMEBU_LAMBDA", "SMEBU_BETA", "SMEBU_KAPPA", "SEQ_BALANCE_ALPHA",
]

_HERE = os.path.dirname(os.path.abspath(__file__))
lib_path = os.path.join(_HERE, "libebl.so")

EBL_OK, EBL_EINVAL, EBL_EUNSUPPORTED, EBL_ECUDA, EBL_EDATA = 0, -1, -2, -3, -4
EBL_ST_BAD_EXPERT, EBL_ST_BAD_DEST, EBL_ST_EMPTY_LOAD, EBL_ST_TIMEOUT, EBL_ST_BAD_COUNTS = 1, 2, 4, 8, 16
EBL_ST_NONFINITE = 32

# Trinity Large's SMEBU constants ("Arcee Trinity Large Technical Report" 2.3)
SMEBU_LAMBDA, SMEBU_BETA, SMEBU_KAPPA = 5e-4, 0.5, 2.0
# coefficient of the sequence-wise balance loss on the Large checkpoint
# ("SMEBU Load Balancing", "How it works")
SEQ_BALANCE_ALPHA = 5e-5

# exported symbol -> (restype, argtypes); the full C ABI of include/ebl.h
_P = ctypes.c_void_p
_I = ctypes.c_int
_F = ctypes.c_float
_SZ = ctypes.c_size_t
SIGNATURES = {
    "ebl_strerror": (ctypes.c_char_p, [_I]),
    "ebl_version": (_I, []),
    "ebl_last_cuda_error": (ctypes.c_char_p, []),
    "ebl_tile_tokens": (_I, []),
    "router_forward": (_I, [_P, _P, _P, _I, _I, _I, _I, _P, _P, _P, _P, _P, _P]),
    "router_forward_zloss": (_I, [_P, _P, _P, _I, _I, _I, _I, _P, _P, _P, _P, _P, _P, _P]),
    "router_forward_logits": (_I, [_P, _P, _I, _I, _I, _P, _P, _P, _P, _P, _P]),
    "router_forward_logits_balance": (_I, [_P, _P, _I, _I, _I, _P, _P, _P, _P, _P, _P, _P]),
    "router_forward_balance": (_I, [_P, _P, _P, _I, _I, _I, _I, _P, _P, _P, _P, _P, _P, _P, _P]),
    "seq_balance_loss": (_I, [_P, _P, _I, _I, _I, _I, _F, _P, _P, _P]),
    "balance_stats_logits": (_I, [_P, _I, _I, _P, _P]),
    "smebu_step": (_I, [_P, _P, _P, _I, _F, _F, _F, _I, _P, _P, _P]),
    "smebu_step_layers": (_I, [_P, _P, _P, _I, _I, _F, _F, _F, _I, _I, _P, _P, _P]),
    "sign_update_step": (_I, [_P, _P, _I, _F, _I, _P, _P, _P]),
    "ebl_dispatch_workspace_bytes": (_SZ, [_I, _I]),
    "moe_dispatch": (_I, [_P, _P, _P, _I, _I, _I, _I, _P, _P, _P, _P, _P, _SZ, _P, _P]),
    "moe_dispatch_static": (_I, [_P, _P, _P, _I, _I, _I, _I, _P, _P, _P, _P, _P, _P]),
    "moe_combine": (_I, [_P, _P, _P, _I, _I, _I, _P, _P, _P]),
    "ebl_read_internal_status": (_I, [_P, _I]),
    "ebl_selftest_wait_timeout": (_I, [_P, ctypes.c_uint, _P]),
    "ebl_selftest_score_error": (_I, [_P, ctypes.c_int64, _P, _P, _P, _P]),
    "ebl_check_finite_f32": (_I, [_P, ctypes.c_int64, _P, _P]),
    "ebl_check_finite_bf16": (_I, [_P, ctypes.c_int64, _P, _P]),
}


class EblError(RuntimeError):
    def __init__(self, fn, code):
        self.code = code
        text = lib().ebl_strerror(code).decode() if _lib is not None else str(code)
        if code == EBL_ECUDA and _lib is not None:
            text += "; " + lib().ebl_last_cuda_error().decode()
        super().__init__("%s failed: %d (%s)" % (fn, code, text))


_lib = None


def lib() -> ctypes.CDLL:
    """Load libebl.so (raises if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(lib_path):
            raise RuntimeError("libebl.so not found at %s; build it with "
                               "`python -m expert_bias_load_b200.build`" % lib_path)
        handle = ctypes.CDLL(lib_path)
        for name, (res, args) in SIGNATURES.items():
            fn = getattr(handle, name)
            fn.restype = res
            fn.argtypes = args
        _lib = handle
    return _lib


def tile_tokens() -> int:
    return lib().ebl_tile_tokens()


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    if stream is None:
        stream = torch.cuda.current_stream()
    elif stream.device.index != torch.cuda.current_device():
        raise ValueError("stream is on %s but the current CUDA device is cuda:%d"
                         % (stream.device, torch.cuda.current_device()))
    return ctypes.c_void_p(stream.cuda_stream)


def _check(t, name, dtype, shape=None):
    if not isinstance(t, torch.Tensor):
        raise TypeError("%s must be a torch.Tensor" % name)
    if t.dtype != dtype:
        raise TypeError("%s must be %s, got %s" % (name, dtype, t.dtype))
    if not t.is_cuda:
        raise ValueError("%s must be on a CUDA device" % name)
    if t.device.index != torch.cuda.current_device():
        # the library launches on the current device; a tensor elsewhere would
        # hand another GPU's pointer to its kernels
        raise ValueError("%s is on %s but the current CUDA device is cuda:%d (use torch.cuda.device(...))"
                         % (name, t.device, torch.cuda.current_device()))
    if not t.is_contiguous():
        raise ValueError("%s must be contiguous" % name)
    if shape is not None and tuple(t.shape) != tuple(shape):
        raise ValueError("%s must have shape %s, got %s" % (name, tuple(shape), tuple(t.shape)))
    return t


def _call(name, *args):
    rc = getattr(lib(), name)(*args)
    if rc != EBL_OK:
        raise EblError(name, rc)


def _out(t, name, shape, dtype, device):
    if t is None:
        return torch.empty(shape, dtype=dtype, device=device)
    return _check(t, name, dtype, shape)


def router_forward(hidden, W_router, bias, K, counts, topk_idx=None, gates=None, tile_counts=None,
                   status=None, stream=None):
    """GEMM-mode router pass (see include/ebl.h).  hidden bf16 [T,d], W_router
    bf16 [N_r,d], bias fp32 [N_r]; counts int32 [N_r] is ACCUMULATED.
    Returns (topk_idx int32 [T,K], gates fp32 [T,K])."""
    _check(hidden, "hidden", torch.bfloat16)
    T, d = hidden.shape
    _check(W_router, "W_router", torch.bfloat16)
    Nr = W_router.shape[0]
    _check(W_router, "W_router", torch.bfloat16, (Nr, d))
    _check(bias, "bias", torch.float32, (Nr,))
    _check(counts, "counts", torch.int32, (Nr,))
    dev = hidden.device
    topk_idx = _out(topk_idx, "topk_idx", (T, K), torch.int32, dev)
    gates = _out(gates, "gates", (T, K), torch.float32, dev)
    if tile_counts is not None:
        _check(tile_counts, "tile_counts", torch.int32, ((T + 127) // 128, Nr))
    if status is not None:
        _check(status, "status", torch.int32, (1,))
    _call("router_forward", _ptr(hidden), _ptr(W_router), _ptr(bias), T, d, Nr, K, _ptr(topk_idx), _ptr(gates),
          _ptr(counts), _ptr(tile_counts), _ptr(status), _stream(stream))
    return topk_idx, gates


def router_forward_zloss(hidden, W_router, bias, K, counts, zloss_sum, topk_idx=None, gates=None, tile_counts=None,
                         status=None, stream=None):
    """router_forward that also adds sum_t logsumexp(x_t)^2 into zloss_sum
    (fp64 [1], caller-zeroed).  Returns (topk_idx, gates)."""
    _check(hidden, "hidden", torch.bfloat16)
    T, d = hidden.shape
    Nr = W_router.shape[0]
    _check(W_router, "W_router", torch.bfloat16, (Nr, d))
    _check(bias, "bias", torch.float32, (Nr,))
    _check(counts, "counts", torch.int32, (Nr,))
    _check(zloss_sum, "zloss_sum", torch.float64, (1,))
    dev = hidden.device
    topk_idx = _out(topk_idx, "topk_idx", (T, K), torch.int32, dev)
    gates = _out(gates, "gates", (T, K), torch.float32, dev)
    if tile_counts is not None:
        _check(tile_counts, "tile_counts", torch.int32, ((T + 127) // 128, Nr))
    _call("router_forward_zloss", _ptr(hidden), _ptr(W_router), _ptr(bias), T, d, Nr, K, _ptr(topk_idx),
          _ptr(gates), _ptr(counts), _ptr(tile_counts), _ptr(zloss_sum), _ptr(status), _stream(stream))
    return topk_idx, gates


def router_forward_balance(hidden, W_router, bias, K, counts, tile_counts, tile_psum, zloss_sum=None, topk_idx=None,
                           gates=None, status=None, stream=None):
    """router_forward that also writes the per-tile statistics of the
    sequence-wise balance loss: tile_counts int32 and tile_psum fp32, both
    [ceil(T/128), N_r] (sums of s / sum_j s over each tile's tokens); with
    zloss_sum (fp64 [1]) it accumulates the z-loss statistic too.
    Returns (topk_idx, gates)."""
    _check(hidden, "hidden", torch.bfloat16)
    T, d = hidden.shape
    Nr = W_router.shape[0]
    _check(W_router, "W_router", torch.bfloat16, (Nr, d))
    _check(bias, "bias", torch.float32, (Nr,))
    _check(counts, "counts", torch.int32, (Nr,))
    tiles = (T + 127) // 128
    _check(tile_counts, "tile_counts", torch.int32, (tiles, Nr))
    _check(tile_psum, "tile_psum", torch.float32, (tiles, Nr))
    if zloss_sum is not None:
        _check(zloss_sum, "zloss_sum", torch.float64, (1,))
    dev = hidden.device
    topk_idx = _out(topk_idx, "topk_idx", (T, K), torch.int32, dev)
    gates = _out(gates, "gates", (T, K), torch.float32, dev)
    _call("router_forward_balance", _ptr(hidden), _ptr(W_router), _ptr(bias), T, d, Nr, K, _ptr(topk_idx),
          _ptr(gates), _ptr(counts), _ptr(tile_counts), _ptr(tile_psum), _ptr(zloss_sum), _ptr(status),
          _stream(stream))
    return topk_idx, gates


def balance_stats_logits(logits, tile_psum=None, stream=None):
    """Logits mode: per-tile sums of s / sum_j s (s the fp64-rounded-once
    score), fp32 [ceil(T/128), N_r].  Returns tile_psum."""
    _check(logits, "logits", torch.float32)
    T, Nr = logits.shape
    tile_psum = _out(tile_psum, "tile_psum", ((T + 127) // 128, Nr), torch.float32, logits.device)
    _call("balance_stats_logits", _ptr(logits), T, Nr, _ptr(tile_psum), _stream(stream))
    return tile_psum


def seq_balance_loss(tile_counts, tile_psum, T, K, seq_len, alpha=SEQ_BALANCE_ALPHA, loss_seq=None, loss=None,
                     stream=None):
    """Sequence-wise balance loss from router_forward_balance's per-tile
    statistics (sequences of seq_len consecutive tokens, seq_len % 128 == 0,
    T % seq_len == 0).  Returns (loss fp64 [1], loss_seq fp64 [T/seq_len])."""
    tiles = (T + 127) // 128
    Nr = tile_counts.shape[1]
    _check(tile_counts, "tile_counts", torch.int32, (tiles, Nr))
    _check(tile_psum, "tile_psum", torch.float32, (tiles, Nr))
    dev = tile_counts.device
    B = T // seq_len if seq_len > 0 else 0
    loss_seq = _out(loss_seq, "loss_seq", (B,), torch.float64, dev)
    loss = _out(loss, "loss", (1,), torch.float64, dev)
    _call("seq_balance_loss", _ptr(tile_counts), _ptr(tile_psum), T, Nr, K, seq_len, alpha, _ptr(loss_seq),
          _ptr(loss), _stream(stream))
    return loss, loss_seq


def router_forward_logits(logits, bias, K, counts, topk_idx=None, gates=None, tile_counts=None, status=None,
                          stream=None):
    """Logits-mode router pass (the bit-exact contract).  logits fp32 [T,N_r]."""
    _check(logits, "logits", torch.float32)
    T, Nr = logits.shape
    _check(bias, "bias", torch.float32, (Nr,))
    _check(counts, "counts", torch.int32, (Nr,))
    dev = logits.device
    topk_idx = _out(topk_idx, "topk_idx", (T, K), torch.int32, dev)
    gates = _out(gates, "gates", (T, K), torch.float32, dev)
    if tile_counts is not None:
        _check(tile_counts, "tile_counts", torch.int32, ((T + 127) // 128, Nr))
    _call("router_forward_logits", _ptr(logits), _ptr(bias), T, Nr, K, _ptr(topk_idx), _ptr(gates),
          _ptr(counts), _ptr(tile_counts), _ptr(status), _stream(stream))
    return topk_idx, gates


def router_forward_logits_balance(logits, bias, K, counts, tile_counts, tile_psum, topk_idx=None, gates=None,
                                  status=None, stream=None):
    """router_forward_logits that also writes the per-tile statistics of the
    sequence-wise balance loss in the same pass over the logits: tile_counts
    int32 and tile_psum fp32, both [ceil(T/128), N_r].  Returns (topk_idx, gates)."""
    _check(logits, "logits", torch.float32)
    T, Nr = logits.shape
    _check(bias, "bias", torch.float32, (Nr,))
    _check(counts, "counts", torch.int32, (Nr,))
    tiles = (T + 127) // 128
    _check(tile_counts, "tile_counts", torch.int32, (tiles, Nr))
    _check(tile_psum, "tile_psum", torch.float32, (tiles, Nr))
    dev = logits.device
    topk_idx = _out(topk_idx, "topk_idx", (T, K), torch.int32, dev)
    gates = _out(gates, "gates", (T, K), torch.float32, dev)
    _call("router_forward_logits_balance", _ptr(logits), _ptr(bias), T, Nr, K, _ptr(topk_idx), _ptr(gates),
          _ptr(counts), _ptr(tile_counts), _ptr(tile_psum), _ptr(status), _stream(stream))
    return topk_idx, gates


def smebu_step(counts, bias, momentum, lam=SMEBU_LAMBDA, beta=SMEBU_BETA, kappa=SMEBU_KAPPA,
               reset_counts=False, maxvio=None, status=None, stream=None):
    """One SMEBU update of bias and momentum (fp32 [N_r], in place)."""
    Nr = bias.shape[0]
    _check(counts, "counts", torch.int32, (Nr,))
    _check(bias, "bias", torch.float32, (Nr,))
    _check(momentum, "momentum", torch.float32, (Nr,))
    if maxvio is not None:
        _check(maxvio, "maxvio", torch.float32, (1,))
    _call("smebu_step", _ptr(counts), _ptr(bias), _ptr(momentum), Nr, lam, beta, kappa, int(bool(reset_counts)),
          _ptr(maxvio), _ptr(status), _stream(stream))


def smebu_step_layers(counts, bias, momentum, lam=SMEBU_LAMBDA, beta=SMEBU_BETA, kappa=SMEBU_KAPPA,
                      linear=False, reset_counts=False, maxvio=None, status=None, stream=None):
    """SMEBU for L layers at once: counts int32 [L,N_r], bias/momentum fp32 [L,N_r]."""
    L, Nr = bias.shape
    _check(counts, "counts", torch.int32, (L, Nr))
    _check(bias, "bias", torch.float32, (L, Nr))
    _check(momentum, "momentum", torch.float32, (L, Nr))
    if maxvio is not None:
        _check(maxvio, "maxvio", torch.float32, (L,))
    _call("smebu_step_layers", _ptr(counts), _ptr(bias), _ptr(momentum), L, Nr, lam, beta, kappa,
          int(bool(linear)), int(bool(reset_counts)), _ptr(maxvio), _ptr(status), _stream(stream))


def sign_update_step(counts, bias, gamma, reset_counts=False, maxvio=None, status=None, stream=None):
    """Aux-loss-free sign update of bias (fp32 [N_r], in place)."""
    Nr = bias.shape[0]
    _check(counts, "counts", torch.int32, (Nr,))
    _check(bias, "bias", torch.float32, (Nr,))
    _call("sign_update_step", _ptr(counts), _ptr(bias), Nr, gamma, int(bool(reset_counts)), _ptr(maxvio),
          _ptr(status), _stream(stream))


def dispatch_workspace_bytes(T, Nr) -> int:
    return int(lib().ebl_dispatch_workspace_bytes(T, Nr))


def moe_dispatch(hidden, topk_idx, Nr, tile_counts=None, offsets=None, perm=None, dest=None, dispatched=None,
                 workspace=None, status=None, stream=None):
    """Stable expert-sorted dispatch.  Returns (offsets, perm, dest, dispatched)."""
    _check(hidden, "hidden", torch.bfloat16)
    T, d = hidden.shape
    _check(topk_idx, "topk_idx", torch.int32)
    K = topk_idx.shape[1]
    _check(topk_idx, "topk_idx", torch.int32, (T, K))
    dev = hidden.device
    offsets = _out(offsets, "offsets", (Nr + 1,), torch.int32, dev)
    perm = _out(perm, "perm", (T * K,), torch.int32, dev)
    dest = _out(dest, "dest", (T * K,), torch.int32, dev)
    dispatched = _out(dispatched, "dispatched", (T * K, d), torch.bfloat16, dev)
    need = dispatch_workspace_bytes(T, Nr)
    if workspace is None:
        workspace = torch.empty(max(need, 16), dtype=torch.uint8, device=dev)
    _check(workspace, "workspace", torch.uint8)
    if tile_counts is not None:
        _check(tile_counts, "tile_counts", torch.int32, ((T + 127) // 128, Nr))
    _call("moe_dispatch", _ptr(hidden), _ptr(topk_idx), _ptr(tile_counts), T, d, Nr, K, _ptr(offsets), _ptr(perm),
          _ptr(dest), _ptr(dispatched), _ptr(workspace), workspace.numel(), _ptr(status), _stream(stream))
    return offsets, perm, dest, dispatched


def moe_combine(expert_out, gates, dest, out=None, status=None, stream=None):
    """out[t] = sum_k gates[t,k] * expert_out[dest[t*K+k]] in fp32.  Returns out fp32 [T,d]."""
    _check(gates, "gates", torch.float32)
    T, K = gates.shape
    _check(expert_out, "expert_out", torch.bfloat16)
    d = expert_out.shape[1]
    _check(expert_out, "expert_out", torch.bfloat16, (T * K, d))
    _check(dest, "dest", torch.int32, (T * K,))
    out = _out(out, "out", (T, d), torch.float32, gates.device)
    _call("moe_combine", _ptr(expert_out), _ptr(gates), _ptr(dest), T, d, K, _ptr(out), _ptr(status),
          _stream(stream))
    return out


def read_internal_status(clear=True) -> int:
    v = ctypes.c_int32(0)
    _call("ebl_read_internal_status", ctypes.c_void_p(ctypes.addressof(v)), int(bool(clear)))
    return int(v.value)


def selftest_wait_timeout(status, limit_us=20000, stream=None):
    """Run the bounded-wait self-test; EBL_ST_TIMEOUT lands in status (int32 [1])."""
    _check(status, "status", torch.int32, (1,))
    _call("ebl_selftest_wait_timeout", _ptr(status), int(limit_us), _stream(stream))


def selftest_score_error(x, max_err=None, exact_out=None, stream=None):
    """Largest distance between the approximate score logits mode ranks with
    and the exact one over the fp32 values in x (device), and the error bound
    that ranking assumes.  Returns (max_err as a float, bound).  If exact_out
    (fp32, same size as x) is given it receives the exact scores."""
    _check(x, "x", torch.float32)
    if max_err is None:
        max_err = torch.empty(1, dtype=torch.float32, device=x.device)
    _check(max_err, "max_err", torch.float32, (1,))
    if exact_out is not None:
        _check(exact_out, "exact_out", torch.float32, tuple(x.shape))
    bound = ctypes.c_float(0.0)
    _call("ebl_selftest_score_error", _ptr(x), int(x.numel()), _ptr(max_err),
          ctypes.c_void_p(ctypes.addressof(bound)), _ptr(exact_out), _stream(stream))
    return float(max_err.item()), float(bound.value)


def check_finite(x, status, stream=None):
    """OR EBL_ST_NONFINITE into status (int32 [1]) if the fp32 or bf16 tensor x
    holds a NaN or an infinity."""
    _check(status, "status", torch.int32, (1,))
    if not isinstance(x, torch.Tensor) or x.dtype not in (torch.float32, torch.bfloat16):
        raise TypeError("x must be a float32 or bfloat16 tensor")
    _check(x, "x", x.dtype)
    name = "ebl_check_finite_f32" if x.dtype == torch.float32 else "ebl_check_finite_bf16"
    _call(name, _ptr(x), int(x.numel()), _ptr(status), _stream(stream))
