"""C-ABI checks that need no GPU: the library loads, exports every function
include/ebl.h declares, and rejects bad arguments before touching CUDA."""
import ctypes
import os
import re

import pytest

import expert_bias_load_b200 as ebl

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "ebl.h")

EINVAL, EUNSUPPORTED = -1, -2
FAKE = ctypes.c_void_p(0x10000)   # an aligned, non-null address that is never dereferenced


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    names = re.findall(r"^\s*(?:const\s+)?[A-Za-z_][A-Za-z_0-9]*\s*\*?\s*([a-z_][a-z_0-9]*)\s*\(", text, re.M)
    return sorted(set(names))


@pytest.fixture(scope="module")
def lib():
    from expert_bias_load_b200 import build
    build.build()
    return ebl.lib()


def test_header_functions_are_exported_and_bound(lib):
    names = declared_functions()
    assert len(names) >= 12
    for n in names:
        assert hasattr(lib, n), n
        assert n in ebl.SIGNATURES, "binding lacks %s" % n
    assert set(ebl.SIGNATURES) == set(names)


def test_host_only_queries(lib):
    assert lib.ebl_version() >= 10000
    assert lib.ebl_tile_tokens() == 128
    assert lib.ebl_strerror(0) == b"ok"
    for code in (-1, -2, -3, -4, -99):
        assert lib.ebl_strerror(code)
    # workspace: (tiles + segments of 32 tiles) * N_r int32
    assert lib.ebl_dispatch_workspace_bytes(1048576, 256) == (8192 + 256) * 256 * 4
    assert lib.ebl_dispatch_workspace_bytes(1, 64) == 2 * 64 * 4
    assert lib.ebl_dispatch_workspace_bytes(-1, 64) == 0


def _router(lib, T=256, d=256, Nr=64, K=4, ptrs=None):
    p = ptrs or {}
    g = lambda k: p.get(k, FAKE)
    return lib.router_forward(g("h"), g("w"), g("b"), T, d, Nr, K, g("i"), g("g"), g("c"), None, None, None)


def test_router_forward_rejects_bad_arguments(lib):
    assert _router(lib, K=0) == EINVAL
    assert _router(lib, K=9) == EINVAL
    assert _router(lib, Nr=4, K=5) == EINVAL
    assert _router(lib, Nr=300) == EINVAL
    assert _router(lib, d=100) == EINVAL
    assert _router(lib, d=0) == EINVAL
    assert _router(lib, T=-1) == EINVAL
    assert _router(lib, Nr=48) == EUNSUPPORTED      # GEMM mode needs N_r % 32 == 0
    assert _router(lib, ptrs={"h": None}) == EINVAL
    assert _router(lib, ptrs={"c": None}) == EINVAL
    assert _router(lib, ptrs={"h": ctypes.c_void_p(0x10008)}) == EINVAL   # not 16-byte aligned
    assert _router(lib, T=0) == 0                    # empty batch: nothing to do
    # with no tokens the token-sized buffers may be NULL (empty tensors have no storage)
    assert _router(lib, T=0, ptrs={"h": None, "i": None, "g": None}) == 0
    assert _router(lib, T=0, ptrs={"w": None}) == EINVAL
    assert _router(lib, T=1, ptrs={"i": None}) == EINVAL
    assert lib.router_forward_logits(None, FAKE, 0, 8, 2, None, None, FAKE, None, None, None) == 0
    assert lib.router_forward_logits(None, FAKE, 1, 8, 2, FAKE, FAKE, FAKE, None, None, None) == EINVAL
    assert lib.moe_combine(None, None, None, 0, 64, 2, None, None, None) == 0
    assert lib.moe_combine(None, FAKE, FAKE, 1, 64, 2, FAKE, None, None) == EINVAL


def test_other_entry_points_reject_bad_arguments(lib):
    assert lib.router_forward_logits(FAKE, FAKE, 10, 8, 9, FAKE, FAKE, FAKE, None, None, None) == EINVAL
    assert lib.router_forward_logits(None, FAKE, 10, 8, 2, FAKE, FAKE, FAKE, None, None, None) == EINVAL
    assert lib.router_forward_logits(FAKE, FAKE, 0, 8, 2, FAKE, FAKE, FAKE, None, None, None) == 0
    assert lib.smebu_step(FAKE, FAKE, FAKE, 0, 5e-4, 0.5, 2.0, 0, None, None, None) == EINVAL
    assert lib.smebu_step(FAKE, FAKE, FAKE, 257, 5e-4, 0.5, 2.0, 0, None, None, None) == EINVAL
    assert lib.smebu_step(None, FAKE, FAKE, 8, 5e-4, 0.5, 2.0, 0, None, None, None) == EINVAL
    assert lib.smebu_step_layers(FAKE, FAKE, FAKE, 0, 8, 5e-4, 0.5, 2.0, 0, 0, None, None, None) == EINVAL
    assert lib.sign_update_step(FAKE, None, 8, 1e-3, 0, None, None, None) == EINVAL
    ws = lib.ebl_dispatch_workspace_bytes(100, 16)
    args = lambda T=100, d=64, Nr=16, K=2, wsb=ws: (FAKE, FAKE, None, T, d, Nr, K, FAKE, FAKE, FAKE, FAKE, FAKE,
                                                   wsb, None, None)
    assert lib.moe_dispatch(*args(wsb=ws - 4)) == EINVAL
    assert lib.moe_dispatch(*args(d=12)) == EINVAL
    assert lib.moe_dispatch(*args(K=3, Nr=2)) == EINVAL
    assert lib.moe_combine(FAKE, FAKE, FAKE, 100, 12, 2, FAKE, None, None) == EINVAL
    assert lib.moe_combine(FAKE, FAKE, FAKE, 100, 64, 9, FAKE, None, None) == EINVAL
    assert lib.moe_combine(FAKE, FAKE, FAKE, 0, 64, 2, FAKE, None, None) == 0
    assert lib.ebl_read_internal_status(None, 0) == EINVAL
    assert lib.ebl_selftest_score_error(FAKE, -1, FAKE, None, None, None) == EINVAL
    assert lib.ebl_selftest_score_error(FAKE, 10, None, None, None, None) == EINVAL
    assert lib.ebl_selftest_score_error(None, 10, FAKE, None, None, None) == EINVAL
    assert lib.ebl_selftest_score_error(FAKE, 10, FAKE, None, ctypes.c_void_p(0x10002), None) == EINVAL
    assert lib.ebl_check_finite_f32(FAKE, -1, FAKE, None) == EINVAL
    assert lib.ebl_check_finite_f32(FAKE, 10, None, None) == EINVAL
    assert lib.ebl_check_finite_f32(ctypes.c_void_p(0x10002), 10, FAKE, None) == EINVAL   # not 4-byte aligned
    assert lib.ebl_check_finite_bf16(ctypes.c_void_p(0x10001), 10, FAKE, None) == EINVAL  # not 2-byte aligned
    assert lib.ebl_check_finite_bf16(None, 0, FAKE, None) == 0                              # empty: nothing to do
    # sequence-wise balance: the option needs tile_counts and tile_psum; the loss
    # wants seq_len a positive multiple of 128 that divides T
    bal = lambda T=256, tc=FAKE, tp=FAKE: lib.router_forward_balance(FAKE, FAKE, FAKE, T, 256, 64, 4, FAKE, FAKE,
                                                                     FAKE, tc, tp, None, None, None)
    assert bal(tc=None) == EINVAL
    assert bal(tp=None) == EINVAL
    assert bal(tp=ctypes.c_void_p(0x10002)) == EINVAL
    assert bal(T=0, tc=None, tp=None) == 0
    sb = lambda T=1024, Nr=64, K=4, S=256, a=5e-5, ls=FAKE, l=FAKE: lib.seq_balance_loss(FAKE, FAKE, T, Nr, K, S, a,
                                                                                         ls, l, None)
    assert sb(S=100) == EINVAL
    assert sb(S=0) == EINVAL
    assert sb(T=1280, S=512) == EINVAL
    assert sb(K=9) == EINVAL
    assert sb(Nr=0) == EINVAL
    assert sb(a=float("nan")) == EINVAL
    assert sb(a=float("inf")) == EINVAL
    assert sb(ls=None) == EINVAL
    assert sb(l=ctypes.c_void_p(0x10004)) == EINVAL                                       # not 8-byte aligned
    assert sb(T=0, ls=None, l=None) == 0                                                  # no tokens: nothing to do
    assert lib.balance_stats_logits(FAKE, 100, 0, FAKE, None) == EINVAL
    assert lib.balance_stats_logits(FAKE, 100, 257, FAKE, None) == EINVAL
    assert lib.balance_stats_logits(None, 100, 8, FAKE, None) == EINVAL
    assert lib.balance_stats_logits(FAKE, 100, 8, None, None) == EINVAL
    assert lib.balance_stats_logits(ctypes.c_void_p(0x10002), 100, 8, FAKE, None) == EINVAL
    assert lib.balance_stats_logits(None, 0, 8, None, None) == 0


def test_binding_has_no_cpu_fallback():
    import torch
    h = torch.zeros(4, 64, dtype=torch.bfloat16)
    with pytest.raises(ValueError):
        ebl.router_forward(h, torch.zeros(32, 64, dtype=torch.bfloat16), torch.zeros(32), 2,
                           torch.zeros(32, dtype=torch.int32))
    # the balance entry points refuse host tensors too
    tc = torch.zeros(1, 32, dtype=torch.int32)
    tp = torch.zeros(1, 32)
    with pytest.raises(ValueError):
        ebl.router_forward_balance(h, torch.zeros(32, 64, dtype=torch.bfloat16), torch.zeros(32), 2,
                                   torch.zeros(32, dtype=torch.int32), tc, tp)
    with pytest.raises(ValueError):
        ebl.balance_stats_logits(torch.zeros(4, 32))
    with pytest.raises(ValueError):
        ebl.seq_balance_loss(tc, tp, 128, 2, 128)
