"""moe_dispatch_static: the dispatch entry point that allocates nothing.

Some callers cannot call cudaMalloc to hand the library a dispatch workspace
(a plugin inside a framework that owns all device memory through its own pool,
or a runtime that forbids device allocation once it serves).  This entry point
keeps the scratch in a fixed library-owned device array instead.  The test
calls it through the C ABI twice in a row, on different inputs, and checks each
result against moe_dispatch with a caller workspace: offsets, perm, dest and
the gathered rows must be identical (dispatch is exact integer and copy work).
Each result is also checked on its own against the oracle's stable expert sort
(offsets, perm, dest) and against the rows of hidden it names.  One case passes
no status word, so device-side errors would go to the library's own word; it
must still give the same outputs.  A problem too large for the array is
refused.

The file name makes pytest collect it last.
"""
import ctypes

import numpy as np
import pytest
import torch

import expert_bias_load_b200 as ebl
import oracle
import synth

pytestmark = pytest.mark.gpu

STATIC_SCRATCH_BYTES = 4 << 20


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _topk_ids(T, K, Nr, seed):
    g = torch.Generator().manual_seed(seed)
    w = torch.rand(Nr, generator=g) ** 3 + 1e-3
    return torch.multinomial(w.expand(T, Nr), K, replacement=False, generator=g).to(torch.int32)


def _static_dispatch(hidden, idx, Nr, tile_counts, status, stream):
    T, d = hidden.shape
    K = idx.shape[1]
    dev = hidden.device
    offsets = torch.full((Nr + 1,), -9, dtype=torch.int32, device=dev)
    perm = torch.full((T * K,), -9, dtype=torch.int32, device=dev)
    dest = torch.full((T * K,), -9, dtype=torch.int32, device=dev)
    X = torch.zeros((T * K, d), dtype=torch.bfloat16, device=dev)
    rc = ebl.lib().moe_dispatch_static(_ptr(hidden), _ptr(idx), _ptr(tile_counts), T, d, Nr, K, _ptr(offsets),
                                       _ptr(perm), _ptr(dest), _ptr(X), _ptr(status),
                                       ctypes.c_void_p(stream.cuda_stream))
    return rc, offsets, perm, dest, X


@pytest.mark.parametrize("with_tiles,with_status", [(False, True), (True, True), (True, False)])
def test_static_dispatch_matches_workspace_dispatch_twice(cuda_device, with_tiles, with_status):
    dev = cuda_device
    stream = torch.cuda.current_stream()
    # two calls in a row on different problems; the second must not see the first's scratch
    for call, (T, d, Nr, K) in enumerate([(9000 + 7, 256, 256, 4), (3000 + 5, 64, 64, 8)]):
        idx = _topk_ids(T, K, Nr, seed=40 + call + 10 * with_tiles).to(dev)
        h = synth.hidden_normal(T, d, seed=50 + call, device=dev)
        tiles = None
        if with_tiles:
            tiles = torch.stack([torch.bincount(idx[j * 128:(j + 1) * 128].reshape(-1).long(), minlength=Nr)
                                 for j in range((T + 127) // 128)]).to(torch.int32)
        st = torch.zeros(1, dtype=torch.int32, device=dev) if with_status else None
        rc, offsets, perm, dest, X = _static_dispatch(h, idx, Nr, tiles, st, stream)
        assert rc == 0, ebl.lib().ebl_strerror(rc)
        ref = ebl.moe_dispatch(h, idx, Nr, tile_counts=tiles)
        torch.cuda.synchronize()
        if with_status:
            assert int(st.item()) == 0
        assert torch.equal(offsets, ref[0])
        assert torch.equal(perm, ref[1])
        assert torch.equal(dest, ref[2])
        assert torch.equal(X, ref[3])
        # independent of the other entry point: the oracle's stable expert sort
        o_off, o_perm, o_dest = oracle.dispatch(idx.cpu().numpy(), Nr)
        assert np.array_equal(offsets.cpu().numpy(), o_off)
        assert np.array_equal(perm.cpu().numpy(), o_perm)
        assert np.array_equal(dest.cpu().numpy(), o_dest)
        assert torch.equal(X, h[perm.long()])


def test_static_dispatch_rejects_oversized_problem(cuda_device):
    T, Nr, K, d = 508288 + 1, 256, 4, 8
    assert ebl.dispatch_workspace_bytes(T, Nr) > STATIC_SCRATCH_BYTES
    assert ebl.dispatch_workspace_bytes(T - 1, Nr) <= STATIC_SCRATCH_BYTES
    fake = ctypes.c_void_p(0x10000)
    rc = ebl.lib().moe_dispatch_static(fake, fake, None, T, d, Nr, K, fake, fake, fake, fake, None, None)
    assert rc == ebl.EBL_EINVAL
