"""rbs_select_noalloc: selection for callers that cannot give the library a
device workspace (a host framework that owns every device allocation, or a
serving loop where an allocation could stall other work).  Its scratch is a
buffer compiled into the library.  Called straight through the C ABI, its
lists must equal rbs_select's (same kernels, same inputs) on two calls in a
row, and a selection too large for the built-in buffer must be refused.

This file is collected last on purpose: it passes whether it runs alone in a
fresh process or after every other test (the buffer keeps the previous call's
contents, and nothing in it is read before being written)."""

import ctypes

import numpy as np
import pytest
import torch

import block_sparse_long_rbs_b200 as rbs
from block_sparse_long_rbs_b200 import _abi
from block_sparse_long_rbs_b200 import _stream, _t
from workloads import make_mixture, make_tiny

pytestmark = pytest.mark.gpu


def _dev(bits):
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).cuda()


def _lists_equal(a, b):
    assert torch.equal(a.row_ptr, b.row_ptr)
    n = a.nnz()
    assert n == b.nnz()
    assert torch.equal(a.col_idx[:n], b.col_idx[:n])
    assert torch.equal(a.flags[:n], b.flags[:n])


@pytest.mark.parametrize("case", ["tiny64", "mixture128"])
def test_noalloc_matches_workspace_select_twice(cuda_ok, case):
    if case == "tiny64":
        inp, blk, rho = make_tiny(L=4096), 64, 0.25
    else:
        inp, blk, rho = make_mixture(L=16384, Hq=16, Hkv=2, block=128, seed=401), 128, 0.07
    Q, K = _dev(inp["Q"]), _dev(inp["K"])
    B, L, Hq, _ = Q.shape
    Hkv = K.shape[2]
    nqb = nkb = L // blk
    p = rbs.SelectParams(block_q=blk, block_k=blk, rho_centroid=rho, rho_rescue=rho)
    C, R = rbs.rbs_block_stats(K, blk)
    ref = rbs.rbs_select(Q, C, R, p)
    L_ = _abi.lib()
    cap = rbs.rbs_select_capacity(B, Hq, nqb, nkb, p)
    pc = p.c()
    tQ = _t(Q, "Q")
    for call in range(2):
        out = rbs.BlockLists.empty(B * Hq * nqb, cap, Q.device)
        out.row_ptr.fill_(-7)
        out.col_idx.fill_(-7)
        lc = out.c()
        st = L_.rbs_select_noalloc(ctypes.byref(tQ), C.data_ptr(), R.data_ptr(), Hkv, nkb, ctypes.byref(pc),
                                   ctypes.byref(lc), None, _stream())
        assert st == 0, L_.rbs_last_error()
        torch.cuda.synchronize()
        assert rbs.rbs_get_device_error() == 0
        _lists_equal(out, ref)


def test_noalloc_runs_the_fused_kernel_when_only_the_masks_fit(cuda_ok):
    # 131072 tokens, 8 q heads over 1 KV head: the full workspace (with the
    # tensor-core path's score matrix) is larger than the built-in buffer, the
    # masks and counts fit, so the fused CUDA-core kernel runs.  rbs_select
    # with a workspace one byte short of the full size takes the same path.
    inp = make_mixture(L=131072, Hq=8, Hkv=1, block=128, seed=402)
    Q, K = _dev(inp["Q"]), _dev(inp["K"])
    B, L, Hq, _ = Q.shape
    nqb = nkb = L // 128
    p = rbs.SelectParams(block_q=128, block_k=128, rho_centroid=0.05, rho_rescue=0.05)
    full = rbs.rbs_select_workspace_bytes(B, Hq, nqb, 1, nkb, p)
    assert full > _abi.NOALLOC_SCRATCH_BYTES
    C, R = rbs.rbs_block_stats(K, 128)
    ws = torch.empty(full - 1, dtype=torch.uint8, device="cuda")
    ref = rbs.rbs_select(Q, C, R, p, workspace=ws)
    L_ = _abi.lib()
    cap = rbs.rbs_select_capacity(B, Hq, nqb, nkb, p)
    pc, tQ = p.c(), _t(Q, "Q")
    for call in range(2):
        out = rbs.BlockLists.empty(B * Hq * nqb, cap, Q.device)
        out.row_ptr.fill_(-7)
        lc = out.c()
        st = L_.rbs_select_noalloc(ctypes.byref(tQ), C.data_ptr(), R.data_ptr(), 1, nkb, ctypes.byref(pc),
                                   ctypes.byref(lc), None, _stream())
        assert st == 0, L_.rbs_last_error()
        torch.cuda.synchronize()
        assert rbs.rbs_get_device_error() == 0
        _lists_equal(out, ref)


def test_noalloc_refuses_selection_larger_than_its_buffer(cuda_ok):
    # Every data pointer is null: whatever the size rule, host validation
    # refuses the call before a launch.  A selection too large for the
    # built-in buffer is refused for its size (the library reports how many
    # bytes it needs); one that fits is refused for the null pointers.
    import re
    L_ = _abi.lib()
    p = rbs.SelectParams()
    pc = p.c()
    big = _abi.Bf16Tensor(None, 1, 262144, 64, 128, 262144 * 64 * 128, 64 * 128, 128)
    lc = _abi.BlockListsC(None, None, None, 1 << 30, 64 * 2048)
    st = L_.rbs_select_noalloc(ctypes.byref(big), None, None, 8, 2048, ctypes.byref(pc), ctypes.byref(lc), None, None)
    assert st == 3
    msg = L_.rbs_last_error().decode()
    assert "built-in buffer" in msg
    need = int(re.search(r"needs (\d+) bytes", msg).group(1))
    assert need > _abi.NOALLOC_SCRATCH_BYTES
    small = _abi.Bf16Tensor(None, 1, 4096, 2, 128, 4096 * 2 * 128, 2 * 128, 128)
    lc = _abi.BlockListsC(None, None, None, 1 << 20, 2 * 32)
    st = L_.rbs_select_noalloc(ctypes.byref(small), None, None, 1, 32, ctypes.byref(pc), ctypes.byref(lc), None, None)
    assert st == 1
