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


def test_noalloc_refuses_selection_larger_than_its_buffer(cuda_ok):
    # 262144 tokens x 64 q heads at 128-token blocks needs far more than the buffer;
    # the call must refuse before touching the (never dereferenced) pointers.
    L_ = _abi.lib()
    p = rbs.SelectParams()
    need = rbs.rbs_select_workspace_bytes(1, 64, 2048, 8, 2048, p)
    assert need > _abi.NOALLOC_SCRATCH_BYTES
    fake = _abi.Bf16Tensor(0x10000, 1, 262144, 64, 128, 262144 * 64 * 128, 64 * 128, 128)
    lc = _abi.BlockListsC(0x20000, 0x30000, None, 1 << 30, 64 * 2048)
    st = L_.rbs_select_noalloc(ctypes.byref(fake), 0x40000, 0x50000, 8, 2048, ctypes.byref(p.c()), ctypes.byref(lc),
                               None, None)
    assert st == 3
    assert b"built-in buffer" in L_.rbs_last_error()
