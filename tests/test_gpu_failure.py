"""Failure handling and the software exponential on the GPU.

A pipeline wait that runs out must end the attention kernel cleanly: the
producer of key tiles is told to stop early (a testing hook), so the waits
for the missing tiles run out after 1 ms; the kernel must record
RBS_DEVERR_TIMEOUT and return, and the next normal call must be correct (no
copy or MMA was left in flight, tensor memory was freed).  No GPU fault is
involved: the missing tiles are simply never requested.

The attention kernel's FMA-pipe exponential (a degree-3 Remez fit after
Cody-Waite range reduction) is checked against exp2 in float64 within its
fitted relative error (4.315e-4 by the Remez fit, plus fp32 rounding)."""

import ctypes

import numpy as np
import pytest
import torch

import block_sparse_long_rbs_b200 as rbs
from block_sparse_long_rbs_b200 import _abi, _stream, _t
from helpers import dev, lists_np, o_rows_close
from oracle import rbs_oracle as O
from workloads import make_mixture

pytestmark = pytest.mark.gpu


def _inputs():
    inp = make_mixture(L=4096, Hq=8, Hkv=2, block=128, seed=601)
    p = rbs.SelectParams(block_q=128, block_k=128, rho_centroid=0.2, rho_rescue=0.2)
    Q, K, V = dev(inp["Q"]), dev(inp["K"]), dev(inp["V"])
    C, R = rbs.rbs_block_stats(K, 128)
    return inp, Q, K, V, rbs.rbs_select(Q, C, R, p)


def test_wait_that_runs_out_returns_timeout_and_the_next_call_is_correct(cuda_ok):
    inp, Q, K, V, lists = _inputs()
    L_ = _abi.lib()
    out = torch.zeros_like(Q)
    lc = lists.c()
    tQ, tK, tV, tO = _t(Q, "Q"), _t(K, "K"), _t(V, "V"), _t(out, "O")
    assert rbs.rbs_get_device_error() == 0
    st = L_.rbs_testing_bsa_prefill_stalled(ctypes.byref(tQ), ctypes.byref(tK), ctypes.byref(tV), ctypes.byref(lc),
                                            128, 128, 1_000_000, 5, ctypes.byref(tO), _stream())
    assert st == 0, L_.rbs_last_error()
    torch.cuda.synchronize()
    code = rbs.rbs_get_device_error()
    assert code & rbs.DEVERR_TIMEOUT, code
    # the context is usable and the kernel's state was released: a normal
    # call right after is correct
    good = rbs.bsa_prefill(Q, K, V, lists, 128, 128)
    torch.cuda.synchronize()
    assert rbs.rbs_get_device_error() == 0
    rp, ci, _ = lists_np(lists)
    rows = list(range(0, rp.size - 1, 7))
    Oo, _ = O.masked_attention(inp["Q"], inp["K"], inp["V"], rp, ci, 128, 128, rows=rows)
    o_rows_close(good, Oo, rows, 8, 32, 128)


def test_stall_hook_rejects_out_of_range_limits(cuda_ok):
    inp, Q, K, V, lists = _inputs()
    L_ = _abi.lib()
    out = torch.zeros_like(Q)
    lc = lists.c()
    tQ, tK, tV, tO = _t(Q, "Q"), _t(K, "K"), _t(V, "V"), _t(out, "O")
    for wait_ns, stall in ((10, 5), (3_000_000_000, 5), (1_000_000, -1)):
        st = L_.rbs_testing_bsa_prefill_stalled(ctypes.byref(tQ), ctypes.byref(tK), ctypes.byref(tV),
                                                ctypes.byref(lc), 128, 128, wait_ns, stall, ctypes.byref(tO), _stream())
        assert st == 1


def test_software_exp2_within_its_fitted_bound(cuda_ok):
    # a dense grid over the range the softmax uses, the reduction's edges
    # (half-integers), and values below the clamp
    grid = np.linspace(-127.0, 8.0, 2_000_001, dtype=np.float32)
    edges = (np.arange(-126, 8, dtype=np.float32)[:, None] + np.array([-0.5, 0.5, 0.0], dtype=np.float32)).ravel()
    low = np.array([-127.0, -150.0, -1e30, -np.inf], dtype=np.float32)
    x = np.concatenate([grid, edges, low]).astype(np.float32)
    xd = torch.from_numpy(x).cuda()
    y = torch.empty_like(xd)
    st = _abi.lib().rbs_testing_exp2(ctypes.c_void_p(xd.data_ptr()), ctypes.c_void_p(y.data_ptr()), x.size, _stream())
    assert st == 0
    torch.cuda.synchronize()
    got = y.cpu().numpy().astype(np.float64)
    ref = np.exp2(x.astype(np.float64))
    normal = x >= -126.0
    rel = np.abs(got[normal] - ref[normal]) / ref[normal]
    # the fit's maximum relative error (4.315e-4, csrc/exp2_poly_fit.py) plus
    # the fp32 rounding of the evaluation
    assert rel.max() <= 4.315e-4 + 5e-7, rel.max()
    # below the normal range the result is only close in absolute terms
    assert np.all(np.abs(got[~normal] - ref[~normal]) <= 2.0 ** -126)
    assert np.all(got[x <= -127.0] == 0.0)
    assert np.all(np.isfinite(got))
