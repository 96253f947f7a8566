"""GPU parity: per-token-max query scoring (query_pool 1, scores on the
tensor core) against the oracle's lists, branch by branch, with the same
near-threshold rule as the mean-query selection."""

import numpy as np
import pytest
import torch

import block_sparse_long_rbs_b200 as rbs
from helpers import TOL_NEAR_TAU, compare_selection, dense_masks, dev, lists_np
from oracle import rbs_oracle as O
from workloads import WORKLOADS, make_inputs, make_mixture, make_tiny

pytestmark = pytest.mark.gpu


def _run(inp, block, rho_c, rho_r, **kw):
    Q, K = inp["Q"], inp["K"]
    B, L, Hq, _ = Q.shape
    nqb, nkb = -(-L // block), -(-K.shape[1] // block)
    p = rbs.SelectParams(block_q=block, block_k=block, rho_centroid=rho_c, rho_rescue=rho_r, query_pool=1, **kw)
    Cg, Rg = rbs.rbs_block_stats(dev(K), block)
    lists = rbs.rbs_select(dev(Q), Cg, Rg, p)
    torch.cuda.synchronize()
    assert rbs.rbs_get_device_error() == 0
    Co, Ro = O.block_stats(K, block)
    f32 = lambda v: float(np.float32(v)) if isinstance(v, float) else v
    po = O.SelectParams(block_q=block, block_k=block, rho_centroid=f32(rho_c), rho_rescue=f32(rho_r), query_pool=1,
                        **{k: f32(v) for k, v in kw.items()})
    ora = O.select_blocks(Q, Co, Ro, po, keep_scores=True)
    return compare_selection(lists, ora, Hq, nqb, nkb, exact_k=kw.get("threshold_mode", 0) == 0)


def test_tokmax_tiny_config(cuda_ok):
    w = WORKLOADS["tiny_rbs_4k"]
    rep = _run(make_inputs(w), 64, w.rho, w.rho)
    print("tokmax tiny", rep)


@pytest.mark.parametrize("beta_mode,const", [(0, 1.0), (1, 0.0)])
def test_tokmax_mixture_gqa(cuda_ok, beta_mode, const):
    inp = make_mixture(L=8192, Hq=8, Hkv=2, block=128, seed=701, batch=2)
    rep = _run(inp, 128, 0.1, 0.1, beta_mode=beta_mode, beta_const=const, force_sink=1)
    print("tokmax mixture", beta_mode, rep)


def test_tokmax_ragged_block64_noncausal_offset(cuda_ok):
    inp = make_mixture(L=4096 + 64, Hq=6, Hkv=2, block=64, seed=702)
    inp = {k: (v[:, :4096 + 37] if k in ("Q", "K", "V") else v) for k, v in inp.items()}
    rep = _run(inp, 64, 0.15, 0.2, causal=0, q_block_offset=3)
    print("tokmax ragged", rep)


def test_tokmax_max_relative(cuda_ok):
    inp = make_mixture(L=8192, Hq=4, Hkv=1, block=128, seed=703)
    rep = _run(inp, 128, 0.1, 0.1, threshold_mode=1, delta_centroid=4.0, delta_rescue=4.0)
    print("tokmax max-relative", rep)


def test_tokmax_32k_config(cuda_ok):
    w = WORKLOADS["gqa_rbs_32k"]
    rep = _run(make_inputs(w), 128, 0.05, 0.05)
    print("tokmax 32k", rep)


def test_tokmax_128k_sampled_rows(cuda_ok):
    # the oracle scores a few rows of the 128K prompt; each GPU branch must
    # agree on them up to the near-threshold rule
    w = WORKLOADS["gqa_rbs_128k"]
    inp = make_inputs(w)
    p = rbs.SelectParams(rho_centroid=w.rho, rho_rescue=w.rho, query_pool=1)
    Cg, Rg = rbs.rbs_block_stats(dev(inp["K"]), 128)
    lists = rbs.rbs_select(dev(inp["Q"]), Cg, Rg, p)
    torch.cuda.synchronize()
    assert rbs.rbs_get_device_error() == 0
    rp, ci, fl = lists_np(lists)
    nqb = nkb = 1024
    _, gc, gr = dense_masks(rp, ci, fl, nkb)
    C, R = O.block_stats(inp["K"], 128)
    po = O.SelectParams(rho_centroid=float(np.float32(w.rho)), rho_rescue=float(np.float32(w.rho)), query_pool=1)
    beta, _ = O.rescue_beta(R, po)
    excused = 0
    for hq, i in ((0, 1023), (5, 700), (13, 512), (22, 301), (31, 1000), (9, 64)):
        kvh = hq // 8
        q = inp["Q"][0, i * 128:(i + 1) * 128, hq][None]
        s_c, s_r = O.token_max_scores(q[0], C[0, kvh], R[0, kvh], beta[0, kvh], 128)
        n = i + 1
        row = hq * nqb + i
        for bi, (s, gm, rho) in enumerate(((s_c[0, :n], gc, po.rho_centroid), (s_r[0, :n], gr, po.rho_rescue))):
            k = O.keep_count(rho, n)
            top = O.top_k_desc(s, k)
            want = np.zeros(n, dtype=bool)
            want[top] = True
            tau = s[top[-1]]
            assert gm[row, :n].sum() == k
            for j in np.nonzero(gm[row, :n] != want)[0]:
                assert abs(s[j] - tau) <= TOL_NEAR_TAU * max(1.0, abs(tau)), (hq, i, bi, j)
                excused += 1
    print("tokmax 128k sampled rows, excused", excused, "nnz", int(rp[-1]))


@pytest.mark.parametrize("case", ["mixture", "max_relative", "32k"])
def test_tokmax_both_topk_paths(cuda_ok, case):
    # with the full workspace the token-max kernel stores both branches' keys
    # and the separate top-k kernel selects from them; one byte short, two
    # warps of the token-max kernel select in place.  Both read the same keys
    # with the same selection code, so their lists must be identical, and
    # both must match the oracle.
    kw = {}
    if case == "mixture":
        inp, block, rho = make_mixture(L=8192, Hq=8, Hkv=2, block=128, seed=704, batch=2), 128, 0.1
    elif case == "max_relative":
        inp, block, rho = make_mixture(L=8192, Hq=4, Hkv=1, block=128, seed=705), 128, 0.1
        kw = dict(threshold_mode=1, delta_centroid=4.0, delta_rescue=4.0)
    else:
        inp, block, rho = make_inputs(WORKLOADS["gqa_rbs_32k"]), 128, 0.05
    Q, K = inp["Q"], inp["K"]
    B, L, Hq, _ = Q.shape
    Hkv, nqb, nkb = K.shape[2], L // block, K.shape[1] // block
    p = rbs.SelectParams(block_q=block, block_k=block, rho_centroid=rho, rho_rescue=rho, query_pool=1, **kw)
    Cg, Rg = rbs.rbs_block_stats(dev(K), block)
    full = rbs.rbs_select_workspace_bytes(B, Hq, nqb, Hkv, nkb, p)
    ws = torch.empty(full + 255, dtype=torch.uint8, device="cuda")
    off = (-ws.data_ptr()) % 256
    lists_sep = rbs.rbs_select(dev(Q), Cg, Rg, p, workspace=ws[off:off + full])
    lists_in = rbs.rbs_select(dev(Q), Cg, Rg, p, workspace=ws[off:off + full - 1])
    torch.cuda.synchronize()
    assert rbs.rbs_get_device_error() == 0
    for a, b in zip(lists_np(lists_sep), lists_np(lists_in)):
        np.testing.assert_array_equal(a, b)
    Co, Ro = O.block_stats(K, block)
    f32 = lambda v: float(np.float32(v)) if isinstance(v, float) else v
    po = O.SelectParams(block_q=block, block_k=block, rho_centroid=f32(rho), rho_rescue=f32(rho), query_pool=1,
                        **{k: f32(v) for k, v in kw.items()})
    ora = O.select_blocks(Q, Co, Ro, po, keep_scores=True)
    rep = compare_selection(lists_sep, ora, Hq, nqb, nkb, exact_k=kw.get("threshold_mode", 0) == 0)
    print("tokmax both top-k paths", case, rep)


def test_tokmax_2048_key_blocks_sampled_rows(cuda_ok):
    # 262144 tokens in 128-token blocks: 2048 key blocks, the most the
    # per-token kernel takes (its 64-slot instantiation).  Sampled rows of
    # each branch against the oracle's scores, and the separate and in-place
    # top-k giving identical lists.
    inp = make_mixture(L=262144, Hq=2, Hkv=1, block=128, seed=706)
    Q, K = inp["Q"], inp["K"]
    B, L, Hq, _ = Q.shape
    nqb = nkb = L // 128
    rho = 0.02
    p = rbs.SelectParams(rho_centroid=rho, rho_rescue=rho, query_pool=1)
    Qd = dev(Q)
    Cg, Rg = rbs.rbs_block_stats(dev(K), 128)
    full = rbs.rbs_select_workspace_bytes(B, Hq, nqb, 1, nkb, p)
    ws = torch.empty(full + 255, dtype=torch.uint8, device="cuda")
    off = (-ws.data_ptr()) % 256
    lists = rbs.rbs_select(Qd, Cg, Rg, p, workspace=ws[off:off + full])
    lists_in = rbs.rbs_select(Qd, Cg, Rg, p, workspace=ws[off:off + full - 1])
    torch.cuda.synchronize()
    assert rbs.rbs_get_device_error() == 0
    for a, b in zip(lists_np(lists), lists_np(lists_in)):
        np.testing.assert_array_equal(a, b)
    rp, ci, fl = lists_np(lists)
    _, gc, gr = dense_masks(rp, ci, fl, nkb)
    C, R = O.block_stats(K, 128)
    po = O.SelectParams(rho_centroid=float(np.float32(rho)), rho_rescue=float(np.float32(rho)), query_pool=1)
    beta, _ = O.rescue_beta(R, po)
    excused = 0
    for hq, i in ((0, 2047), (1, 2047), (0, 1500), (1, 1100), (0, 1030), (1, 700)):
        q = Q[0, i * 128:(i + 1) * 128, hq][None]
        s_c, s_r = O.token_max_scores(q[0], C[0, 0], R[0, 0], beta[0, 0], 128)
        n = i + 1
        row = hq * nqb + i
        for bi, (s, gm, r) in enumerate(((s_c[0, :n], gc, po.rho_centroid), (s_r[0, :n], gr, po.rho_rescue))):
            k = O.keep_count(r, n)
            top = O.top_k_desc(s, k)
            want = np.zeros(n, dtype=bool)
            want[top] = True
            tau = s[top[-1]]
            assert gm[row, :n].sum() == k
            for j in np.nonzero(gm[row, :n] != want)[0]:
                assert abs(s[j] - tau) <= TOL_NEAR_TAU * max(1.0, abs(tau)), (hq, i, bi, j)
                excused += 1
    print("tokmax 2048 key blocks, sampled rows, excused", excused, "nnz", int(rp[-1]))
