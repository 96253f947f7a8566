"""GPU parity: KV-group lists (list_mode 1: one list per (batch, KV head,
query block), the union of its q heads' selections, used by all of them).

The group lists must equal, bit for bit and flag for flag, the union of the
GPU's own per-head lists from the same inputs; against the oracle's group
lists they must agree on every row except rows whose per-head selection
already had an excused near-threshold disagreement.  Attention on group lists
is checked against the oracle run on the same lists, and at 100% density
against the per-head full lists.
"""

import numpy as np
import pytest
import torch

import block_sparse_long_rbs_b200 as rbs
from helpers import compare_selection, dense_masks, dev, lists_np, o_rows_close
from oracle import rbs_oracle as O
from workloads import WORKLOADS, make_inputs, make_mixture

pytestmark = pytest.mark.gpu


def _select_both(inp, block, rho, **kw):
    Q, K = inp["Q"], inp["K"]
    Cg, Rg = rbs.rbs_block_stats(dev(K), block)
    mk = lambda mode: rbs.SelectParams(block_q=block, block_k=block, rho_centroid=rho, rho_rescue=rho,
                                       list_mode=mode, **kw)
    per = rbs.rbs_select(dev(Q), Cg, Rg, mk(0))
    grp = rbs.rbs_select(dev(Q), Cg, Rg, mk(1))
    torch.cuda.synchronize()
    assert rbs.rbs_get_device_error() == 0
    return per, grp


def _check_group(inp, block, rho, **kw):
    Q, K = inp["Q"], inp["K"]
    B, L, Hq, _ = Q.shape
    Hkv = K.shape[2]
    G, nqb, nkb = Hq // Hkv, L // block, K.shape[1] // block
    per, grp = _select_both(inp, block, rho, **kw)
    assert grp.num_rows == B * Hkv * nqb
    # 1. group rows = union of the GPU's per-head rows (entries and flags)
    prp, pci, pfl = lists_np(per)
    grp_, gci, gfl = lists_np(grp)
    pflag = np.zeros((B * Hq * nqb, nkb), dtype=np.uint8)
    pflag[np.repeat(np.arange(prp.size - 1), np.diff(prp)), pci] = pfl
    want = np.bitwise_or.reduce(pflag.reshape(B, Hkv, G, nqb, nkb), axis=2).reshape(B * Hkv * nqb, nkb)
    got = np.zeros_like(want)
    got[np.repeat(np.arange(grp_.size - 1), np.diff(grp_)), gci] = gfl
    assert np.array_equal(got, want)
    for r in range(grp_.size - 1):
        assert np.all(np.diff(gci[grp_[r]:grp_[r + 1]]) > 0)
    # 2. per-head parity with the oracle, then group rows against the oracle's
    Co, Ro = O.block_stats(K, block)
    f32 = lambda v: float(np.float32(v))
    po = dict(block_q=block, block_k=block, rho_centroid=f32(rho), rho_rescue=f32(rho), **kw)
    ora = O.select_blocks(Q, Co, Ro, O.SelectParams(**po), keep_scores=True)
    rep = compare_selection(per, ora, Hq, nqb, nkb)
    ogrp = O.select_blocks(Q, Co, Ro, O.SelectParams(list_mode=1, **po))
    gu, _, _ = dense_masks(grp_, gci, gfl, nkb)
    ou, _, _ = dense_masks(ogrp["row_ptr"], ogrp["col_idx"], ogrp["flags"], nkb)
    hu, _, _ = dense_masks(prp, pci, pfl, nkb)
    hou, _, _ = dense_masks(ora["row_ptr"], ora["col_idx"], ora["flags"], nkb)
    head_rows_off = np.any(hu != hou, axis=1).reshape(B, Hkv, G, nqb).any(axis=2).reshape(-1)
    group_rows_off = np.any(gu != ou, axis=1)
    assert not np.any(group_rows_off & ~head_rows_off)
    rep["group_rows_off"] = int(group_rows_off.sum())
    rep["nnz_group"] = int(grp_[-1])
    return per, grp, rep


def test_group_lists_mixture_gqa(cuda_ok):
    inp = make_mixture(L=8192, Hq=8, Hkv=2, block=128, seed=401, batch=2)
    _, grp, rep = _check_group(inp, 128, 0.1, force_sink=1)
    print("group mixture", rep)


def test_group_lists_block64_ragged_group_noncausal_offset(cuda_ok):
    # G = 3 (R = 3 heads per selection CTA), 64-token blocks, non-causal with
    # a query-block offset
    inp = make_mixture(L=4096, Hq=6, Hkv=2, block=64, seed=402)
    _, _, rep = _check_group(inp, 64, 0.15, causal=0, q_block_offset=2)
    print("group g3", rep)


def test_group_lists_32k_config_and_attention(cuda_ok):
    w = WORKLOADS["gqa_rbs_32k"]
    inp = make_inputs(w)
    Co, Ro = O.block_stats(inp["K"], 128)
    rho, _ = O.bisect_rho(inp["Q"], Co, Ro, O.SelectParams(), w.density_target)
    per, grp, rep = _check_group(inp, 128, float(np.float32(rho)))
    print("group 32k", rep)
    Q, K, V = dev(inp["Q"]), dev(inp["K"]), dev(inp["V"])
    out, lse = rbs.bsa_prefill(Q, K, V, grp, 128, 128, return_lse=True)
    torch.cuda.synchronize()
    assert rbs.rbs_get_device_error() == 0
    Hq, nqb = inp["Q"].shape[2], inp["Q"].shape[1] // 128
    rng = np.random.default_rng(7)
    rows = sorted(set(rng.integers(0, Hq * nqb, 40).tolist()) | {nqb - 1, Hq * nqb - 1, 9 * nqb + 200})
    rp, ci, _ = lists_np(grp)
    Oo, Lo = O.masked_attention(inp["Q"], inp["K"], inp["V"], rp, ci, 128, 128, rows=rows)
    worst = o_rows_close(out, Oo, rows, Hq, nqb, 128)
    lg = lse.cpu().numpy()
    for row in rows:
        hq, i = divmod(row, nqb)
        sl = slice(i * 128, (i + 1) * 128)
        np.testing.assert_allclose(lg[0, hq, sl], Lo[0, hq, sl], atol=1e-3)
    print("group 32k attention worst", worst)


def test_group_full_lists_equal_per_head_full_lists_attention(cuda_ok):
    # causal-full lists built with heads = Hkv serve as group lists: the
    # attention output must be identical (bit for bit) to the per-head lists'
    inp = make_mixture(L=4096, Hq=8, Hkv=2, block=128, seed=403)
    Q, K, V = dev(inp["Q"]), dev(inp["K"]), dev(inp["V"])
    per = rbs.rbs_lists_causal_full(1, 8, 32)
    grp = rbs.rbs_lists_causal_full(1, 2, 32)
    a = rbs.bsa_prefill(Q, K, V, per, 128, 128)
    b = rbs.bsa_prefill(Q, K, V, grp, 128, 128)
    torch.cuda.synchronize()
    assert rbs.rbs_get_device_error() == 0
    assert torch.equal(a, b)


def test_group_lists_128k_sampled_attention(cuda_ok):
    w = WORKLOADS["gqa_rbs_128k"]
    inp = make_inputs(w)
    per, grp = _select_both(inp, 128, w.rho)
    assert grp.nnz() >= per.nnz() // 8
    Q, K, V = dev(inp["Q"]), dev(inp["K"]), dev(inp["V"])
    out = rbs.bsa_prefill(Q, K, V, grp, 128, 128)
    torch.cuda.synchronize()
    assert rbs.rbs_get_device_error() == 0
    Hq, nqb = 32, 1024
    rows = [nqb - 1, 8 * nqb + 777, 17 * nqb + 1023, 31 * nqb + 512, 5 * nqb + 3]
    rp, ci, _ = lists_np(grp)
    Oo, _ = O.masked_attention(inp["Q"], inp["K"], inp["V"], rp, ci, 128, 128, rows=rows)
    print("group 128k worst", o_rows_close(out, Oo, rows, Hq, nqb, 128), "nnz", grp.nnz(), per.nnz())
