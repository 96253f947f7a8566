"""GPU parity at sequence lengths that are not block multiples (the last
query and key blocks are shorter): statistics and pooling of the short
blocks, selection over ceil(L / block) blocks, attention that never reads a
key past Lk and writes no row past Lq, with the same tolerances as the
block-multiple tests.  Inputs are the seeded generators' tensors cut to L."""

import numpy as np
import pytest
import torch

import block_sparse_long_rbs_b200 as rbs
from helpers import TOL_STATS_REL, compare_selection, dev, lists_np, o_rows_close
from oracle import rbs_oracle as O
from workloads import make_mixture, make_tiny

pytestmark = pytest.mark.gpu


def _cut(inp, L):
    return {k: (v[:, :L] if k in ("Q", "K", "V") else v) for k, v in inp.items()}


def _mixture(L, block, Hq, Hkv, seed):
    up = -(-L // block) * block
    return _cut(make_mixture(L=up, Hq=Hq, Hkv=Hkv, block=block, seed=seed), L)


@pytest.mark.parametrize("block,L", [(64, 4096 + 77), (128, 8192 + 100), (128, 8192 + 1)])
def test_ragged_stats_and_pooling(cuda_ok, block, L):
    inp = _mixture(L, block, 4, 2, 601)
    Cg, Rg = rbs.rbs_block_stats(dev(inp["K"]), block)
    qg, ng = rbs.rbs_pool_queries(dev(inp["Q"]), block)
    torch.cuda.synchronize()
    Co, Ro = O.block_stats(inp["K"], block)
    qo, no = O.pooled_queries(inp["Q"], block)
    assert Cg.shape == Co.shape and qg.shape == qo.shape
    Cg, Rg, qg, ng = (x.cpu().numpy().astype(np.float64) for x in (Cg, Rg, qg, ng))
    rel = np.linalg.norm(Cg - Co, axis=-1) / np.maximum(np.linalg.norm(Co, axis=-1), 1e-6)
    assert rel.max() <= TOL_STATS_REL
    assert (np.abs(Rg - Ro) / np.maximum(Ro, 1e-6)).max() <= TOL_STATS_REL
    relq = np.linalg.norm(qg - qo, axis=-1) / np.maximum(np.linalg.norm(qo, axis=-1), 1e-6)
    assert relq.max() <= TOL_STATS_REL
    np.testing.assert_allclose(ng, no, rtol=TOL_STATS_REL)


@pytest.mark.parametrize("block,L,Hq,Hkv,rho", [(64, 4096 + 77, 2, 1, 0.25), (128, 8192 + 100, 8, 2, 0.1)])
def test_ragged_select_and_attention(cuda_ok, block, L, Hq, Hkv, rho):
    inp = _mixture(L, block, Hq, Hkv, 602)
    nqb = nkb = -(-L // block)
    p = rbs.SelectParams(block_q=block, block_k=block, rho_centroid=rho, rho_rescue=rho)
    Cg, Rg = rbs.rbs_block_stats(dev(inp["K"]), block)
    lists = rbs.rbs_select(dev(inp["Q"]), Cg, Rg, p)
    Q, K, V = dev(inp["Q"]), dev(inp["K"]), dev(inp["V"])
    out, lse = rbs.bsa_prefill(Q, K, V, lists, block, block, return_lse=True)
    torch.cuda.synchronize()
    assert rbs.rbs_get_device_error() == 0
    Co, Ro = O.block_stats(inp["K"], block)
    po = O.SelectParams(block_q=block, block_k=block, rho_centroid=float(np.float32(rho)),
                        rho_rescue=float(np.float32(rho)))
    rep = compare_selection(lists, O.select_blocks(inp["Q"], Co, Ro, po, keep_scores=True), Hq, nqb, nkb)
    rp, ci, _ = lists_np(lists)
    rows = sorted({h * nqb + i for h in range(Hq) for i in (0, 1, nqb // 2, nqb - 2, nqb - 1)})
    Oo, Lo = O.masked_attention(inp["Q"], inp["K"], inp["V"], rp, ci, block, block, rows=rows)
    worst = o_rows_close(out, Oo, rows, Hq, nqb, block)
    lg = lse.cpu().numpy()
    for row in rows:
        h, i = divmod(row, nqb)
        sl = slice(i * block, min((i + 1) * block, L))
        np.testing.assert_allclose(lg[0, h, sl], Lo[0, h, sl], atol=1e-3)
    print("ragged", L, block, rep, "worst", worst)


def test_ragged_rows_past_lq_untouched(cuda_ok):
    # the output buffer is one block longer than Lq; the extra rows (a view
    # past the end of O) must keep their sentinel values
    L, block, Hq = 1000, 128, 4
    inp = _mixture(L, block, Hq, 2, 603)
    Q, K, V = dev(inp["Q"]), dev(inp["K"]), dev(inp["V"])
    big = torch.full((1, 1024 + 128, Hq, 128), 7.0, dtype=torch.bfloat16, device="cuda")
    out = big[:, :L]
    lists = rbs.rbs_lists_causal_full(1, Hq, 8)
    rbs.bsa_prefill(Q, K, V, lists, block, block, out=out)
    empty = rbs.BlockLists.empty(Hq * 8, 1, "cuda")
    empty.row_ptr.zero_()
    big2 = torch.full_like(big, 7.0)
    rbs.bsa_prefill(Q, K, V, empty, block, block, out=big2[:, :L])  # empty rows: zeros up to Lq only
    torch.cuda.synchronize()
    assert rbs.rbs_get_device_error() == 0
    assert bool(torch.all(big[:, L:] == 7.0)) and bool(torch.all(big2[:, L:] == 7.0))
    assert bool(torch.all(big2[:, :L] == 0.0))
    Od = O.dense_causal_attention(inp["Q"], inp["K"], inp["V"])
    assert np.abs(out.float().cpu().numpy() - Od).max() <= 2e-2


@pytest.mark.parametrize("causal", [1, 0])
def test_ragged_keys_with_query_offset(cuda_ok, causal):
    # 141 queries at the end of 4173 keys (64-token blocks: the last key block
    # holds 13 keys, the last query block 13 queries); query block 0 is key
    # block 63.  Full lists over the visible (or all) key blocks.
    block, Lk, q_off = 64, 4173, 4032
    inp = _cut(make_tiny(L=4224, Hq=4, Hkv=2, block=block, seed=604), Lk)
    Qh = np.ascontiguousarray(inp["Q"][:, q_off:])
    Lq, nqb, nkb, Hq = Qh.shape[1], 3, 66, 4
    if causal:
        lists = rbs.rbs_lists_causal_full(1, Hq, nqb, q_off // block)
        rp, ci, _ = lists_np(lists)
    else:
        rp = np.arange(0, Hq * nqb * nkb + 1, nkb)
        ci = np.tile(np.arange(nkb), Hq * nqb)
        lists = rbs.BlockLists.empty(Hq * nqb, ci.size, "cuda")
        lists.row_ptr.copy_(torch.from_numpy(rp.astype(np.int32)))
        lists.col_idx.copy_(torch.from_numpy(ci.astype(np.int32)))
    out, lse = rbs.bsa_prefill(dev(Qh), dev(inp["K"]), dev(inp["V"]), lists, block, block, q_offset=q_off,
                               causal=bool(causal), return_lse=True)
    torch.cuda.synchronize()
    assert rbs.rbs_get_device_error() == 0
    Oo, Lo = O.masked_attention(Qh, inp["K"], inp["V"], rp, ci, block, block, q_offset=q_off, causal=causal)
    o_rows_close(out, Oo, range(Hq * nqb), Hq, nqb, block)
    np.testing.assert_allclose(lse.cpu().numpy(), Lo, atol=1e-3)
    if causal:
        np.testing.assert_allclose(Oo, O.dense_causal_attention(Qh, inp["K"], inp["V"], q_offset=q_off), atol=1e-12)
