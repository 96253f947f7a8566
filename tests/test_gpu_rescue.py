"""GPU parity: rescue blocks with a controlled contribution
(bsa_prefill_rescue_weighted) against the oracle, which attends the regular
and the rescue blocks separately and merges the two partials with the rescue
partial's softmax mass scaled by the weight; special cases: weight 1 is
bsa_prefill, weight 0 is attention over the regular blocks alone, a row made
of rescue blocks only does not depend on a positive weight."""

import numpy as np
import pytest
import torch

import block_sparse_long_rbs_b200 as rbs
from helpers import dev, lists_np, o_rows_close
from oracle import rbs_oracle as O
from workloads import WORKLOADS, make_inputs, make_mixture

pytestmark = pytest.mark.gpu


def _setup(inp, block, rho_c, rho_r):
    p = rbs.SelectParams(block_q=block, block_k=block, rho_centroid=rho_c, rho_rescue=rho_r)
    C, R = rbs.rbs_block_stats(dev(inp["K"]), block)
    lists = rbs.rbs_select(dev(inp["Q"]), C, R, p)
    return lists, dev(inp["Q"]), dev(inp["K"]), dev(inp["V"])


def _rescue_rows(lists, limit):
    rp, ci, fl = lists_np(lists)
    rows = [r for r in range(rp.size - 1) if np.any(fl[rp[r]:rp[r + 1]] == O.FLAG_RESCUE)]
    step = max(1, len(rows) // limit)
    return rows[::step][:limit], rp, ci, fl


@pytest.mark.parametrize("w", [0.0, 0.25, 4.0])
def test_rescue_weighted_mixture_gqa(cuda_ok, w):
    inp = make_mixture(L=8192, Hq=8, Hkv=2, block=128, seed=501)
    lists, Q, K, V = _setup(inp, 128, 0.05, 0.15)
    rows, rp, ci, fl = _rescue_rows(lists, 24)
    assert len(rows) >= 8
    out, lse = rbs.bsa_prefill_rescue_weighted(Q, K, V, lists, w, 128, 128, return_lse=True)
    torch.cuda.synchronize()
    assert rbs.rbs_get_device_error() == 0
    Oo, Lo = O.rescue_weighted_attention(inp["Q"], inp["K"], inp["V"], rp, ci, fl, w, 128, 128, rows=rows)
    Hq, nqb = 8, 64
    worst = o_rows_close(out, Oo, rows, Hq, nqb, 128)
    lg = lse.cpu().numpy()
    for row in rows:
        hq, i = divmod(row, nqb)
        sl = slice(i * 128, (i + 1) * 128)
        np.testing.assert_allclose(lg[0, hq, sl], Lo[0, hq, sl], atol=1e-3)
    print("rescue weight", w, "worst", worst)


def test_rescue_weight_one_and_zero_special_cases(cuda_ok):
    inp = make_mixture(L=4096, Hq=4, Hkv=1, block=128, seed=502)
    lists, Q, K, V = _setup(inp, 128, 0.05, 0.2)
    base = rbs.bsa_prefill(Q, K, V, lists, 128, 128)
    one = rbs.bsa_prefill_rescue_weighted(Q, K, V, lists, 1.0, 128, 128)
    zero = rbs.bsa_prefill_rescue_weighted(Q, K, V, lists, 0.0, 128, 128)
    # the regular blocks alone, as ordinary lists
    rp, ci, fl = lists_np(lists)
    keep = (fl & (O.FLAG_CENTROID | O.FLAG_FORCED)) > 0
    counts = np.array([keep[rp[r]:rp[r + 1]].sum() for r in range(rp.size - 1)])
    reg = rbs.BlockLists.empty(rp.size - 1, int(keep.sum()), "cuda")
    reg.row_ptr.copy_(torch.from_numpy(np.concatenate([[0], np.cumsum(counts)]).astype(np.int32)))
    reg.col_idx.copy_(torch.from_numpy(ci[keep].astype(np.int32)))
    reg.flags.copy_(torch.from_numpy(fl[keep]))
    regular = rbs.bsa_prefill(Q, K, V, reg, 128, 128)
    torch.cuda.synchronize()
    assert rbs.rbs_get_device_error() == 0
    assert torch.equal(one, base)
    diff = (zero.float() - regular.float()).abs().max().item()
    print("weight 0 vs regular-only lists: max diff", diff, "identical", torch.equal(zero, regular))
    assert diff <= 2e-3
    assert not torch.equal(zero, base)


def test_rescue_only_rows(cuda_ok):
    # hand-built lists: rows made of rescue blocks only.  Weight 0 leaves them
    # empty (O = 0, lse = -inf); any positive weight cancels in the softmax.
    inp = make_mixture(L=1024, Hq=2, Hkv=1, block=128, seed=503)
    Q, K, V = dev(inp["Q"]), dev(inp["K"]), dev(inp["V"])
    nqb = 8
    rows = 2 * nqb
    ptr, idx, flg = [0], [], []
    for r in range(rows):
        i = r % nqb
        blocks = list(range(0, i + 1, 2))  # every other visible block
        idx += blocks
        flg += [O.FLAG_RESCUE] * len(blocks)
        ptr.append(len(idx))
    lists = rbs.BlockLists.empty(rows, len(idx), "cuda")
    lists.row_ptr.copy_(torch.tensor(ptr, dtype=torch.int32))
    lists.col_idx.copy_(torch.tensor(idx, dtype=torch.int32))
    lists.flags.copy_(torch.tensor(flg, dtype=torch.uint8))
    plain = rbs.bsa_prefill(Q, K, V, lists, 128, 128)
    half, lse_h = rbs.bsa_prefill_rescue_weighted(Q, K, V, lists, 0.5, 128, 128, return_lse=True)
    zero, lse0 = rbs.bsa_prefill_rescue_weighted(Q, K, V, lists, 0.0, 128, 128, return_lse=True)
    torch.cuda.synchronize()
    assert rbs.rbs_get_device_error() == 0
    assert (zero.float().abs().max().item() == 0.0) and bool(torch.all(torch.isneginf(lse0)))
    assert (half.float() - plain.float()).abs().max().item() <= 2e-3
    Oo, Lo = O.rescue_weighted_attention(inp["Q"], inp["K"], inp["V"], np.array(ptr), np.array(idx),
                                         np.array(flg, dtype=np.uint8), 0.5, 128, 128)
    o_rows_close(half, Oo, range(rows), 2, nqb, 128)
    np.testing.assert_allclose(lse_h.cpu().numpy(), Lo, atol=1e-3)


def test_rescue_weighted_128k_sampled(cuda_ok):
    w = WORKLOADS["gqa_rbs_128k"]
    inp = make_inputs(w)
    lists, Q, K, V = _setup(inp, 128, w.rho, w.rho)
    out = rbs.bsa_prefill_rescue_weighted(Q, K, V, lists, 0.5, 128, 128)
    torch.cuda.synchronize()
    assert rbs.rbs_get_device_error() == 0
    rows, rp, ci, fl = _rescue_rows(lists, 6)
    Oo, _ = O.rescue_weighted_attention(inp["Q"], inp["K"], inp["V"], rp, ci, fl, 0.5, 128, 128, rows=rows)
    print("rescue weighted 128k worst", o_rows_close(out, Oo, rows, 32, 1024, 128))


def test_rescue_weight_validation(cuda_ok):
    inp = make_mixture(L=1024, Hq=2, Hkv=1, block=128, seed=504)
    lists, Q, K, V = _setup(inp, 128, 0.25, 0.25)
    for bad in (-0.5, float("nan"), float("inf")):
        with pytest.raises(rbs.RbsError):
            rbs.bsa_prefill_rescue_weighted(Q, K, V, lists, bad, 128, 128)
    noflags = rbs.BlockLists(lists.row_ptr, lists.col_idx, None, lists.num_rows)
    with pytest.raises(rbs.RbsError):
        rbs.bsa_prefill_rescue_weighted(Q, K, V, noflags, 0.5, 128, 128)
    rbs.bsa_prefill_rescue_weighted(Q, K, V, noflags, 1.0, 128, 128)  # weight 1 needs no flags
    torch.cuda.synchronize()
