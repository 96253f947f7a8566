"""GPU parity: block-sparse prefill attention (tcgen05 kernel) against the
fp64 oracle run on the GPU's own lists; 100% density against dense causal
attention; the Block-attention RAG flow; edge cases and device-error paths."""

import math

import numpy as np
import pytest
import torch

import block_sparse_long_rbs_b200 as rbs
from helpers import TOL_O_ABS, dev, lists_np, o_rows_close
from oracle import rbs_oracle as O
from workloads import WORKLOADS, make_block_attention, make_inputs, make_mixture, make_tiny

pytestmark = pytest.mark.gpu


def _select(inp, block, rho):
    p = rbs.SelectParams(block_q=block, block_k=block, rho_centroid=rho, rho_rescue=rho)
    C, R = rbs.rbs_block_stats(dev(inp["K"]), block)
    return rbs.rbs_select(dev(inp["Q"]), C, R, p)


def _attn_check(inp, lists, block, rows=None, q_offset=0, Qbits=None, lse_check=True):
    Qb = inp["Q"] if Qbits is None else Qbits
    Q, K, V = dev(Qb), dev(inp["K"]), dev(inp["V"])
    out, lse = rbs.bsa_prefill(Q, K, V, lists, block, block, q_offset=q_offset, return_lse=True)
    torch.cuda.synchronize()
    assert rbs.rbs_get_device_error() == 0
    rp, ci, _ = lists_np(lists)
    Oo, Lo = O.masked_attention(Qb, inp["K"], inp["V"], rp, ci, block, block, q_offset=q_offset, rows=rows)
    Hq = Qb.shape[2]
    nqb = Qb.shape[1] // block
    use_rows = range(rp.size - 1) if rows is None else rows
    worst = o_rows_close(out, Oo, use_rows, Hq, nqb, block)
    if lse_check:
        lg = lse.cpu().numpy()
        for row in use_rows:
            b, rem = divmod(int(row), Hq * nqb)
            hq, i = divmod(rem, nqb)
            sl = slice(i * block, (i + 1) * block)
            np.testing.assert_allclose(lg[b, hq, sl], Lo[b, hq, sl], atol=1e-3)
    return out, worst


def test_attention_tiny_config_block64(cuda_ok):
    w = WORKLOADS["tiny_rbs_4k"]
    inp = make_inputs(w)
    _, worst = _attn_check(inp, _select(inp, 64, w.rho), 64)
    print("tiny worst", worst)


def test_attention_mixture_gqa_block128(cuda_ok):
    inp = make_mixture(L=8192, Hq=16, Hkv=2, block=128, seed=301, batch=2)
    _, worst = _attn_check(inp, _select(inp, 128, 0.1), 128)
    print("mixture worst", worst)


@pytest.mark.parametrize("block", [64, 128])
def test_full_density_equals_dense_causal(cuda_ok, block):
    inp = make_tiny(L=2048, Hq=4, Hkv=2, block=block, seed=302)
    lists = rbs.rbs_lists_causal_full(1, 4, 2048 // block)
    out = rbs.bsa_prefill(dev(inp["Q"]), dev(inp["K"]), dev(inp["V"]), lists, block, block)
    ref = O.dense_causal_attention(inp["Q"], inp["K"], inp["V"])
    err = np.abs(out.float().cpu().numpy() - ref).max()
    assert err <= TOL_O_ABS, err


def test_full_density_query_offset(cuda_ok):
    # the last 4 query blocks of a 2048-token prompt against all of its keys
    inp = make_tiny(L=2048, Hq=2, Hkv=1, block=128, seed=303)
    Qtail = inp["Q"][:, 1536:]
    lists = rbs.rbs_lists_causal_full(1, 2, 4, q_block_offset=12)
    out = rbs.bsa_prefill(dev(Qtail), dev(inp["K"]), dev(inp["V"]), lists, 128, 128, q_offset=1536)
    ref = O.dense_causal_attention(Qtail, inp["K"], inp["V"], q_offset=1536)
    assert np.abs(out.float().cpu().numpy() - ref).max() <= TOL_O_ABS


def test_attention_128k_sampled_rows(cuda_ok):
    w = WORKLOADS["gqa_rbs_128k"]
    inp = make_inputs(w)
    lists = _select(inp, 128, w.rho)
    rp, _, _ = lists_np(lists)
    Hq, nqb = 32, 1024
    lens = np.diff(rp)
    rng = np.random.default_rng(0)
    rows = set(rng.choice(rp.size - 1, 48, replace=False).tolist())
    rows |= {0, nqb - 1, (Hq - 1) * nqb, rp.size - 2}
    rows |= set(np.argsort(-lens, kind="stable")[:12].tolist())
    _, worst = _attn_check(inp, lists, 128, rows=sorted(rows))
    print("128k sampled worst", worst, "rows", len(rows))


def test_block_attention_rag_flow(cuda_ok):
    # 4 passages x 2048 + 512-token final block at the full head counts
    P, PL, FL = 4, 2048, 512
    inp = make_block_attention(passages=P, passage_len=PL, final_len=FL, Hq=32, Hkv=8)
    blk, theta = 128, 500000.0
    L = P * PL + FL
    Qraw, Kraw, V = dev(inp["Q"]), dev(inp["K"]), dev(inp["V"])
    zero = torch.zeros(L, dtype=torch.int32, device="cuda")
    loc = torch.from_numpy(inp["local_pos"]).cuda()
    glob = torch.from_numpy(inp["global_pos"]).cuda()
    # cache build: passages encoded at local positions, block-diagonal mask
    Kc = rbs.rope_reencode(Kraw, zero, loc, theta)
    Qc = rbs.rope_reencode(Qraw, zero, loc, theta)
    seg = inp["seg_start"].tolist()
    cache_lists = rbs.rbs_lists_block_attention(seg, inp["final_start"], blk, 1, 32, 0, P * PL // blk)
    Opass = rbs.bsa_prefill(Qc[:, :P * PL], Kc[:, :P * PL], V[:, :P * PL], cache_lists, blk, blk)
    # re-encode the cached keys to their global offsets; final block at global positions
    Kg = rbs.rope_reencode(Kc, loc, glob, theta)
    Qf = rbs.rope_reencode(Qraw[:, P * PL:].contiguous(), zero[:FL], glob[P * PL:], theta)
    final_lists = rbs.rbs_lists_block_attention(seg, inp["final_start"], blk, 1, 32, P * PL // blk, FL // blk)
    Ofin = rbs.bsa_prefill(Qf, Kg, V, final_lists, blk, blk, q_offset=P * PL)
    torch.cuda.synchronize()
    assert rbs.rbs_get_device_error() == 0
    # lists equal the oracle's builder exactly
    for gl, (f, n) in ((cache_lists, (0, P * PL // blk)), (final_lists, (P * PL // blk, FL // blk))):
        rp, ci = O.block_attention_lists(seg, inp["final_start"], blk, 1, 32, f, n)
        grp, gci, _ = lists_np(gl)
        assert np.array_equal(grp, rp) and np.array_equal(gci, ci)
    # oracle: keys encoded directly at global positions, final block attends causally to all
    Kglob = O.rope_rotate(inp["K"], inp["global_pos"], theta)
    Qglob_f = O.rope_rotate(inp["Q"][:, P * PL:], inp["global_pos"][P * PL:], theta)
    rp, ci = O.block_attention_lists(seg, inp["final_start"], blk, 1, 32, P * PL // blk, FL // blk)
    rows = [0, 3, 5, 40, 77, 101, 127]
    Oo, _ = O.masked_attention(Qglob_f, Kglob, O.bf16_to_f64(inp["V"]), rp, ci, blk, blk, q_offset=P * PL, rows=rows)
    o_rows_close(Ofin, Oo, rows, 32, FL // blk, blk)
    # passages: encoded at local positions, each only within itself
    Kloc = O.rope_rotate(inp["K"][:, :P * PL], inp["local_pos"][:P * PL], theta)
    Qloc = O.rope_rotate(inp["Q"][:, :P * PL], inp["local_pos"][:P * PL], theta)
    rp, ci = O.block_attention_lists(seg, inp["final_start"], blk, 1, 32, 0, P * PL // blk)
    prow = [0, 15, 16, 33, 63, 64 * 7 + 20, 64 * 31 + 63]
    Op, _ = O.masked_attention(Qloc, Kloc, O.bf16_to_f64(inp["V"][:, :P * PL]), rp, ci, blk, blk, rows=prow)
    o_rows_close(Opass, Op, prow, 32, P * PL // blk, blk)


def test_block_attention_passage_independence_on_gpu(cuda_ok):
    inp = make_block_attention(passages=3, passage_len=1024, final_len=256, Hq=4, Hkv=2, seed=310)
    other = make_block_attention(passages=3, passage_len=1024, final_len=256, Hq=4, Hkv=2, seed=311)
    seg = inp["seg_start"].tolist()
    L = inp["Q"].shape[1]
    lists = rbs.rbs_lists_block_attention(seg, inp["final_start"], 128, 1, 4, 0, L // 128)
    a = rbs.bsa_prefill(dev(inp["Q"]), dev(inp["K"]), dev(inp["V"]), lists, 128, 128)
    Q2, K2, V2 = other["Q"].copy(), other["K"].copy(), other["V"].copy()
    sl = slice(1024, 2048)
    Q2[:, sl], K2[:, sl], V2[:, sl] = inp["Q"][:, sl], inp["K"][:, sl], inp["V"][:, sl]
    b = rbs.bsa_prefill(dev(Q2), dev(K2), dev(V2), lists, 128, 128)
    assert torch.equal(a[:, sl], b[:, sl])  # bit for bit
    assert not torch.equal(a[:, 3072:], b[:, 3072:])


def test_empty_rows_give_zero_and_neg_inf_lse(cuda_ok):
    inp = make_tiny(L=512, Hq=2, Hkv=1, block=128, seed=320)
    # rows: head 0 -> [0], [], [0, 2], [3]; head 1 -> [], [1], [], [0, 1, 2, 3]
    rows = [[0], [], [0, 2], [3], [], [1], [], [0, 1, 2, 3]]
    rp = np.concatenate([[0], np.cumsum([len(r) for r in rows])]).astype(np.int32)
    ci = np.array(sum(rows, []), dtype=np.int32)
    lists = rbs.BlockLists(torch.from_numpy(rp).cuda(), torch.from_numpy(ci).cuda(), None, 8)
    out, lse = rbs.bsa_prefill(dev(inp["Q"]), dev(inp["K"]), dev(inp["V"]), lists, 128, 128, return_lse=True)
    torch.cuda.synchronize()
    assert rbs.rbs_get_device_error() == 0
    Oo, Lo = O.masked_attention(inp["Q"], inp["K"], inp["V"], rp.astype(np.int64), ci.astype(np.int64), 128, 128)
    o_rows_close(out, Oo, range(8), 2, 4, 128)
    assert torch.all(out[0, 128:256, 0] == 0) and torch.all(torch.isneginf(lse[0, 1, :128]))


def test_bad_block_index_sets_device_error_without_fault(cuda_ok):
    inp = make_tiny(L=512, Hq=2, Hkv=1, block=128, seed=321)
    rp = np.array([0, 1, 2, 3, 4, 5, 6, 7, 8], dtype=np.int32)
    ci = np.array([0, 1, 2, 3, 0, 99, 2, 3], dtype=np.int32)  # 99 is out of range
    lists = rbs.BlockLists(torch.from_numpy(rp).cuda(), torch.from_numpy(ci).cuda(), None, 8)
    out = rbs.bsa_prefill(dev(inp["Q"]), dev(inp["K"]), dev(inp["V"]), lists, 128, 128)
    torch.cuda.synchronize()
    assert rbs.rbs_get_device_error() & rbs.DEVERR_BLOCK_INDEX
    assert rbs.rbs_get_device_error() == 0  # read-and-clear
    good = torch.isfinite(out.float()).all()
    assert bool(good)


def test_row_ptr_beyond_capacity_is_skipped(cuda_ok):
    inp = make_tiny(L=256, Hq=1, Hkv=1, block=128, seed=322)
    rp = torch.tensor([0, 1, 50], dtype=torch.int32, device="cuda")  # row 1 overruns the 2-entry capacity
    ci = torch.tensor([0, 1], dtype=torch.int32, device="cuda")
    lists = rbs.BlockLists(rp, ci, None, 2)
    rbs.bsa_prefill(dev(inp["Q"]), dev(inp["K"]), dev(inp["V"]), lists, 128, 128)
    torch.cuda.synchronize()
    assert rbs.rbs_get_device_error() & rbs.DEVERR_ROW_PTR


def test_strided_qkv_views(cuda_ok):
    # Q, K, V as slices of one fused [B, L, Hq + 2 Hkv, 128] projection output
    inp = make_mixture(L=2048, Hq=8, Hkv=2, block=128, seed=323)
    fused = np.concatenate([inp["Q"], inp["K"], inp["V"]], axis=2)
    F = dev(fused)
    Q, K, V = F[:, :, :8], F[:, :, 8:10], F[:, :, 10:12]
    lists = _select(inp, 128, 0.25)
    a = rbs.bsa_prefill(Q, K, V, lists, 128, 128)
    b = rbs.bsa_prefill(dev(inp["Q"]), dev(inp["K"]), dev(inp["V"]), lists, 128, 128)
    assert torch.equal(a, b)


def test_attention_deterministic(cuda_ok):
    inp = make_mixture(L=4096, Hq=8, Hkv=2, block=128, seed=324)
    lists = _select(inp, 128, 0.2)
    Q, K, V = dev(inp["Q"]), dev(inp["K"]), dev(inp["V"])
    a = rbs.bsa_prefill(Q, K, V, lists, 128, 128)
    b = rbs.bsa_prefill(Q, K, V, lists, 128, 128)
    assert torch.equal(a, b)
