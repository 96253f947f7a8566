"""GPU parity for the Block-attention mask with passages at any token offset
("Block-Attention for Efficient Prefilling", 2.2 Block segmentation and 2.4
Block fine-tune): lists equal the oracle's builder, bsa_prefill_segments
equals the oracle's masked attention with the token bound, and a passage's
outputs do not depend on the other passages, bit for bit."""

import numpy as np
import pytest
import torch

import block_sparse_long_rbs_b200 as rbs
from helpers import TOL_O_ABS, dev, lists_np, o_rows_close
from oracle import rbs_oracle as O
from workloads import make_block_attention

pytestmark = pytest.mark.gpu

LENS = [1999, 2100, 517]  # no passage boundary on a block boundary
BLK = 128


def _inputs(seed=501, final_len=300, Hq=8, Hkv=2):
    return make_block_attention(final_len=final_len, Hq=Hq, Hkv=Hkv, block=BLK, seed=seed, passage_lens=LENS)


def test_ragged_segment_lists_match_the_oracle(cuda_ok):
    inp = _inputs()
    seg, final = inp["seg_start"].tolist(), inp["final_start"]
    L = inp["Q"].shape[1]
    nqb = -(-L // BLK)
    for first, num in ((0, nqb), (final // BLK, nqb - final // BLK), (5, 17)):
        gl = rbs.rbs_lists_block_attention(seg, final, BLK, 2, 8, first, num)
        rp, ci = O.block_attention_lists(seg, final, BLK, 2, 8, first, num)
        grp, gci, _ = lists_np(gl)
        assert np.array_equal(grp, rp) and np.array_equal(gci, ci)


def test_ragged_segment_attention_matches_the_oracle(cuda_ok):
    inp = _inputs()
    seg, final = inp["seg_start"].tolist(), inp["final_start"]
    L = inp["Q"].shape[1]
    nqb = -(-L // BLK)
    lists = rbs.rbs_lists_block_attention(seg, final, BLK, 1, 8, 0, nqb)
    out, lse = rbs.bsa_prefill_segments(dev(inp["Q"]), dev(inp["K"]), dev(inp["V"]), lists, seg, final,
                                        return_lse=True)
    torch.cuda.synchronize()
    assert rbs.rbs_get_device_error() == 0
    rp, ci, _ = lists_np(lists)
    ks = O.block_attention_key_start(seg, final, range(L))
    Oo, Lo = O.masked_attention(inp["Q"], inp["K"], inp["V"], rp, ci, BLK, BLK, key_start=ks)
    og = out.float().cpu().numpy()
    assert np.abs(og - Oo).max() <= 2e-2
    np.testing.assert_allclose(lse.cpu().numpy(), Lo, atol=1e-3)


def test_ragged_final_block_pass_with_query_offset(cuda_ok):
    # the final pass starts at the query block holding the final block's first
    # token; that block's passage tokens keep their passage mask
    inp = _inputs(seed=502)
    seg, final = inp["seg_start"].tolist(), inp["final_start"]
    L = inp["Q"].shape[1]
    nqb = -(-L // BLK)
    f0 = final // BLK
    lists = rbs.rbs_lists_block_attention(seg, final, BLK, 1, 8, f0, nqb - f0)
    Qf = inp["Q"][:, f0 * BLK:]
    out = rbs.bsa_prefill_segments(dev(Qf), dev(inp["K"]), dev(inp["V"]), lists, seg, final, q_offset=f0 * BLK)
    torch.cuda.synchronize()
    assert rbs.rbs_get_device_error() == 0
    rp, ci, _ = lists_np(lists)
    ks = O.block_attention_key_start(seg, final, range(f0 * BLK, L))
    Oo, _ = O.masked_attention(Qf, inp["K"], inp["V"], rp, ci, BLK, BLK, q_offset=f0 * BLK, key_start=ks)
    o_rows_close(out, Oo, range(rp.size - 1), 8, nqb - f0, BLK)


def test_ragged_passage_independence_on_gpu(cuda_ok):
    inp, other = _inputs(seed=503), _inputs(seed=504)
    seg, final = inp["seg_start"].tolist(), inp["final_start"]
    L = inp["Q"].shape[1]
    lists = rbs.rbs_lists_block_attention(seg, final, BLK, 1, 8, 0, -(-L // BLK))
    a = rbs.bsa_prefill_segments(dev(inp["Q"]), dev(inp["K"]), dev(inp["V"]), lists, seg, final)
    lo, hi = seg[1], seg[2]  # passage 1: tokens 1999 .. 4098
    Q2, K2, V2 = other["Q"].copy(), other["K"].copy(), other["V"].copy()
    Q2[:, lo:hi], K2[:, lo:hi], V2[:, lo:hi] = inp["Q"][:, lo:hi], inp["K"][:, lo:hi], inp["V"][:, lo:hi]
    b = rbs.bsa_prefill_segments(dev(Q2), dev(K2), dev(V2), lists, seg, final)
    torch.cuda.synchronize()
    assert torch.equal(a[:, lo:hi], b[:, lo:hi])  # bit for bit
    assert not torch.equal(a[:, final:], b[:, final:])
    # without the token bound the block lists alone let passage 1 see keys
    # of passages 0 and 2 that share its edge blocks
    c = rbs.bsa_prefill(dev(inp["Q"]), dev(inp["K"]), dev(inp["V"]), lists, BLK, BLK)
    d = rbs.bsa_prefill(dev(Q2), dev(K2), dev(V2), lists, BLK, BLK)
    assert not torch.equal(c[:, lo:hi], d[:, lo:hi])


def test_block_aligned_segments_equal_plain_prefill(cuda_ok):
    # with passages on block boundaries the token bound removes nothing the
    # lists keep: bsa_prefill_segments equals bsa_prefill bit for bit
    inp = make_block_attention(passages=3, passage_len=1024, final_len=256, Hq=4, Hkv=2, seed=505)
    seg, final = inp["seg_start"].tolist(), inp["final_start"]
    L = inp["Q"].shape[1]
    lists = rbs.rbs_lists_block_attention(seg, final, BLK, 1, 4, 0, L // BLK)
    Q, K, V = dev(inp["Q"]), dev(inp["K"]), dev(inp["V"])
    a = rbs.bsa_prefill_segments(Q, K, V, lists, seg, final)
    b = rbs.bsa_prefill(Q, K, V, lists, BLK, BLK)
    assert torch.equal(a, b)


FULL_RAGGED = [2048] * 7 + [1999, 2100, 2045] + [2048] * 6  # the bench's ragged variant (same total)


@pytest.mark.parametrize("ragged", [False, True])
def test_block_attention_full_config_sampled_rows(cuda_ok, ragged):
    # The Block-attention workload at its full size: 16 passages (2048 tokens
    # each, or three of 1,999 / 2,100 / 2,045 tokens), a 512-token final
    # block, 32 q / 8 KV heads.  Cache build at local positions, re-encoding
    # of the cached keys, final pass at global positions, as the bench runs
    # them; sampled rows against the oracle (keys encoded directly at their
    # positions), including query blocks that straddle a passage boundary.
    theta = 500000.0
    inp = make_block_attention(passages=16, passage_len=2048, final_len=512, Hq=32, Hkv=8, block=BLK,
                               passage_lens=FULL_RAGGED if ragged else None)
    seg, final = inp["seg_start"].tolist(), inp["final_start"]
    L = inp["Q"].shape[1]
    nqb, fb = L // BLK, final // BLK
    Qraw, Kraw, V = dev(inp["Q"]), dev(inp["K"]), dev(inp["V"])
    zero = torch.zeros(L, dtype=torch.int32, device="cuda")
    loc = torch.from_numpy(inp["local_pos"]).cuda()
    glob = torch.from_numpy(inp["global_pos"]).cuda()
    Kc = rbs.rope_reencode(Kraw, zero, loc, theta)
    Qc = rbs.rope_reencode(Qraw, zero, loc, theta)
    cache = rbs.rbs_lists_block_attention(seg, final, BLK, 1, 32, 0, fb)
    Opass = rbs.bsa_prefill_segments(Qc[:, :final], Kc[:, :final], V[:, :final], cache, seg, final)
    Kg = rbs.rope_reencode(Kc, loc, glob, theta)
    Qf = rbs.rope_reencode(Qraw[:, final:].contiguous(), zero[:L - final], glob[final:], theta)
    fin = rbs.rbs_lists_block_attention(seg, final, BLK, 1, 32, fb, nqb - fb)
    Ofin = rbs.bsa_prefill_segments(Qf, Kg, V, fin, seg, final, q_offset=final)
    torch.cuda.synchronize()
    assert rbs.rbs_get_device_error() == 0
    Vf = O.bf16_to_f64(inp["V"])
    # final block: every key of the prompt, causally, at global positions
    Kglob = O.rope_rotate(inp["K"], inp["global_pos"], theta)
    Qg = O.rope_rotate(inp["Q"][:, final:], inp["global_pos"][final:], theta)
    rp, ci = O.block_attention_lists(seg, final, BLK, 1, 32, fb, nqb - fb)
    ks = O.block_attention_key_start(seg, final, range(final, L))
    rows = [0 * 4 + 0, 7 * 4 + 3, 19 * 4 + 1, 31 * 4 + 3]  # (q head, final query block)
    Oo, _ = O.masked_attention(Qg, Kglob, Vf, rp, ci, BLK, BLK, q_offset=final, rows=rows, key_start=ks)
    o_rows_close(Ofin, Oo, rows, 32, nqb - fb, BLK)
    # passages: each token sees only its own passage, at local positions
    Kloc = O.rope_rotate(inp["K"][:, :final], inp["local_pos"][:final], theta)
    og = Opass.float().cpu().numpy()
    for i0, h in ((0, 0), (127, 5), (128, 12), (143, 30), (160, 21), (fb - 1, 9)):
        sl = slice(i0 * BLK, (i0 + 1) * BLK)
        Qs = O.rope_rotate(inp["Q"][:, sl], inp["local_pos"][sl], theta)
        rp, ci = O.block_attention_lists(seg, final, BLK, 1, 32, i0, 1)
        ks = O.block_attention_key_start(seg, final, range(i0 * BLK, (i0 + 1) * BLK))
        Oo, _ = O.masked_attention(Qs, Kloc, Vf[:, :final], rp, ci, BLK, BLK, q_offset=i0 * BLK, rows=[h], key_start=ks)
        got, ref = og[0, sl, h], Oo[0, :, h]
        assert np.all(np.isfinite(got)) and np.all(np.isfinite(ref))
        assert np.abs(got - ref).max() <= TOL_O_ABS, (i0, h, float(np.abs(got - ref).max()))
