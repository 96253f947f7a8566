"""GPU parity at the longest sequences the selection supports: 2048 and
4096 key blocks per sequence (the kernel variants with 64 and 128 key slots
per lane and one query block per CTA), with one branch on the pruned top-k
(k <= 64) and the other on the full bitwise search (k > 64), then exact
attention on sampled rows of the resulting lists."""

import numpy as np
import pytest
import torch

import block_sparse_long_rbs_b200 as rbs
from helpers import compare_selection, dev, lists_np, o_rows_close
from oracle import rbs_oracle as O
from workloads import make_mixture

pytestmark = pytest.mark.gpu


def _select_and_attend(inp, block, rho_c, rho_r, rows):
    Q, K, V = inp["Q"], inp["K"], inp["V"]
    B, L, Hq, _ = Q.shape
    nqb = nkb = L // block
    p = rbs.SelectParams(block_q=block, block_k=block, rho_centroid=rho_c, rho_rescue=rho_r)
    Qd, Kd, Vd = dev(Q), dev(K), dev(V)
    Cg, Rg = rbs.rbs_block_stats(Kd, block)
    lists = rbs.rbs_select(Qd, Cg, Rg, p)
    torch.cuda.synchronize()
    assert rbs.rbs_get_device_error() == 0
    Co, Ro = O.block_stats(K, block)
    po = O.SelectParams(block_q=block, block_k=block, rho_centroid=float(np.float32(rho_c)),
                        rho_rescue=float(np.float32(rho_r)))
    rep = compare_selection(lists, O.select_blocks(Q, Co, Ro, po, keep_scores=True), Hq, nqb, nkb)
    out = rbs.bsa_prefill(Qd, Kd, Vd, lists, block, block)
    torch.cuda.synchronize()
    assert rbs.rbs_get_device_error() == 0
    rp, ci, _ = lists_np(lists)
    Oo, _ = O.masked_attention(Q, K, V, rp, ci, block, block, rows=rows)
    worst = o_rows_close(out, Oo, rows, Hq, nqb, block)
    return rep, worst


def test_2048_key_blocks(cuda_ok):
    # 262144 tokens, 128-token blocks: k_c <= 41 (pruned search), k_r up to 205 (full search)
    inp = make_mixture(L=262144, Hq=2, Hkv=1, block=128, seed=401)
    nqb = 2048
    rows = [nqb - 1, nqb - 2, 1500, 777, 64, 2 * nqb - 1, nqb + 1024]
    rep, worst = _select_and_attend(inp, 128, 0.02, 0.1, rows)
    print("2048 blocks", rep, worst)


def test_4096_key_blocks(cuda_ok):
    # 262144 tokens, 64-token blocks: the largest block count the selection takes
    inp = make_mixture(L=262144, Hq=1, Hkv=1, block=64, seed=402)
    nqb = 4096
    rows = [nqb - 1, nqb - 2, 3000, 2049, 1000, 31]
    rep, worst = _select_and_attend(inp, 64, 0.01, 0.05, rows)
    print("4096 blocks", rep, worst)
