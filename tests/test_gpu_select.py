"""GPU parity: two-branch selection -> CSR lists, against the oracle's lists.

Lists must match exactly, branch by branch, except for blocks whose oracle
score lies within 1e-3 * max(1, |tau|) of that branch's threshold tau; those
are counted.  Each GPU branch must keep exactly k_i blocks, the union must be
the two branches plus the forced blocks, rows ascending.
"""

import numpy as np
import pytest
import torch

import block_sparse_long_rbs_b200 as rbs
from helpers import compare_selection, dense_masks, dev, lists_np
from oracle import rbs_oracle as O
from workloads import WORKLOADS, make_inputs, make_mixture, make_tied, make_tiny

pytestmark = pytest.mark.gpu


def _run(inp, block, rho_c, rho_r, **kw):
    Q, K = inp["Q"], inp["K"]
    B, L, Hq, _ = Q.shape
    Hkv = K.shape[2]
    nqb = L // block
    nkb = K.shape[1] // block
    p = rbs.SelectParams(block_q=block, block_k=block, rho_centroid=rho_c, rho_rescue=rho_r, **kw)
    Cg, Rg = rbs.rbs_block_stats(dev(K), block)
    lists = rbs.rbs_select(dev(Q), Cg, Rg, p)
    torch.cuda.synchronize()
    assert rbs.rbs_get_device_error() == 0
    Co, Ro = O.block_stats(K, block)
    po = O.SelectParams(block_q=block, block_k=block, rho_centroid=float(np.float32(rho_c)),
                        rho_rescue=float(np.float32(rho_r)), **{k: (float(np.float32(v)) if isinstance(v, float) else v)
                                                                for k, v in kw.items()})
    ora = O.select_blocks(Q, Co, Ro, po, keep_scores=True)
    return compare_selection(lists, ora, Hq, nqb, nkb, exact_k=kw.get("threshold_mode", 0) == 0)


def test_select_tiny_config(cuda_ok):
    w = WORKLOADS["tiny_rbs_4k"]
    rep = _run(make_inputs(w), 64, w.rho, w.rho)
    print("tiny", rep)


@pytest.mark.parametrize("beta_mode,const", [(0, 1.0), (1, 1.0), (1, 0.0)])
def test_select_mixture_small_beta_modes(cuda_ok, beta_mode, const):
    inp = make_mixture(L=8192, Hq=16, Hkv=2, block=128, seed=201)
    rep = _run(inp, 128, 0.1, 0.15, beta_mode=beta_mode, beta_const=const)
    print("mixture8k", beta_mode, const, rep)


def test_select_force_sink_batch2_ragged_group(cuda_ok):
    # batch 2, G = 6 (rows per CTA fall back to 6), sink forced
    inp = make_mixture(L=4096, Hq=12, Hkv=2, block=128, seed=202, batch=2)
    rep = _run(inp, 128, 0.2, 0.1, force_sink=1)
    print("sink", rep)


def test_select_noncausal_with_offset(cuda_ok):
    inp = make_mixture(L=4096, Hq=4, Hkv=1, block=64, seed=203)
    rep = _run(inp, 64, 0.1, 0.1, causal=0)
    print("noncausal", rep)


def test_select_32k_gqa_config(cuda_ok):
    w = WORKLOADS["gqa_rbs_32k"]
    inp = make_inputs(w)
    Co, Ro = O.block_stats(inp["K"], 128)
    rho, dens = O.bisect_rho(inp["Q"], Co, Ro, O.SelectParams(), w.density_target)
    rho32 = float(np.float32(rho))
    rep = _run(inp, 128, rho32, rho32)
    print("32k", rho32, dens, rep)
    assert abs(rep["nnz_gpu"] - rep["nnz_oracle"]) <= rep["centroid"] + rep["rescue"]


def test_select_128k_config(cuda_ok):
    w = WORKLOADS["gqa_rbs_128k"]
    rep = _run(make_inputs(w), 128, w.rho, w.rho)
    print("128k", rep)


@pytest.mark.parametrize("n_patterns", [3, 40, 128])
def test_select_exact_ties(cuda_ok, n_patterns):
    # Scores tie exactly (repeated integer block contents): each branch must
    # keep the oracle's set exactly, ties at the threshold going to the lowest
    # block indices, with no near-threshold excuse.  Few patterns put hundreds
    # of ties at the threshold (more candidates than the pruned searches
    # hold), many put a handful.  512 key blocks: the widest top-k rows.
    block, rho = 128, 0.05
    inp = make_tied(L=65536, Hq=2, Hkv=1, block=block, n_patterns=n_patterns, seed=211)
    Q, K = inp["Q"], inp["K"]
    nqb = nkb = 65536 // block
    p = rbs.SelectParams(block_q=block, block_k=block, rho_centroid=rho, rho_rescue=rho)
    Cg, Rg = rbs.rbs_block_stats(dev(K), block)
    lists = rbs.rbs_select(dev(Q), Cg, Rg, p)
    torch.cuda.synchronize()
    assert rbs.rbs_get_device_error() == 0
    Co, Ro = O.block_stats(K, block)
    ora = O.select_blocks(Q, Co, Ro, O.SelectParams(block_q=block, block_k=block, rho_centroid=float(np.float32(rho)),
                                                     rho_rescue=float(np.float32(rho))), keep_scores=True)
    grp, gci, gfl = lists_np(lists)
    _, gc, gr = dense_masks(grp, gci, gfl, nkb)
    _, oc, orr = dense_masks(ora["row_ptr"], ora["col_idx"], ora["flags"], nkb)
    assert np.array_equal(gc, oc) and np.array_equal(gr, orr)
    # the ties are real: rows whose centroid threshold is shared by more
    # blocks than the branch keeps
    s_c = ora["scores"][(0, 0)][0]
    tau = ora["tau"][0, 0, :, 0]
    tied = [int((s_c[i, :i + 1] == tau[i]).sum()) for i in range(nqb)]
    assert max(tied) > 1
    print("ties", n_patterns, "max tied at tau", max(tied))


def test_select_deterministic(cuda_ok):
    inp = make_tiny(L=2048)
    p = rbs.SelectParams(block_q=64, block_k=64, rho_centroid=0.25, rho_rescue=0.25)
    Cg, Rg = rbs.rbs_block_stats(dev(inp["K"]), 64)
    a = rbs.rbs_select(dev(inp["Q"]), Cg, Rg, p)
    b = rbs.rbs_select(dev(inp["Q"]), Cg, Rg, p)
    assert torch.equal(a.row_ptr, b.row_ptr)
    n = a.nnz()
    assert torch.equal(a.col_idx[:n], b.col_idx[:n]) and torch.equal(a.flags[:n], b.flags[:n])


def test_select_graph_capture_matches_eager(cuda_ok):
    # Selection captured into a CUDA graph (every launch on the capturing
    # stream, no host synchronisation inside the call) gives the eager lists,
    # and a replayed graph recomputes them from new inputs in the same
    # buffers.
    inp = make_mixture(L=8192, Hq=16, Hkv=2, block=128, seed=207)
    Q, K = dev(inp["Q"]), dev(inp["K"])
    B, L, Hq, _ = Q.shape
    Hkv, nqb, nkb = K.shape[2], L // 128, L // 128
    p = rbs.SelectParams(block_q=128, block_k=128, rho_centroid=0.1, rho_rescue=0.1)
    C, R = rbs.rbs_block_stats(K, 128)
    eager = rbs.rbs_select(Q, C, R, p)
    ws = torch.empty(rbs.rbs_select_workspace_bytes(B, Hq, nqb, Hkv, nkb, p), dtype=torch.uint8, device="cuda")
    out = rbs.BlockLists.empty(B * Hq * nqb, rbs.rbs_select_capacity(B, Hq, nqb, nkb, p), "cuda")
    Qg = torch.zeros_like(Q)
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        rbs.rbs_select(Qg, C, R, p, workspace=ws, out=out)  # warm-up outside the capture
    torch.cuda.current_stream().wait_stream(s)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        rbs.rbs_select(Qg, C, R, p, workspace=ws, out=out)
    Qg.copy_(Q)
    g.replay()
    torch.cuda.synchronize()
    assert rbs.rbs_get_device_error() == 0
    n = eager.nnz()
    assert out.nnz() == n
    assert torch.equal(out.row_ptr, eager.row_ptr)
    assert torch.equal(out.col_idx[:n], eager.col_idx[:n]) and torch.equal(out.flags[:n], eager.flags[:n])
    del g


def test_select_rho_one_is_causal_full(cuda_ok):
    inp = make_tiny(L=1024)
    p = rbs.SelectParams(block_q=64, block_k=64, rho_centroid=1.0, rho_rescue=1.0)
    Cg, Rg = rbs.rbs_block_stats(dev(inp["K"]), 64)
    s = rbs.rbs_select(dev(inp["Q"]), Cg, Rg, p)
    f = rbs.rbs_lists_causal_full(1, 2, 16, 0)
    assert torch.equal(s.row_ptr, f.row_ptr)
    assert torch.equal(s.col_idx[:s.nnz()], f.col_idx[:f.nnz()])


@pytest.mark.parametrize("dc,dr", [(0.1, 0.5), (0.5, 2.0)])
def test_select_max_relative_tiny(cuda_ok, dc, dr):
    w = WORKLOADS["tiny_rbs_4k"]
    rep = _run(make_inputs(w), 64, w.rho, w.rho, threshold_mode=1, delta_centroid=dc, delta_rescue=dr)
    print("max-relative tiny", dc, dr, rep)


def test_select_max_relative_mixture_gqa(cuda_ok):
    inp = make_mixture(L=8192, Hq=16, Hkv=2, block=128, seed=201)
    rep = _run(inp, 128, 0.05, 0.05, threshold_mode=1, delta_centroid=0.5, delta_rescue=2.0)
    print("max-relative mixture", rep)


@pytest.mark.parametrize("case", ["mixture", "32k"])
def test_select_fused_kernel_with_smaller_workspace(cuda_ok, case):
    # a workspace one byte short of rbs_select_workspace_bytes has no room for
    # the score matrix: the fused CUDA-core scoring kernel runs instead of the
    # tensor-core scores; both must match the oracle
    if case == "mixture":
        inp, block, rho = make_mixture(L=8192, Hq=8, Hkv=2, block=128, seed=205, batch=2), 128, 0.1
    else:
        inp, block, rho = make_inputs(WORKLOADS["gqa_rbs_32k"]), 128, 0.05
    Q, K = inp["Q"], inp["K"]
    B, L, Hq, _ = Q.shape
    Hkv, nqb, nkb = K.shape[2], L // block, K.shape[1] // block
    p = rbs.SelectParams(block_q=block, block_k=block, rho_centroid=rho, rho_rescue=rho)
    Cg, Rg = rbs.rbs_block_stats(dev(K), block)
    full = rbs.rbs_select_workspace_bytes(B, Hq, nqb, Hkv, nkb, p)
    ws = torch.empty(full + 255, dtype=torch.uint8, device="cuda")
    off = (-ws.data_ptr()) % 256
    small = ws[off:off + full - 1]
    lists = rbs.rbs_select(dev(Q), Cg, Rg, p, workspace=small)
    ref = rbs.rbs_select(dev(Q), Cg, Rg, p)
    torch.cuda.synchronize()
    assert rbs.rbs_get_device_error() == 0
    Co, Ro = O.block_stats(K, block)
    po = O.SelectParams(block_q=block, block_k=block, rho_centroid=float(np.float32(rho)),
                        rho_rescue=float(np.float32(rho)))
    ora = O.select_blocks(Q, Co, Ro, po, keep_scores=True)
    rep_small = compare_selection(lists, ora, Hq, nqb, nkb)
    rep_full = compare_selection(ref, ora, Hq, nqb, nkb)
    print("fused", rep_small, "tensor-core", rep_full)


@pytest.mark.parametrize("layout", ["fused_qkv_view", "head_major"])
@pytest.mark.parametrize("small_ws", [False, True])
def test_select_strided_and_head_major_q(cuda_ok, layout, small_ws):
    # Q as a slice of a fused [B, L, 3 * Hq, 128] buffer (token stride > Hq * 128)
    # or as a head-major [B, Hq, L, 128] buffer seen as [B, L, Hq, 128] (token
    # stride 128): the lists must equal those of the contiguous Q, on the
    # tensor-core path and on the fused kernel (a workspace without room for
    # the score matrix)
    inp = make_mixture(L=8192, Hq=8, Hkv=2, block=128, seed=206)
    Qc = dev(inp["Q"])
    if layout == "fused_qkv_view":
        big = torch.zeros(1, 8192, 24, 128, dtype=torch.bfloat16, device="cuda")
        big[:, :, 8:16] = Qc
        Qv = big[:, :, 8:16]
    else:
        Qv = Qc.permute(0, 2, 1, 3).contiguous().permute(0, 2, 1, 3)
        assert Qv.stride(1) == 128
    assert torch.equal(Qv, Qc) and not Qv.is_contiguous()
    p = rbs.SelectParams(block_q=128, block_k=128, rho_centroid=0.1, rho_rescue=0.1)
    Cg, Rg = rbs.rbs_block_stats(dev(inp["K"]), 128)
    ws = None
    if small_ws:
        full = rbs.rbs_select_workspace_bytes(1, 8, 64, 2, 64, p)
        buf = torch.empty(full + 255, dtype=torch.uint8, device="cuda")
        off = (-buf.data_ptr()) % 256
        ws = buf[off:off + full - 1]
    a = rbs.rbs_select(Qc, Cg, Rg, p, workspace=ws)
    b = rbs.rbs_select(Qv, Cg, Rg, p, workspace=ws)
    torch.cuda.synchronize()
    assert rbs.rbs_get_device_error() == 0
    assert torch.equal(a.row_ptr, b.row_ptr)
    n = a.nnz()
    assert torch.equal(a.col_idx[:n], b.col_idx[:n]) and torch.equal(a.flags[:n], b.flags[:n])
