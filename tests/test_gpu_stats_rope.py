"""GPU parity: block statistics, beta, query pooling and RoPE re-encoding
against the fp64 oracle, through the C ABI."""

import numpy as np
import pytest
import torch

import block_sparse_long_rbs_b200 as rbs
from helpers import TOL_STATS_REL, dev, host_bits
from oracle import rbs_oracle as O
from workloads import WORKLOADS, make_block_attention, make_inputs, make_mixture, make_tiny

pytestmark = pytest.mark.gpu


def _stats_check(K_bits, block):
    Cg, Rg = rbs.rbs_block_stats(dev(K_bits), block)
    torch.cuda.synchronize()
    Co, Ro = O.block_stats(K_bits, block)
    Cg, Rg = Cg.cpu().numpy().astype(np.float64), Rg.cpu().numpy().astype(np.float64)
    rel_c = np.linalg.norm(Cg - Co, axis=-1) / np.maximum(np.linalg.norm(Co, axis=-1), 1e-30)
    rel_r = np.abs(Rg - Ro) / np.maximum(Ro, 1e-30)
    assert rel_c.max() <= TOL_STATS_REL, rel_c.max()
    assert rel_r.max() <= TOL_STATS_REL, rel_r.max()
    return rel_c.max(), rel_r.max()


def test_stats_tiny_block64(cuda_ok):
    inp = make_tiny()
    _stats_check(inp["K"], 64)


def test_stats_mixture_batch2_block128(cuda_ok):
    inp = make_mixture(L=8192, Hq=8, Hkv=2, block=128, seed=101, batch=2)
    _stats_check(inp["K"], 128)


def test_stats_full_128k(cuda_ok):
    w = WORKLOADS["gqa_rbs_128k"]
    inp = make_inputs(w)
    _stats_check(inp["K"], 128)


def test_stats_strided_view(cuda_ok):
    # K as the middle slice of a fused [B, L, 3*H, 128] QKV-style buffer
    inp = make_mixture(L=2048, Hq=4, Hkv=4, block=128, seed=102)
    big = np.zeros((1, 2048, 12, 128), dtype=np.uint16)
    big[:, :, 4:8] = inp["K"]
    Kv = dev(big)[:, :, 4:8]
    assert not Kv.is_contiguous()
    Cg, Rg = rbs.rbs_block_stats(Kv, 128)
    Cc, Rc = rbs.rbs_block_stats(dev(inp["K"]), 128)
    assert torch.equal(Cg, Cc) and torch.equal(Rg, Rc)


@pytest.mark.parametrize("mode,plo,phi,const", [(0, 0.0, 1.0, 1.0), (0, -1.0, 1.0, 1.0), (0, 0.1, 0.9, 1.0),
                                                (1, 0.0, 1.0, 0.35)])
def test_beta_matches_oracle(cuda_ok, mode, plo, phi, const):
    rng = np.random.default_rng(5)
    R = rng.gamma(2.0, 3.0, size=(2, 3, 1000)).astype(np.float32)
    R[1, 2] = 4.0  # a degenerate head
    p = rbs.SelectParams(beta_mode=mode, beta_p_lo=plo, beta_p_hi=phi, beta_const=const)
    bg, rg = rbs.rbs_block_beta(torch.from_numpy(R).cuda(), p)
    po = O.SelectParams(beta_mode=mode, beta_p_lo=float(np.float32(plo)), beta_p_hi=float(np.float32(phi)),
                        beta_const=float(np.float32(const)))
    bo, ro = O.rescue_beta(R.astype(np.float64), po)
    np.testing.assert_allclose(bg.cpu().numpy(), bo, atol=2e-6)
    if mode == 0:
        np.testing.assert_allclose(rg.cpu().numpy(), ro, rtol=1e-6)


@pytest.mark.parametrize("block,L,Hq", [(64, 4096, 2), (128, 8192, 6), (128, 2048, 64)])
def test_pool_matches_oracle(cuda_ok, block, L, Hq):
    inp = make_mixture(L=L, Hq=Hq, Hkv=Hq // 2 if Hq % 2 == 0 else 1, block=block, seed=103)
    qg, ng = rbs.rbs_pool_queries(dev(inp["Q"]), block)
    qo, no = O.pooled_queries(inp["Q"], block)
    np.testing.assert_allclose(qg.cpu().numpy(), qo, atol=1e-5)
    np.testing.assert_allclose(ng.cpu().numpy(), no, rtol=1e-5)


def _rope_check(x_bits, old, new, theta, style):
    x = dev(x_bits)
    y = rbs.rope_reencode(x, torch.from_numpy(old).int().cuda(), torch.from_numpy(new).int().cuda(), theta, style)
    ref = O.rope_reencode(x_bits, old, new, theta, style)
    yf = y.float().cpu().numpy()
    err = np.abs(yf - ref)
    assert err.max() <= 2e-2, err.max()
    # at most one bf16 ulp of the reference for 99.9% of the elements
    ulp = np.exp2(np.floor(np.log2(np.maximum(np.abs(ref), 2.0 ** -126))) - 7)
    frac = np.mean(err <= ulp)
    assert frac >= 0.999, frac
    return y


@pytest.mark.parametrize("style", [0, 1])
def test_rope_reencode_block_attention_cache(cuda_ok, style):
    inp = make_block_attention(passages=4, passage_len=2048, final_len=512, Hq=32, Hkv=8)
    K = inp["K"]
    old = np.zeros(K.shape[1], dtype=np.int32)
    loc = inp["local_pos"]
    glob = inp["global_pos"]
    # encode at local positions (re-encoding from 0), then move to global positions
    cached = _rope_check(K, old, loc, 500000.0, style)
    moved = rbs.rope_reencode(cached, torch.from_numpy(loc).cuda(), torch.from_numpy(glob).cuda(), 500000.0, style)
    direct = O.rope_rotate(K, glob, 500000.0, style)
    # two bf16 roundings (cache at local positions, then re-encoded) vs one exact rotation
    err = np.abs(moved.float().cpu().numpy() - direct)
    assert np.all(err <= 2e-2 + 2.0 ** -7 * np.abs(direct)), err.max()


def test_rope_in_place_and_identity(cuda_ok):
    inp = make_tiny(L=1024)
    x = dev(inp["K"])
    pos = torch.arange(1024, dtype=torch.int32, device="cuda")
    y = rbs.rope_reencode(x, pos, pos, 500000.0, 0)
    assert torch.equal(y, x)  # zero angle: exact identity
    x2 = x.clone()
    rbs.rope_reencode(x2, torch.zeros_like(pos), pos, 10000.0, 0, out=x2)
    ref = rbs.rope_reencode(x, torch.zeros_like(pos), pos, 10000.0, 0)
    assert torch.equal(x2, ref)
