"""Pins for the CPU fp64 oracle: closed forms, library routines, the pages'
invariants and brute force on tiny inputs.  CPU only.

Each test names what fixes the expected value.  None of them re-types the
oracle's own formula.
"""

import itertools
import math
import os

import numpy as np
import pytest
import torch

from oracle import rbs_oracle as O
from workloads import make_block_attention, make_mixture, make_tiny

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _read_kv(path):
    out = {}
    for line in open(path):
        line = line.strip()
        if not line or line.startswith("#"):
            continue
        k, v = line.split()
        out[k] = float(v)
    return out


# --------------------------------------------------------------------------
# Block statistics: closed forms


def test_stats_outlier_block_golden():
    g = _read_kv(os.path.join(GOLDEN, "stats_outlier_block.txt"))
    n, D = int(g["n"]), g["D"]
    d = 128
    a = np.zeros(d)
    a[:3] = (1.0, -2.0, 0.5)
    K = np.tile(a, (n, 1))
    K[17, 7] += D  # the outlier at an arbitrary position inside the block
    K = K[None, :, None, :]
    C, R = O.block_stats(K, n)
    assert C[0, 0, 0, 7] == pytest.approx(g["centroid_coord7"], abs=1e-15)
    assert C[0, 0, 0, 0] == pytest.approx(g["centroid_coord0"], abs=1e-15)
    assert C[0, 0, 0, 1] == pytest.approx(g["centroid_coord1"], abs=1e-15)
    assert C[0, 0, 0, 2] == pytest.approx(g["centroid_coord2"], abs=1e-15)
    assert R[0, 0, 0] == pytest.approx(g["radius"], abs=1e-12)


def test_stats_constant_and_two_point_blocks():
    rng = np.random.default_rng(1)
    d, n = 128, 64
    x, y, z = rng.standard_normal((3, d))
    K = np.empty((1, 3 * n, 2, d))
    K[0, :n, 0] = z  # constant block: c = z, r = 0
    K[0, n:2 * n:2, 0] = x  # two-point block (alternating): c = (x+y)/2, r = |x-y|/2
    K[0, n + 1:2 * n:2, 0] = y
    K[0, 2 * n:, 0] = 0.0
    K[0, :, 1] = K[0, ::-1, 0]  # head 1 = token-reversed head 0 (blocks reversed)
    C, R = O.block_stats(K, n)
    np.testing.assert_allclose(C[0, 0, 0], z, atol=1e-14)
    assert R[0, 0, 0] == pytest.approx(0.0, abs=1e-13)
    np.testing.assert_allclose(C[0, 0, 1], (x + y) / 2, atol=1e-14)
    assert R[0, 0, 1] == pytest.approx(np.linalg.norm(x - y) / 2, rel=1e-13)
    assert R[0, 0, 2] == 0.0
    np.testing.assert_allclose(C[0, 1, 2], z, atol=1e-14)
    np.testing.assert_allclose(R[0, 1, ::-1], R[0, 0], atol=1e-13)


def test_stats_reads_bf16_bits_exactly():
    # 1.5 and -0.25 are exact in bf16: bits 0x3FC0 and 0xBE80.
    bits = np.zeros((1, 2, 1, 128), dtype=np.uint16)
    bits[0, 0, 0, 0] = 0x3FC0
    bits[0, 1, 0, 0] = 0xBE80
    C, R = O.block_stats(bits, 2)
    assert C[0, 0, 0, 0] == 0.625
    assert R[0, 0, 0] == 0.875


# --------------------------------------------------------------------------
# beta: quantile vs numpy, closed forms


@pytest.mark.parametrize("p", [0.0, 0.1, 0.25, 0.5, 0.9, 1.0])
def test_quantile_type7_matches_numpy(p):
    x = np.random.default_rng(2).standard_normal(37)
    assert O.quantile_type7(x, p) == pytest.approx(float(np.quantile(x, p, method="linear")), abs=1e-15)


def test_quantile_type7_hand_values():
    assert O.quantile_type7(np.array([4.0, 1.0, 3.0, 2.0]), 0.5) == 2.5
    assert O.quantile_type7(np.array([10.0, 20.0]), 0.25) == 12.5


def test_beta_closed_forms():
    R = np.array([[[1.0, 2.0, 3.0, 5.0]]])
    b, rng = O.rescue_beta(R, O.SelectParams())
    np.testing.assert_allclose(b[0, 0], [0.0, 0.25, 0.5, 1.0])
    assert tuple(rng[0, 0]) == (1.0, 5.0)
    b, _ = O.rescue_beta(R, O.SelectParams(beta_p_lo=-1.0))
    np.testing.assert_allclose(b[0, 0], [0.2, 0.4, 0.6, 1.0])
    # quantiles 0.25 / 0.75 of {1,2,3,5} are 1.75 / 3.5: clamped both ends
    b, _ = O.rescue_beta(R, O.SelectParams(beta_p_lo=0.25, beta_p_hi=0.75))
    np.testing.assert_allclose(b[0, 0], [0.0, 0.25 / 1.75, 1.25 / 1.75, 1.0])
    b, _ = O.rescue_beta(np.full((1, 1, 5), 2.0), O.SelectParams())
    np.testing.assert_array_equal(b, 1.0)  # degenerate range
    b, _ = O.rescue_beta(R, O.SelectParams(beta_mode=1, beta_const=0.3))
    np.testing.assert_array_equal(b, 0.3)


def test_beta_is_per_prompt_and_head():
    R = np.array([[[1.0, 3.0], [10.0, 20.0]], [[0.0, 4.0], [5.0, 5.0]]])
    b, _ = O.rescue_beta(R, O.SelectParams())
    np.testing.assert_allclose(b, [[[0, 1], [0, 1]], [[0, 1], [1, 1]]])


# --------------------------------------------------------------------------
# Pooled query: closed forms


def test_pooled_queries_closed_forms():
    d = 128
    x = np.zeros(d)
    x[:2] = (3.0, 4.0)
    Q = np.zeros((1, 8, 2, d))
    Q[0, :4, 0] = x  # block 0 of head 0: identical rows -> mean x, norm 5
    Q[0, 4:8:2, 0] = x  # block 1 of head 0: rows x, -x -> mean 0
    Q[0, 5:8:2, 0] = -x
    Q[0, :, 1] = np.arange(8)[:, None]  # head 1: mean of 0..3 = 1.5, of 4..7 = 5.5
    qbar, qn = O.pooled_queries(Q, 4)
    np.testing.assert_allclose(qbar[0, 0, 0], x)
    assert qn[0, 0, 0] == pytest.approx(5.0)
    np.testing.assert_allclose(qbar[0, 0, 1], 0.0)
    np.testing.assert_allclose(qbar[0, 1, :, 0], [1.5, 5.5])
    assert qn[0, 1, 1] == pytest.approx(5.5 * math.sqrt(d))


# --------------------------------------------------------------------------
# Cauchy-Schwarz bound with beta = 1 (brute force, tiny inputs)


def _tiny(L=1024, Hq=2, Hkv=1, block=64):
    return make_tiny(L=L, Hq=Hq, Hkv=Hkv, block=block, seed=7)


def test_cauchy_schwarz_bound_pooled_and_per_token():
    inp = _tiny()
    Q, K = inp["Q"], inp["K"]
    blk = inp["block"]
    C, R = O.block_stats(K, blk)
    p = O.SelectParams(block_q=blk, block_k=blk, beta_mode=1, beta_const=1.0)
    beta, _ = O.rescue_beta(R, p)
    qbar, qn = O.pooled_queries(Q, blk)
    Kf = O.bf16_to_f64(K)
    Qf = O.bf16_to_f64(Q)
    nb = C.shape[2]
    for hq in range(Q.shape[2]):
        s_c, s_r = O.branch_scores(qbar[0, hq], qn[0, hq], C[0, 0], R[0, 0], beta[0, 0])
        for j in range(nb):
            kb = Kf[0, j * blk:(j + 1) * blk, 0]
            true_max = (qbar[0, hq] @ kb.T).max(axis=1)  # per query block i
            assert np.all(true_max <= s_r[:, j] + 1e-9)
            qt = Qf[0, j * blk:(j + 1) * blk, hq]  # a sample of individual tokens
            per_tok = (qt @ kb.T).max(axis=1)
            bound = qt @ C[0, 0, j] + np.linalg.norm(qt, axis=1) * R[0, 0, j]
            assert np.all(per_tok <= bound + 1e-9)


def test_cauchy_schwarz_bound_is_tight():
    # keys c + r*u and c - r*u with u = q/|q|: the max dot product equals the bound.
    d = 128
    rng = np.random.default_rng(3)
    q = rng.standard_normal(d)
    c = rng.standard_normal(d)
    r = 2.5
    u = q / np.linalg.norm(q)
    K = np.stack([c + r * u, c - r * u] * 2)[None, :, None, :]
    C, R = O.block_stats(K, 4)
    assert R[0, 0, 0] == pytest.approx(r, rel=1e-12)
    s_c, s_r = O.branch_scores(q[None], np.array([np.linalg.norm(q)]), C[0, 0], R[0, 0], np.ones(1))
    assert s_r[0, 0] == pytest.approx(float((K[0, :, 0] @ q).max()), rel=1e-12)


# --------------------------------------------------------------------------
# Top-k with ties: brute force


def test_keep_count_values():
    assert O.keep_count(0.25, 4) == 1
    assert O.keep_count(0.25, 5) == 2
    assert O.keep_count(0.1, 10) == 1
    assert O.keep_count(1.0, 7) == 7
    assert O.keep_count(1e-6, 7) == 1
    assert O.keep_count(0.05, 1024) == 52
    assert O.keep_count(float(np.float32(0.05)), 20) == 1  # float32 rho, exact product 1.0000000149
    assert O.keep_count(float(np.float32(0.1)), 30) == 3


def test_top_k_matches_brute_force_with_ties():
    rng = np.random.default_rng(4)
    for _ in range(200):
        n = int(rng.integers(1, 9))
        s = rng.integers(-2, 3, size=n).astype(np.float64)  # many ties
        k = int(rng.integers(1, n + 1))
        got = set(O.top_k_desc(s, k).tolist())
        # brute force: among all k-subsets, the one that dominates every outside element
        ok = []
        for sub in itertools.combinations(range(n), k):
            inside = set(sub)
            if all((s[a] > s[b]) or (s[a] == s[b] and a < b) for a in inside for b in range(n) if b not in inside):
                ok.append(inside)
        assert ok == [got]


# --------------------------------------------------------------------------
# Selection invariants (the pages: independent branch thresholds, masks OR-ed)


def _select(inp, **kw):
    blk = inp["block"]
    C, R = O.block_stats(inp["K"], blk)
    p = O.SelectParams(block_q=blk, block_k=blk, **kw)
    return O.select_blocks(inp["Q"], C, R, p), C, R, p


def test_select_branch_sizes_union_and_diag():
    inp = _tiny()
    sel, C, R, p = _select(inp, rho_centroid=0.25, rho_rescue=0.25)
    rp, ci, fl = sel["row_ptr"], sel["col_idx"], sel["flags"]
    nqb = C.shape[2]
    for row in range(rp.size - 1):
        i = row % nqb
        cols = ci[rp[row]:rp[row + 1]]
        f = fl[rp[row]:rp[row + 1]]
        assert np.all(np.diff(cols) > 0)
        assert cols[-1] == i and f[-1] & O.FLAG_FORCED
        assert np.all(cols <= i)
        k = O.keep_count(0.25, i + 1)
        assert np.count_nonzero(f & O.FLAG_CENTROID) == k
        assert np.count_nonzero(f & O.FLAG_RESCUE) == k
        assert np.all(f != 0)
        assert len(cols) <= min(i + 1, 2 * k + 1)


def test_select_beta_zero_reduces_to_centroid_only():
    inp = _tiny()
    sel, *_ = _select(inp, rho_centroid=0.25, rho_rescue=0.25, beta_mode=1, beta_const=0.0)
    fl = sel["flags"]
    assert np.array_equal((fl & O.FLAG_CENTROID) > 0, (fl & O.FLAG_RESCUE) > 0)


def test_select_rho_one_keeps_every_causal_block():
    inp = _tiny(L=512)
    sel, C, *_ = _select(inp, rho_centroid=1.0, rho_rescue=1.0)
    rp, ci = O.causal_full_lists(1, inp["Q"].shape[2], C.shape[2])
    assert np.array_equal(sel["row_ptr"], rp) and np.array_equal(sel["col_idx"], ci)


def test_select_nested_in_rho():
    inp = _tiny(L=512)
    small, *_ = _select(inp, rho_centroid=0.1, rho_rescue=0.1)
    big, *_ = _select(inp, rho_centroid=0.3, rho_rescue=0.3)
    for row in range(small["row_ptr"].size - 1):
        a = set(small["col_idx"][small["row_ptr"][row]:small["row_ptr"][row + 1]].tolist())
        b = set(big["col_idx"][big["row_ptr"][row]:big["row_ptr"][row + 1]].tolist())
        assert a <= b


def test_select_gqa_head_mapping_and_rescue():
    # Two KV heads of 2 q heads each.  KV head 0 hides one big key in block 3,
    # KV head 1 in block 5, each aligned with every query of its q heads.  With
    # beta = 1 and a one-block rescue budget, the rescue branch of q heads 0,1
    # must pick block 3 and of q heads 2,3 block 5 (for the last query block).
    d, blk, nb = 128, 16, 8
    rng = np.random.default_rng(5)
    Q = np.zeros((1, nb * blk, 4, d))
    Q[..., 0] = 1.0
    Q += 0.01 * rng.standard_normal(Q.shape)
    K = 0.01 * rng.standard_normal((1, nb * blk, 2, d))
    K[0, 3 * blk + 5, 0, 0] = 40.0
    K[0, 5 * blk + 2, 1, 0] = 40.0
    C, R = O.block_stats(K, blk)
    p = O.SelectParams(block_q=blk, block_k=blk, rho_centroid=1e-6, rho_rescue=1e-6, beta_mode=1,
                       beta_const=1.0, force_diag=0)
    sel = O.select_blocks(Q, C, R, p)
    rp, ci, fl = sel["row_ptr"], sel["col_idx"], sel["flags"]
    last = [hq * nb + nb - 1 for hq in range(4)]
    for hq, row in enumerate(last):
        cols = ci[rp[row]:rp[row + 1]]
        f = fl[rp[row]:rp[row + 1]]
        assert cols[f & O.FLAG_RESCUE > 0].tolist() == ([3] if hq < 2 else [5])


def test_bisect_rho_hits_density():
    inp = make_mixture(L=4096, Hq=4, Hkv=2, block=128, seed=11)
    C, R = O.block_stats(inp["K"], 128)
    p = O.SelectParams()
    rho, dens = O.bisect_rho(inp["Q"], C, R, p, 0.25)
    assert abs(dens - 0.25) < 0.0025 + 1.0 / (4 * 32 * 33 / 2)  # one pair of granularity
    p.rho_centroid = p.rho_rescue = rho
    sel = O.select_blocks(inp["Q"], C, R, p)
    assert O.list_density(sel["row_ptr"], 32, 32) == pytest.approx(dens, abs=1e-12)


# --------------------------------------------------------------------------
# Attention: 100% density == textbook dense causal attention == torch SDPA


def _sdpa_ref(Q, K, V, q_offset=0):
    q = torch.from_numpy(O.bf16_to_f64(Q)).permute(0, 2, 1, 3)
    k = torch.from_numpy(O.bf16_to_f64(K)).permute(0, 2, 1, 3)
    v = torch.from_numpy(O.bf16_to_f64(V)).permute(0, 2, 1, 3)
    G = q.shape[1] // k.shape[1]
    k = k.repeat_interleave(G, dim=1)
    v = v.repeat_interleave(G, dim=1)
    Lq, Lk = q.shape[2], k.shape[2]
    allowed = torch.arange(Lk)[None, :] <= (torch.arange(Lq)[:, None] + q_offset)
    o = torch.nn.functional.scaled_dot_product_attention(q, k, v, attn_mask=allowed)
    return o.permute(0, 2, 1, 3).numpy()


def test_dense_attention_matches_sdpa_gqa():
    inp = make_tiny(L=256, Hq=4, Hkv=2, block=64, seed=8)
    ref = _sdpa_ref(inp["Q"], inp["K"], inp["V"])
    got = O.dense_causal_attention(inp["Q"], inp["K"], inp["V"])
    np.testing.assert_allclose(got, ref, atol=1e-12)


def test_full_lists_equal_dense_attention_with_offset():
    inp = make_tiny(L=512, Hq=4, Hkv=2, block=64, seed=9)
    Q = inp["Q"][:, 256:]  # the last 4 query blocks, at positions 256..511
    rp, ci = O.causal_full_lists(1, 4, 4, q_block_offset=4)
    got, lse = O.masked_attention(Q, inp["K"], inp["V"], rp, ci, 64, 64, q_offset=256)
    ref = _sdpa_ref(Q, inp["K"], inp["V"], q_offset=256)
    np.testing.assert_allclose(got, ref, atol=1e-12)
    np.testing.assert_allclose(got, O.dense_causal_attention(Q, inp["K"], inp["V"], q_offset=256), atol=1e-12)
    # lse against its definition through torch.logsumexp on the masked logits
    q = O.bf16_to_f64(Q[0, :, 3])
    k = O.bf16_to_f64(inp["K"][0, :, 1])
    s = torch.from_numpy(q @ k.T / math.sqrt(128))
    s[torch.arange(512)[None, :] > torch.arange(256)[:, None] + 256] = -math.inf
    np.testing.assert_allclose(lse[0, 3], torch.logsumexp(s, dim=1).numpy(), atol=1e-12)


def test_masked_attention_hand_cases():
    d = 128
    v = np.arange(2 * 1 * d, dtype=np.float64).reshape(1, 2, 1, d)
    q = np.zeros((1, 2, 1, d))
    k = np.zeros((1, 2, 1, d))
    # row 0 (token 0) sees only key 0 -> output v0; token 1 sees two equal logits -> mean
    O_, lse = O.masked_attention(q, k, v, np.array([0, 1]), np.array([0]), 2, 2)
    np.testing.assert_allclose(O_[0, 0, 0], v[0, 0, 0])
    np.testing.assert_allclose(O_[0, 1, 0], v[0, :, 0].mean(axis=0))
    assert lse[0, 0, 0] == 0.0 and lse[0, 0, 1] == pytest.approx(math.log(2))
    # an empty list gives zeros and lse = -inf
    O_, lse = O.masked_attention(q, k, v, np.array([0, 0]), np.array([], dtype=np.int64), 2, 2)
    assert np.all(O_ == 0) and np.all(lse == -np.inf)


# --------------------------------------------------------------------------
# Block-attention: hand-enumerated lists and the independence invariant


def test_block_attention_lists_golden():
    exp = {}
    for line in open(os.path.join(GOLDEN, "block_attention_lists_tiny.txt")):
        if line.strip() and not line.startswith("#"):
            a, b = line.split(":")
            exp[int(a)] = [int(x) for x in b.split()]
    rp, ci = O.block_attention_lists([0, 256], 512, 128, 1, 1, 0, 5)
    for i in range(5):
        assert ci[rp[i]:rp[i + 1]].tolist() == exp[i]
    # rows of the final block only (a final-block pass with a query offset)
    rp, ci = O.block_attention_lists([0, 256], 512, 128, 1, 1, 4, 1)
    assert ci.tolist() == exp[4]


def test_block_attention_passages_are_independent():
    inp = make_block_attention(passages=3, passage_len=128, final_len=64, Hq=2, Hkv=1, block=64, seed=12)
    blk = 64
    L = inp["Q"].shape[1]
    rp, ci = O.block_attention_lists(inp["seg_start"], inp["final_start"], blk, 1, 2, 0, L // blk)
    base, _ = O.masked_attention(inp["Q"], inp["K"], inp["V"], rp, ci, blk, blk)
    other = make_block_attention(passages=3, passage_len=128, final_len=64, Hq=2, Hkv=1, block=64, seed=13)
    Q2, K2, V2 = other["Q"].copy(), other["K"].copy(), other["V"].copy()
    Q2[:, 128:256], K2[:, 128:256], V2[:, 128:256] = inp["Q"][:, 128:256], inp["K"][:, 128:256], inp["V"][:, 128:256]
    out2, _ = O.masked_attention(Q2, K2, V2, rp, ci, blk, blk)
    assert np.array_equal(base[:, 128:256], out2[:, 128:256])  # passage 1 unchanged, bit for bit
    assert not np.allclose(base[:, 384:], out2[:, 384:])  # the final block sees everything


# --------------------------------------------------------------------------
# RoPE: complex-number form, re-encoding == direct encoding, invariants


def test_rope_matches_complex_rotation():
    rng = np.random.default_rng(14)
    x = rng.standard_normal((1, 5, 2, 128))
    pos = np.array([0, 1, 7, 2048, 33279])
    theta = 500000.0
    got = O.rope_rotate(x, pos, theta, 0)
    freqs = np.power(theta, -np.arange(64) / 64.0)
    z = (x[..., :64] + 1j * x[..., 64:]) * np.exp(1j * pos[None, :, None, None] * freqs)
    np.testing.assert_allclose(got[..., :64], z.real, atol=1e-12)
    np.testing.assert_allclose(got[..., 64:], z.imag, atol=1e-12)
    got1 = O.rope_rotate(x, pos, theta, 1)
    z1 = (x[..., 0::2] + 1j * x[..., 1::2]) * np.exp(1j * pos[None, :, None, None] * freqs)
    np.testing.assert_allclose(got1[..., 0::2], z1.real, atol=1e-12)
    np.testing.assert_allclose(got1[..., 1::2], z1.imag, atol=1e-12)


@pytest.mark.parametrize("style", [0, 1])
def test_rope_reencode_equals_direct_encoding(style):
    rng = np.random.default_rng(15)
    x = rng.standard_normal((1, 6, 3, 128))
    old = np.array([0, 5, 100, 2047, 3, 0])
    new = np.array([0, 2053, 30820, 32767, 3, 1])
    cached = O.rope_rotate(x, old, 500000.0, style)
    np.testing.assert_allclose(O.rope_reencode(cached, old, new, 500000.0, style),
                               O.rope_rotate(x, new, 500000.0, style), atol=1e-11)
    np.testing.assert_allclose(O.rope_reencode(cached, old, old, 500000.0, style), cached, atol=1e-12)
    pairs = lambda a: a[..., :64] ** 2 + a[..., 64:] ** 2 if style == 0 else a[..., 0::2] ** 2 + a[..., 1::2] ** 2
    np.testing.assert_allclose(pairs(cached), pairs(x), rtol=1e-12)


def test_rope_relative_position_invariance():
    rng = np.random.default_rng(16)
    q = rng.standard_normal((1, 1, 1, 128))
    k = rng.standard_normal((1, 1, 1, 128))
    dots = []
    for shift in (0, 37, 32768):
        qr = O.rope_rotate(q, np.array([shift + 9]), 500000.0)
        kr = O.rope_rotate(k, np.array([shift + 2]), 500000.0)
        dots.append(float((qr * kr).sum()))
    assert dots[1] == pytest.approx(dots[0], abs=1e-10)
    assert dots[2] == pytest.approx(dots[0], abs=1e-10)


# --------------------------------------------------------------------------
# Planted mistakes: each pin above must fail on a plausible oracle bug.


def test_pins_catch_planted_mistakes(monkeypatch):
    good_scores = O.branch_scores

    def wrong_sign(qbar, qnorm, C, R, beta):
        s_c, s_r = good_scores(qbar, qnorm, C, R, beta)
        return s_c, 2 * s_c - s_r  # rescue term subtracted
    monkeypatch.setattr(O, "branch_scores", wrong_sign)
    with pytest.raises(AssertionError):
        test_cauchy_schwarz_bound_pooled_and_per_token()
    monkeypatch.setattr(O, "branch_scores", good_scores)

    good_stats = O.block_stats

    def radius_from_mean_distance(K, bk):
        C, R = good_stats(K, bk)
        return C, R * (bk - 1) / bk  # a "mean distance"-like shrink of the radius
    monkeypatch.setattr(O, "block_stats", radius_from_mean_distance)
    with pytest.raises(AssertionError):
        test_stats_outlier_block_golden()
    monkeypatch.setattr(O, "block_stats", good_stats)

    good_rot = O.rope_rotate

    def transposed(x, pos, theta, style=0):
        return good_rot(x, -np.asarray(pos), theta, style)  # rotation the wrong way
    monkeypatch.setattr(O, "rope_rotate", transposed)
    with pytest.raises(AssertionError):
        test_rope_matches_complex_rotation()


# ---- max-relative threshold mode ([RBS-en] "How This Fits Into the Broader
# Sparse Attention Landscape": thresholding against the row maximum, no sort)


def test_max_relative_hand_built_scores():
    # Every key of block j is v_j * e_0 (radius 0, so both branches score
    # v_j); every query is e_0, so s(i, j) = v_j exactly.
    d, blk, nb = 128, 16, 6
    v = np.array([1.0, 5.0, 4.5, 2.0, 4.9, 0.5])
    K = np.zeros((1, nb * blk, 1, d))
    for j in range(nb):
        K[0, j * blk:(j + 1) * blk, 0, 0] = v[j]
    Q = np.zeros((1, nb * blk, 1, d))
    Q[..., 0] = 1.0
    C, R = O.block_stats(K, blk)
    assert np.allclose(R, 0.0)
    p = O.SelectParams(block_q=blk, block_k=blk, threshold_mode=1, delta_centroid=0.55, delta_rescue=0.15,
                       force_diag=0)
    sel = O.select_blocks(Q, C, R, p)
    rp, ci, fl = sel["row_ptr"], sel["col_idx"], sel["flags"]
    # row i sees blocks 0..i; centroid keeps v_j >= max - 0.55, rescue v_j >= max - 0.15
    want_c = {0: [0], 1: [1], 2: [1, 2], 3: [1, 2], 4: [1, 2, 4], 5: [1, 2, 4]}
    want_r = {0: [0], 1: [1], 2: [1], 3: [1], 4: [1, 4], 5: [1, 4]}
    for i in range(nb):
        cols = ci[rp[i]:rp[i + 1]]
        f = fl[rp[i]:rp[i + 1]]
        assert cols[(f & O.FLAG_CENTROID) > 0].tolist() == want_c[i]
        assert cols[(f & O.FLAG_RESCUE) > 0].tolist() == want_r[i]
        assert sel["k"][0, 0, i].tolist() == [len(want_c[i]), len(want_r[i])]


def test_max_relative_zero_delta_is_top1_and_infinite_delta_is_full():
    inp = _tiny(L=512)
    top1, *_ = _select(inp, rho_centroid=1e-6, rho_rescue=1e-6)  # k = 1 per branch
    zero, *_ = _select(inp, threshold_mode=1, delta_centroid=0.0, delta_rescue=0.0)
    assert np.array_equal(top1["row_ptr"], zero["row_ptr"]) and np.array_equal(top1["col_idx"], zero["col_idx"])
    assert np.array_equal(top1["flags"], zero["flags"])
    full, C, *_ = _select(inp, threshold_mode=1, delta_centroid=np.inf, delta_rescue=np.inf)
    rp, ci = O.causal_full_lists(1, inp["Q"].shape[2], C.shape[2])
    assert np.array_equal(full["row_ptr"], rp) and np.array_equal(full["col_idx"], ci)


def test_max_relative_nested_in_delta():
    inp = _tiny(L=512)
    small, *_ = _select(inp, threshold_mode=1, delta_centroid=5.0, delta_rescue=5.0)
    big, *_ = _select(inp, threshold_mode=1, delta_centroid=20.0, delta_rescue=20.0)
    for row in range(small["row_ptr"].size - 1):
        a = set(small["col_idx"][small["row_ptr"][row]:small["row_ptr"][row + 1]].tolist())
        b = set(big["col_idx"][big["row_ptr"][row]:big["row_ptr"][row + 1]].tolist())
        assert a <= b


# --------------------------------------------------------------------------
# KV-group lists (one list per KV head, shared by its q heads)


def _rows_as_sets(sel):
    rp, ci = sel["row_ptr"], sel["col_idx"]
    return [set(ci[rp[r]:rp[r + 1]].tolist()) for r in range(rp.size - 1)]


def test_group_lists_with_one_head_per_group_are_the_head_lists():
    # Hq == Hkv: every group is a single q head, so the union is that head's list
    inp = make_mixture(L=2048, Hq=2, Hkv=2, block=128, seed=21)
    C, R = O.block_stats(inp["K"], 128)
    kw = dict(block_q=128, block_k=128, rho_centroid=0.2, rho_rescue=0.2)
    a = O.select_blocks(inp["Q"], C, R, O.SelectParams(**kw))
    b = O.select_blocks(inp["Q"], C, R, O.SelectParams(list_mode=1, **kw))
    for key in ("row_ptr", "col_idx", "flags"):
        assert np.array_equal(a[key], b[key])


def test_group_lists_are_the_set_union_of_their_heads():
    # 4 q heads on 2 KV heads, 2 batch entries: group row (b, g, i) must be
    # exactly the set union of rows (b, 2g, i) and (b, 2g + 1, i), with each
    # entry's flags the OR of the heads' flags for that block
    inp = make_mixture(L=2048, Hq=4, Hkv=2, block=128, seed=22, batch=2)
    C, R = O.block_stats(inp["K"], 128)
    kw = dict(block_q=128, block_k=128, rho_centroid=0.15, rho_rescue=0.15, force_sink=1)
    per = O.select_blocks(inp["Q"], C, R, O.SelectParams(**kw))
    grp = O.select_blocks(inp["Q"], C, R, O.SelectParams(list_mode=1, **kw))
    nqb, B, Hq, Hkv = 16, 2, 4, 2
    assert grp["row_ptr"].size - 1 == B * Hkv * nqb
    hs, gs = _rows_as_sets(per), _rows_as_sets(grp)
    grew = 0
    for b in range(B):
        for g in range(Hkv):
            for i in range(nqb):
                heads = [hs[(b * Hq + hq) * nqb + i] for hq in (2 * g, 2 * g + 1)]
                row = (b * Hkv + g) * nqb + i
                assert gs[row] == heads[0] | heads[1]
                grew += len(gs[row]) > max(len(h) for h in heads)
                e0, e1 = grp["row_ptr"][row], grp["row_ptr"][row + 1]
                assert np.all(np.diff(grp["col_idx"][e0:e1]) > 0)
                for e in range(e0, e1):
                    j, want = int(grp["col_idx"][e]), 0
                    for hq in (2 * g, 2 * g + 1):
                        r = (b * Hq + hq) * nqb + i
                        hit = np.nonzero(per["col_idx"][per["row_ptr"][r]:per["row_ptr"][r + 1]] == j)[0]
                        if hit.size:
                            want |= int(per["flags"][per["row_ptr"][r] + hit[0]])
                    assert int(grp["flags"][e]) == want
    assert grew > 0  # the heads of a group do select different blocks here


def test_group_lists_attention_is_per_head_attention_on_the_shared_row():
    # attention with one list per KV head equals attention with per-q-head
    # lists in which every q head carries its group's list
    inp = make_mixture(L=1024, Hq=4, Hkv=2, block=128, seed=23)
    C, R = O.block_stats(inp["K"], 128)
    grp = O.select_blocks(inp["Q"], C, R, O.SelectParams(block_q=128, block_k=128, rho_centroid=0.2,
                                                          rho_rescue=0.2, list_mode=1))
    nqb, Hq, G = 8, 4, 2
    rp, ci = [0], []
    for hq in range(Hq):
        for i in range(nqb):
            r = (hq // G) * nqb + i
            ci.extend(grp["col_idx"][grp["row_ptr"][r]:grp["row_ptr"][r + 1]].tolist())
            rp.append(len(ci))
    rows = [0, 7, 9, 14, 21, 31]
    Og, lg = O.masked_attention(inp["Q"], inp["K"], inp["V"], grp["row_ptr"], grp["col_idx"], 128, 128, rows=rows)
    Oe, le = O.masked_attention(inp["Q"], inp["K"], inp["V"], np.asarray(rp), np.asarray(ci), 128, 128, rows=rows)
    for row in rows:
        hq, i = divmod(row, nqb)
        t = slice(i * 128, (i + 1) * 128)
        assert np.array_equal(Og[0, t, hq], Oe[0, t, hq])
        assert np.array_equal(lg[0, hq, t], le[0, hq, t])
    # and the q heads of one group really differ in their queries: same list, different outputs
    assert not np.allclose(Og[0, 7 * 128:8 * 128, 0], Og[0, 7 * 128:8 * 128, 1])


def test_group_pins_catch_planted_mistakes(monkeypatch):
    good_union = O.group_union_lists

    def interleaved_groups(row_ptr, cols, flags, B, Hq, Hkv, nqb, nkb):
        # q head hq assigned to group hq % Hkv instead of hq // (Hq / Hkv)
        perm = [hq for g in range(Hkv) for hq in range(g, Hq, Hkv)]
        rp, ci, fl = [0], [], []
        for b in range(B):
            for hq in perm:
                for i in range(nqb):
                    r = (b * Hq + hq) * nqb + i
                    ci.extend(cols[row_ptr[r]:row_ptr[r + 1]])
                    fl.extend(flags[row_ptr[r]:row_ptr[r + 1]])
                    rp.append(len(ci))
        return good_union(rp, ci, fl, B, Hq, Hkv, nqb, nkb)
    monkeypatch.setattr(O, "group_union_lists", interleaved_groups)
    with pytest.raises(AssertionError):
        test_group_lists_are_the_set_union_of_their_heads()
    monkeypatch.setattr(O, "group_union_lists", good_union)

    good_attn = O.masked_attention

    def per_head_rows_only(Q, K, V, row_ptr, col_idx, *a, **kw):
        # a group row read as if it were per-head: q head hq takes row hq * nqb + i
        B, Lq, Hq, _ = Q.shape
        nqb = Lq // a[0]
        rows_in = len(row_ptr) - 1
        if rows_in == B * Hq * nqb:
            return good_attn(Q, K, V, row_ptr, col_idx, *a, **kw)
        rp = list(row_ptr) + [row_ptr[-1]] * (B * Hq * nqb - rows_in)
        return good_attn(Q, K, V, np.asarray(rp), col_idx, *a, **kw)
    monkeypatch.setattr(O, "masked_attention", per_head_rows_only)
    with pytest.raises(AssertionError):
        test_group_lists_attention_is_per_head_attention_on_the_shared_row()


# --------------------------------------------------------------------------
# Rescue blocks handled separately with a weighted contribution
# ([RBS-id] "Dual-Branch Selection")


def _weighted_case(seed=31):
    inp = make_mixture(L=1024, Hq=2, Hkv=1, block=128, seed=seed)
    C, R = O.block_stats(inp["K"], 128)
    sel = O.select_blocks(inp["Q"], C, R, O.SelectParams(block_q=128, block_k=128, rho_centroid=0.2,
                                                          rho_rescue=0.3))
    return inp, sel


def _filtered(sel, keep):
    rp, ci, fl = sel["row_ptr"], sel["col_idx"], sel["flags"]
    out_p, out_c = [0], []
    for r in range(rp.size - 1):
        out_c.extend(int(ci[e]) for e in range(rp[r], rp[r + 1]) if keep(int(fl[e])))
        out_p.append(len(out_c))
    return np.asarray(out_p), np.asarray(out_c, dtype=np.int64)


def test_rescue_weight_one_is_union_attention_and_zero_is_regular_only():
    inp, sel = _weighted_case()
    args = (inp["Q"], inp["K"], inp["V"])
    rescue_rows = 0
    for r in range(sel["row_ptr"].size - 1):
        f = sel["flags"][sel["row_ptr"][r]:sel["row_ptr"][r + 1]]
        rescue_rows += bool(np.any(f == O.FLAG_RESCUE))
    assert rescue_rows >= 4  # the case exercises rescue-only blocks
    W1, l1 = O.rescue_weighted_attention(*args, sel["row_ptr"], sel["col_idx"], sel["flags"], 1.0, 128, 128)
    U, lu = O.masked_attention(*args, sel["row_ptr"], sel["col_idx"], 128, 128)
    np.testing.assert_allclose(W1, U, atol=1e-12)
    np.testing.assert_allclose(l1, lu, atol=1e-12)
    W0, l0 = O.rescue_weighted_attention(*args, sel["row_ptr"], sel["col_idx"], sel["flags"], 0.0, 128, 128)
    rp, ci = _filtered(sel, lambda f: bool(f & (O.FLAG_CENTROID | O.FLAG_FORCED)))
    G0, lg0 = O.masked_attention(*args, rp, ci, 128, 128)
    np.testing.assert_allclose(W0, G0, atol=1e-12)
    np.testing.assert_allclose(l0, lg0, atol=1e-12)
    assert not np.allclose(W0, U, atol=1e-6)


def test_rescue_weight_closed_form_two_keys():
    # one query token at position 1 sees key 0 (a rescue-only block) and key 1
    # (its forced diagonal block), blocks of one token: the output is the
    # two-term weighted softmax (e^{s1} v1 + g e^{s0} v0) / (e^{s1} + g e^{s0})
    rng = np.random.default_rng(32)
    d = 128
    Q = rng.standard_normal((1, 2, 1, d))
    K = rng.standard_normal((1, 2, 1, d))
    V = rng.standard_normal((1, 2, 1, d))
    rp = np.array([0, 1, 3])
    ci = np.array([0, 0, 1])
    fl = np.array([O.FLAG_FORCED, O.FLAG_RESCUE, O.FLAG_FORCED], dtype=np.uint8)
    for g in (0.0, 0.3, 1.0, 7.5):
        W, lse = O.rescue_weighted_attention(Q, K, V, rp, ci, fl, g, 1, 1)
        s0 = float(Q[0, 1, 0] @ K[0, 0, 0]) / math.sqrt(d)
        s1 = float(Q[0, 1, 0] @ K[0, 1, 0]) / math.sqrt(d)
        z = math.exp(s1) + g * math.exp(s0)
        want = (math.exp(s1) * V[0, 1, 0] + g * math.exp(s0) * V[0, 0, 0]) / z
        np.testing.assert_allclose(W[0, 1, 0], want, rtol=1e-12, atol=1e-13)
        assert lse[0, 0, 1] == pytest.approx(math.log(z), abs=1e-12)
        np.testing.assert_allclose(W[0, 0, 0], V[0, 0, 0], atol=1e-15)  # row 0: its diagonal key only


def test_rescue_weight_large_limit_is_rescue_only_attention():
    inp, sel = _weighted_case(seed=33)
    args = (inp["Q"], inp["K"], inp["V"])
    rp, ci = _filtered(sel, lambda f: f == O.FLAG_RESCUE)
    Wb, _ = O.rescue_weighted_attention(*args, sel["row_ptr"], sel["col_idx"], sel["flags"], 1e30, 128, 128)
    Rb, lrb = O.masked_attention(*args, rp, ci, 128, 128)
    nqb = 8
    for row in range(rp.size - 1):
        if rp[row + 1] == rp[row]:
            continue
        hq, i = divmod(row, nqb)
        t = slice(i * 128, (i + 1) * 128)
        np.testing.assert_allclose(Wb[0, t, hq], Rb[0, t, hq], atol=1e-9)


def test_rescue_weight_pins_catch_planted_mistakes(monkeypatch):
    good = O.split_regular_rescue

    def forced_as_rescue(row_ptr, col_idx, flags):
        # a forced block that the rescue branch also kept treated as rescue
        fl = [O.FLAG_RESCUE if (int(f) & O.FLAG_RESCUE and not int(f) & O.FLAG_CENTROID) else int(f) for f in flags]
        return good(row_ptr, col_idx, fl)
    monkeypatch.setattr(O, "split_regular_rescue", forced_as_rescue)
    with pytest.raises(AssertionError):
        test_rescue_weight_closed_form_two_keys_forced_and_rescue()
    monkeypatch.setattr(O, "split_regular_rescue", good)

    def swapped(row_ptr, col_idx, flags):  # the weight lands on the regular partial instead
        reg_p, reg_i, res_p, res_i = good(row_ptr, col_idx, flags)
        return res_p, res_i, reg_p, reg_i
    monkeypatch.setattr(O, "split_regular_rescue", swapped)
    with pytest.raises(AssertionError):
        test_rescue_weight_closed_form_two_keys()


def test_rescue_weight_closed_form_two_keys_forced_and_rescue():
    # a block both forced and kept by the rescue branch is regular: its weight
    # does not depend on gamma
    rng = np.random.default_rng(34)
    d = 128
    Q = rng.standard_normal((1, 2, 1, d))
    K = rng.standard_normal((1, 2, 1, d))
    V = rng.standard_normal((1, 2, 1, d))
    rp = np.array([0, 1, 3])
    ci = np.array([0, 0, 1])
    fl = np.array([O.FLAG_FORCED, O.FLAG_RESCUE, O.FLAG_FORCED | O.FLAG_RESCUE], dtype=np.uint8)
    a, _ = O.rescue_weighted_attention(Q, K, V, rp, ci, fl, 0.25, 1, 1)
    s0 = float(Q[0, 1, 0] @ K[0, 0, 0]) / math.sqrt(d)
    s1 = float(Q[0, 1, 0] @ K[0, 1, 0]) / math.sqrt(d)
    want = (math.exp(s1) * V[0, 1, 0] + 0.25 * math.exp(s0) * V[0, 0, 0]) / (math.exp(s1) + 0.25 * math.exp(s0))
    np.testing.assert_allclose(a[0, 1, 0], want, rtol=1e-12, atol=1e-13)


# --------------------------------------------------------------------------
# Sequence lengths that are not block multiples: the last block is shorter


def test_partial_last_key_block_closed_form():
    # 2 full blocks of 64 plus a last block of 3 keys {x, x, y}:
    # c = (2x + y) / 3 and r = |y - c| = (2/3) |x - y|
    rng = np.random.default_rng(41)
    d, bk = 128, 64
    x, y = rng.standard_normal((2, d))
    K = rng.standard_normal((1, 2 * bk + 3, 1, d))
    K[0, 2 * bk:2 * bk + 2, 0] = x
    K[0, 2 * bk + 2, 0] = y
    C, R = O.block_stats(K, bk)
    assert C.shape == (1, 1, 3, d) and R.shape == (1, 1, 3)
    np.testing.assert_allclose(C[0, 0, 2], (2 * x + y) / 3, atol=1e-14)
    assert R[0, 0, 2] == pytest.approx(2 / 3 * np.linalg.norm(x - y), rel=1e-13)
    full, _ = O.block_stats(K[:, :2 * bk], bk)  # the full blocks are unaffected by the tail
    np.testing.assert_array_equal(C[0, 0, :2], full[0, 0])
    Kone = K[:, :2 * bk + 1]  # a last block of a single key: c = k, r = 0
    C1, R1 = O.block_stats(Kone, bk)
    np.testing.assert_array_equal(C1[0, 0, 2], Kone[0, 2 * bk, 0])
    assert R1[0, 0, 2] == 0.0


def test_partial_last_query_block_is_numpy_mean():
    rng = np.random.default_rng(42)
    Q = rng.standard_normal((2, 300, 3, 128))
    qbar, qnorm = O.pooled_queries(Q, 128)
    assert qbar.shape == (2, 3, 3, 128)
    np.testing.assert_allclose(qbar[1, 2, 2], Q[1, 256:300, 2].mean(axis=0), atol=1e-15)
    np.testing.assert_allclose(qbar[0, 1, 0], Q[0, 0:128, 1].mean(axis=0), atol=1e-15)
    np.testing.assert_allclose(qnorm, np.linalg.norm(qbar, axis=-1), atol=1e-15)


def test_ragged_full_lists_equal_dense_attention():
    # 1000 query and key tokens in 128-token blocks (the last holds 104):
    # full causal lists give textbook causal attention; non-causal full lists
    # give plain softmax attention over all 1000 keys (torch SDPA, no mask)
    rng = np.random.default_rng(43)
    L, d = 1000, 128
    Q, K, V = (rng.standard_normal((1, L, h, d)) for h in (4, 2, 2))
    nqb = 8
    rp, ci = O.causal_full_lists(1, 4, nqb)
    Om, lm = O.masked_attention(Q, K, V, rp, ci, 128, 128)
    Od = O.dense_causal_attention(Q, K, V)
    np.testing.assert_allclose(Om, Od, atol=1e-12)
    rpn = np.arange(0, 4 * nqb * nqb + 1, nqb)
    cin = np.tile(np.arange(nqb), 4 * nqb)
    On, _ = O.masked_attention(Q, K, V, rpn, cin, 128, 128, causal=0)
    t = lambda a: torch.from_numpy(a).permute(0, 2, 1, 3)
    ref = torch.nn.functional.scaled_dot_product_attention(t(Q), t(K).repeat_interleave(2, 1),
                                                           t(V).repeat_interleave(2, 1)).permute(0, 2, 1, 3).numpy()
    np.testing.assert_allclose(On, ref, atol=1e-12)


def test_ragged_pins_catch_planted_mistakes(monkeypatch):
    good = O.block_stats

    def full_block_divisor(K, bk):
        C, R = good(K, bk)
        L = K.shape[1]
        nb = L - (C.shape[2] - 1) * bk
        if nb < bk:  # the tail's sum divided by block_k instead of n_b
            C = C.copy()
            C[:, :, -1] *= nb / bk
        return C, R
    monkeypatch.setattr(O, "block_stats", full_block_divisor)
    with pytest.raises(AssertionError):
        test_partial_last_key_block_closed_form()


# --------------------------------------------------------------------------
# Per-token-max query scoring (query_pool = 1)


def test_token_max_brute_force_tiny():
    # pure-Python loops over tokens, blocks and dims on a tiny case (7 tokens,
    # 3-token query blocks: the last holds one token)
    rng = np.random.default_rng(51)
    L, d, nkb = 7, 5, 3
    Q = rng.standard_normal((L, d))
    C = rng.standard_normal((nkb, d))
    R = rng.uniform(0.5, 2.0, nkb)
    beta = rng.uniform(0.0, 1.0, nkb)
    s_c, s_r = O.token_max_scores(Q, C, R, beta, 3)
    for i, toks in enumerate(([0, 1, 2], [3, 4, 5], [6])):
        for j in range(nkb):
            dots = [sum(Q[t, e] * C[j, e] for e in range(d)) for t in toks]
            norms = [math.sqrt(sum(Q[t, e] ** 2 for e in range(d))) for t in toks]
            assert s_c[i, j] == pytest.approx(max(dots), abs=1e-12)
            assert s_r[i, j] == pytest.approx(max(x + n * R[j] * beta[j] for x, n in zip(dots, norms)), abs=1e-12)


def test_token_max_equals_mean_when_a_block_repeats_one_query():
    # every query block made of one repeated query: max over its tokens = its
    # mean, so both representatives give the same scores and lists
    inp = make_mixture(L=2048, Hq=4, Hkv=2, block=128, seed=52)
    Q = inp["Q"].copy()
    Q[:] = np.repeat(Q[:, ::128], 128, axis=1)
    C, R = O.block_stats(inp["K"], 128)
    kw = dict(block_q=128, block_k=128, rho_centroid=0.2, rho_rescue=0.2)
    a = O.select_blocks(Q, C, R, O.SelectParams(**kw), keep_scores=True)
    b = O.select_blocks(Q, C, R, O.SelectParams(query_pool=1, **kw), keep_scores=True)
    for key in ("row_ptr", "col_idx", "flags"):
        assert np.array_equal(a[key], b[key])
    for hk in a["scores"]:
        np.testing.assert_allclose(a["scores"][hk][0], b["scores"][hk][0], atol=1e-12)
        np.testing.assert_allclose(a["scores"][hk][1], b["scores"][hk][1], atol=1e-12)


def test_token_max_bounds():
    # the best token beats the mean query (the dot is linear in q), the rescue
    # score bounds the centroid score, and with beta = 1 the rescue score bounds
    # every (token, key) logit of the pair (Cauchy-Schwarz per token, [RBS-en]
    # "The Fix")
    inp = make_tiny(L=1024, seed=53)
    C, R = O.block_stats(inp["K"], 64)
    p = O.SelectParams(block_q=64, block_k=64, beta_mode=1, beta_const=1.0, query_pool=1)
    beta, _ = O.rescue_beta(R, p)
    Qf = O.as_f64(inp["Q"])
    Kf = O.as_f64(inp["K"])
    qbar, qnorm = O.pooled_queries(inp["Q"], 64)
    for hq in range(2):
        s_c, s_r = O.token_max_scores(inp["Q"][0, :, hq], C[0, 0], R[0, 0], beta[0, 0], 64)
        m_c, _ = O.branch_scores(qbar[0, hq], qnorm[0, hq], C[0, 0], R[0, 0], beta[0, 0])
        assert np.all(s_c >= m_c - 1e-12) and np.all(s_r >= s_c)
        for i in (3, 9, 15):
            for j in (0, 5, 15):
                logits = Qf[0, i * 64:(i + 1) * 64, hq] @ Kf[0, j * 64:(j + 1) * 64, 0].T
                assert logits.max() <= s_r[i, j] + 1e-9


def test_token_max_pins_catch_planted_mistakes(monkeypatch):
    good = O.token_max_scores

    def mean_not_max(Qbh, C, R, beta, block_q):
        L = Qbh.shape[0]
        nqb = -(-L // block_q)
        q = O.as_f64(Qbh)
        s_c = np.stack([(q[i * block_q:(i + 1) * block_q] @ C.T).mean(axis=0) for i in range(nqb)])
        return s_c, good(Qbh, C, R, beta, block_q)[1]
    monkeypatch.setattr(O, "token_max_scores", mean_not_max)
    with pytest.raises(AssertionError):
        test_token_max_brute_force_tiny()

    def norm_of_mean(Qbh, C, R, beta, block_q):  # rescue term with |qbar| instead of |q_t|
        s_c, _ = good(Qbh, C, R, beta, block_q)
        L = Qbh.shape[0]
        q = O.as_f64(Qbh)
        nqb = -(-L // block_q)
        s_r = np.stack([((q[i * block_q:(i + 1) * block_q] @ C.T)
                         + np.linalg.norm(q[i * block_q:(i + 1) * block_q].mean(axis=0)) * (R * beta)).max(axis=0)
                        for i in range(nqb)])
        return s_c, s_r
    monkeypatch.setattr(O, "token_max_scores", norm_of_mean)
    with pytest.raises(AssertionError):
        test_token_max_bounds()


# --------------------------------------------------------------------------
# Block-attention with passage boundaries inside blocks: the token-level mask


def _token_mask_golden():
    g = {"list": {}, "mask": {}}
    for line in open(os.path.join(GOLDEN, "block_attention_token_mask_tiny.txt")):
        line = line.strip()
        if not line or line.startswith("#"):
            continue
        if line.startswith("key_start:"):
            g["key_start"] = [int(x) for x in line.split(":")[1].split()]
            continue
        kind, rest = line.split(" ", 1)
        idx, val = rest.split(":")
        g[kind][int(idx)] = val.split() if kind == "list" else val.strip()
    return g


def test_block_attention_token_mask_golden():
    g = _token_mask_golden()
    seg, final = [0, 6, 9], 13
    assert O.block_attention_key_start(seg, final, range(16)).tolist() == g["key_start"]
    rp, ci = O.block_attention_lists(seg, final, 4, 1, 1, 0, 4)
    for i in range(4):
        assert ci[rp[i]:rp[i + 1]].tolist() == [int(x) for x in g["list"][i]]
    # masked_attention on those lists with the token bound equals a direct
    # softmax over the hand-enumerated visibility matrix
    rng = np.random.default_rng(41)
    q = rng.standard_normal((1, 16, 2, 128))
    k = rng.standard_normal((1, 16, 1, 128))
    v = rng.standard_normal((1, 16, 1, 128))
    got, _ = O.masked_attention(q, k, v, np.concatenate([rp, rp[-1] + rp[1:]]), np.concatenate([ci, ci]), 4, 4,
                                key_start=g["key_start"])
    vis = np.array([[c == "1" for c in g["mask"][t]] for t in range(16)])
    for h in range(2):
        s = (q[0, :, h] @ k[0, :, 0].T) / math.sqrt(128)
        s = np.where(vis, s, -np.inf)
        w = np.exp(s - s.max(axis=1, keepdims=True))
        ref = (w / w.sum(axis=1, keepdims=True)) @ v[0, :, 0]
        np.testing.assert_allclose(got[0, :, h], ref, rtol=1e-12, atol=1e-12)


def test_ragged_passages_are_independent_and_need_the_token_mask():
    # passages of 100, 37 and 91 tokens and a 29-token final block, 32-token
    # blocks: every passage boundary falls inside a key block
    lens, blk = [100, 37, 91], 32
    inp = make_block_attention(final_len=29, Hq=2, Hkv=1, block=blk, seed=42, passage_lens=lens)
    other = make_block_attention(final_len=29, Hq=2, Hkv=1, block=blk, seed=43, passage_lens=lens)
    seg, final = inp["seg_start"], inp["final_start"]
    L = inp["Q"].shape[1]
    nqb = -(-L // blk)
    rp, ci = O.block_attention_lists(seg, final, blk, 1, 2, 0, nqb)
    ks = O.block_attention_key_start(seg, final, range(L))
    base, _ = O.masked_attention(inp["Q"], inp["K"], inp["V"], rp, ci, blk, blk, key_start=ks)
    a, e = 100, 137  # passage 1
    Q2, K2, V2 = other["Q"].copy(), other["K"].copy(), other["V"].copy()
    Q2[:, a:e], K2[:, a:e], V2[:, a:e] = inp["Q"][:, a:e], inp["K"][:, a:e], inp["V"][:, a:e]
    out2, _ = O.masked_attention(Q2, K2, V2, rp, ci, blk, blk, key_start=ks)
    assert np.array_equal(base[:, a:e], out2[:, a:e])  # passage 1 unchanged, bit for bit
    assert not np.allclose(base[:, final:], out2[:, final:])  # the final block sees everything
    # a plausible mistake -- the block lists without the token bound -- lets
    # passage 1 see the keys of passage 0 that share its first key block
    bad, _ = O.masked_attention(inp["Q"], inp["K"], inp["V"], rp, ci, blk, blk)
    bad2, _ = O.masked_attention(Q2, K2, V2, rp, ci, blk, blk)
    assert not np.allclose(bad[:, a:e], bad2[:, a:e])
    # block-aligned passages give the same lists with or without the bound
    rp0, ci0 = O.block_attention_lists([0, 64], 128, blk, 1, 1, 0, 5)
    assert ci0.tolist() == [0, 0, 1, 2, 2, 3, 0, 1, 2, 3, 4]


def test_mixture_generator_fills_a_ragged_tail():
    # a prompt that is not a block multiple gets a last, shorter key block of
    # real values (no uninitialised memory), and a block-multiple prompt is the
    # same whether or not a longer tail exists elsewhere
    rag = make_mixture(L=2048 + 77, Hq=4, Hkv=2, block=128, seed=61)
    k = O.bf16_to_f64(rag["K"])
    assert np.all(np.isfinite(k)) and np.abs(k).max() < 100.0
    assert all(q_tok < 2048 + 77 for (_, _, _, _, _, q_tok) in rag["plants"])
    a = make_mixture(L=2048, Hq=4, Hkv=2, block=128, seed=62)
    b = make_mixture(L=2048, Hq=4, Hkv=2, block=128, seed=62)
    assert np.array_equal(a["K"], b["K"]) and np.array_equal(a["Q"], b["Q"])
