"""The C-ABI library without a GPU: it loads, exports every entry point the
header declares, answers the host-only size queries, and rejects bad
arguments before touching CUDA."""

import ctypes
import os
import re

import numpy as np
import pytest

from block_sparse_long_rbs_b200 import _abi
from block_sparse_long_rbs_b200 import SelectParams, BlockLists  # noqa: F401
from oracle import rbs_oracle as O

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def L():
    from block_sparse_long_rbs_b200 import build
    build.build()
    return _abi.lib()


def _declared():
    names = []
    for h in os.listdir(os.path.join(ROOT, "include")):
        src = open(os.path.join(ROOT, "include", h)).read()
        names += re.findall(r"^RBS_API\s+[\w\s\*]+?\b(\w+)\(", src, flags=re.M)
    return names


def test_header_declares_the_pages_calls():
    names = set(_declared())
    for required in ("rbs_block_stats", "rbs_select", "bsa_prefill", "rope_reencode"):
        assert required in names


def test_every_declared_symbol_is_exported(L):
    names = _declared()
    assert len(names) >= 17
    for n in names:
        assert hasattr(L, n), n
    assert set(names) == set(_abi.SIGNATURES)


def test_housekeeping(L):
    assert L.rbs_abi_version() == 5
    assert L.rbs_status_string(0) == b"ok"
    assert L.rbs_status_string(3) == b"capacity"
    p = _abi.SelectParamsC()
    L.rbs_select_params_default(ctypes.byref(p))
    d = SelectParams()
    for f in _abi.SelectParamsC._fields_:
        assert getattr(p, f[0]) == pytest.approx(getattr(d, f[0]))


@pytest.mark.parametrize("rho,off,diag,sink", [(0.05, 0, 1, 0), (0.25, 0, 1, 1), (1.0, 3, 0, 0), (0.1, 0, 1, 0)])
def test_select_capacity_bounds_oracle_rows(L, rho, off, diag, sink):
    nqb, nkb = 40, 40 + off
    p = SelectParams(rho_centroid=rho, rho_rescue=rho, force_diag=diag, force_sink=sink, q_block_offset=off)
    cap = L.rbs_select_capacity(2, 3, nqb, nkb, ctypes.byref(p.c()))
    rho32 = float(np.float32(rho))
    expect = 0
    for i in range(nqb):
        n = min(nkb, i + off + 1)
        expect += min(n, 2 * O.keep_count(rho32, n) + diag + sink)
    assert cap == 6 * expect


def test_causal_full_nnz(L):
    for nqb, off in ((1, 0), (64, 0), (4, 256)):
        rp, ci = O.causal_full_lists(2, 3, nqb, off)
        assert L.rbs_lists_causal_full_nnz(2, 3, nqb, off) == ci.size


def test_block_attention_nnz_matches_oracle(L):
    seg = [0, 256, 1024, 1536]
    arr = (ctypes.c_int32 * 4)(*seg)
    for first, num in ((0, 13), (12, 1), (3, 9)):
        rp, ci = O.block_attention_lists(seg, 1536 + 128, 128, 2, 5, first, num)
        assert L.rbs_lists_block_attention_nnz(arr, 4, 1536 + 128, 128, 2, 5, first, num) == ci.size


def test_block_attention_rejects_bad_segments(L):
    desc = (ctypes.c_int32 * 2)(128, 256)  # does not start at 0
    assert L.rbs_lists_block_attention_nnz(desc, 2, 512, 128, 1, 1, 0, 4) == -1
    down = (ctypes.c_int32 * 3)(0, 300, 200)  # not ascending
    assert L.rbs_lists_block_attention_nnz(down, 3, 512, 128, 1, 1, 0, 4) == -1
    late = (ctypes.c_int32 * 2)(0, 600)  # final block before the last passage
    assert L.rbs_lists_block_attention_nnz(late, 2, 512, 128, 1, 1, 0, 6) == -1


def test_block_attention_nnz_with_ragged_passages(L):
    # passage starts at any token offset: the library's closed-form row
    # offsets equal the oracle builder's entry counts
    rng = np.random.default_rng(77)
    cases = [([0, 1999, 4099], 4616, 128), ([0, 100, 137], 228, 32), ([0, 6, 9], 13, 4)]
    for _ in range(20):
        n = int(rng.integers(1, 8))
        starts = np.concatenate([[0], np.sort(rng.choice(np.arange(1, 3000), n - 1, replace=False))]).tolist()
        cases.append((starts, starts[-1] + int(rng.integers(1, 700)), int(rng.choice([64, 128]))))
    for seg, final, blk in cases:
        if blk not in (64, 128):
            continue
        arr = (ctypes.c_int32 * len(seg))(*seg)
        nqb = -(-(final + 300) // blk)
        for first, num in ((0, nqb), (final // blk, nqb - final // blk), (1, max(1, nqb // 2))):
            rp, ci = O.block_attention_lists(seg, final, blk, 2, 3, first, num)
            assert L.rbs_lists_block_attention_nnz(arr, len(seg), final, blk, 2, 3, first, num) == ci.size


def _fake(B=1, Lq=256, H=2, D=128, sb=None, ss=None, sh=None, ptr=0x10000):
    sh = D if sh is None else sh
    ss = H * D if ss is None else ss
    sb = Lq * H * D if sb is None else sb
    return _abi.Bf16Tensor(ptr, B, Lq, H, D, sb, ss, sh)


def test_validation_before_any_launch(L):
    C = ctypes.c_void_p(0x20000)
    R = ctypes.c_void_p(0x30000)
    s = ctypes.c_void_p(0)
    null = _abi.Bf16Tensor()
    assert L.rbs_block_stats(ctypes.byref(null), 128, C, R, s) == 1
    assert L.rbs_block_stats(ctypes.byref(_fake(D=64)), 128, C, R, s) == 2
    assert L.rbs_block_stats(ctypes.byref(_fake()), 96, C, R, s) == 2
    # a length that is not a block multiple is taken (a last, shorter block):
    # past validation, so no GPU here
    assert L.rbs_block_stats(ctypes.byref(_fake(Lq=200)), 128, C, R, s) == 4
    assert L.rbs_block_stats(ctypes.byref(_fake(ptr=0x10002)), 128, C, R, s) == 1
    assert L.rbs_block_stats(ctypes.byref(_fake(ss=260)), 128, C, R, s) == 1
    assert b"strides" in L.rbs_last_error()
    # valid arguments on a machine without a GPU fail loudly with a CUDA status
    assert L.rbs_block_stats(ctypes.byref(_fake()), 128, C, R, s) == 4


def test_select_rejects_small_capacity_and_workspace(L):
    p = SelectParams(block_q=64, block_k=64)
    pc = p.c()
    q = _fake(Lq=512)
    rows = 1 * 2 * 8
    need = L.rbs_select_capacity(1, 2, 8, 8, ctypes.byref(pc))
    ws = L.rbs_select_workspace_bytes(1, 2, 8, 1, 8, ctypes.byref(pc))
    assert ws > 0
    small = _abi.BlockListsC(0x40000, 0x50000, None, need - 1, rows)
    st = L.rbs_select(ctypes.byref(q), 0x20000, 0x30000, 1, 8, ctypes.byref(pc), 0x60000, ws, ctypes.byref(small),
                      None, None)
    assert st == 3
    ok = _abi.BlockListsC(0x40000, 0x50000, None, need, rows)
    # a workspace below the full size still runs (the fused scoring kernel) ...
    st = L.rbs_select(ctypes.byref(q), 0x20000, 0x30000, 1, 8, ctypes.byref(pc), 0x60000, ws - 1, ctypes.byref(ok),
                      None, None)
    assert st == 4  # past validation: no GPU here
    # ... down to the masks and counts it needs
    st = L.rbs_select(ctypes.byref(q), 0x20000, 0x30000, 1, 8, ctypes.byref(pc), 0x60000, 256, ctypes.byref(ok),
                      None, None)
    assert st == 3
    wrong_rows = _abi.BlockListsC(0x40000, 0x50000, None, need, rows + 1)
    st = L.rbs_select(ctypes.byref(q), 0x20000, 0x30000, 1, 8, ctypes.byref(pc), 0x60000, ws, ctypes.byref(wrong_rows),
                      None, None)
    assert st == 1
    st = L.rbs_select(ctypes.byref(q), 0x20000, 0x30000, 3, 8, ctypes.byref(pc), 0x60000, ws, ctypes.byref(ok),
                      None, None)
    assert st == 1  # 2 q heads cannot share 3 KV heads


def test_bsa_prefill_validation(L):
    q = _fake(Lq=256, H=4)
    k = _fake(Lq=256, H=2)
    o = _fake(Lq=256, H=4)
    lists = _abi.BlockListsC(0x40000, 0x50000, None, 100, 1 * 4 * 2)
    s = ctypes.c_void_p(0)
    f = L.bsa_prefill
    assert f(ctypes.byref(q), ctypes.byref(k), ctypes.byref(k), ctypes.byref(lists), 128, 64, 0, 0.0, 1,
             ctypes.byref(o), None, s) == 2  # block_q != block_k
    assert f(ctypes.byref(q), ctypes.byref(k), ctypes.byref(k), ctypes.byref(lists), 128, 128, 64, 0.0, 1,
             ctypes.byref(o), None, s) == 2  # q_offset not a block multiple
    k3 = _fake(Lq=256, H=3)
    assert f(ctypes.byref(q), ctypes.byref(k3), ctypes.byref(k3), ctypes.byref(lists), 128, 128, 0, 0.0, 1,
             ctypes.byref(o), None, s) == 1
    bad_rows = _abi.BlockListsC(0x40000, 0x50000, None, 100, 7)
    assert f(ctypes.byref(q), ctypes.byref(k), ctypes.byref(k), ctypes.byref(bad_rows), 128, 128, 0, 0.0, 1,
             ctypes.byref(o), None, s) == 1


def test_rope_validation(L):
    x = _fake()
    s = ctypes.c_void_p(0)
    assert L.rope_reencode(ctypes.byref(x), ctypes.byref(_fake(Lq=128)), 0x1000, 0x2000, 5e5, 0, s) == 1
    assert L.rope_reencode(ctypes.byref(x), ctypes.byref(x), None, 0x2000, 5e5, 0, s) == 1
    assert L.rope_reencode(ctypes.byref(x), ctypes.byref(x), 0x1000, 0x2000, 5e5, 2, s) == 1
    assert L.rope_reencode(ctypes.byref(x), ctypes.byref(x), 0x1000, 0x2000, -1.0, 0, s) == 1


def test_max_relative_capacity_is_every_visible_block(L):
    p = SelectParams(threshold_mode=1, delta_centroid=1.0, delta_rescue=2.0)
    cap = L.rbs_select_capacity(1, 2, 16, 16, ctypes.byref(p.c()))
    assert cap == 2 * sum(i + 1 for i in range(16))


def test_select_rejects_bad_threshold_fields(L):
    q = _fake(Lq=512)
    rows = 1 * 2 * 8
    ok = _abi.BlockListsC(0x40000, 0x50000, None, 1 << 20, rows)
    for kw in ({"threshold_mode": 2}, {"threshold_mode": 1, "delta_centroid": -1.0},
               {"threshold_mode": 1, "delta_rescue": float("nan")}):
        pc = SelectParams(block_q=64, block_k=64, **kw).c()
        st = L.rbs_select(ctypes.byref(q), 0x20000, 0x30000, 1, 8, ctypes.byref(pc), 0x60000, 1 << 20,
                          ctypes.byref(ok), None, None)
        assert st == 1, kw
    # MAX_RELATIVE ignores rho (it may be zero)
    pc = SelectParams(block_q=64, block_k=64, rho_centroid=0.0, rho_rescue=0.0, threshold_mode=1,
                      delta_centroid=1.0, delta_rescue=1.0).c()
    st = L.rbs_select(ctypes.byref(q), 0x20000, 0x30000, 1, 8, ctypes.byref(pc), 0x60000, 1 << 20,
                      ctypes.byref(ok), None, None)
    assert st == 4  # past validation: no GPU here


def test_kv_group_lists_validation(L):
    """KV_GROUP lists have one row per (batch, KV head, query block); both entry
    points take exactly that row count in that mode (and reject others)."""
    s = ctypes.c_void_p(0)
    q = _fake(Lq=512, H=4)  # 4 q heads, 64-token blocks -> 8 query blocks
    group = _abi.BlockListsC(0x40000, 0x50000, None, 1 << 20, 1 * 2 * 8)  # 2 KV heads
    per_head = _abi.BlockListsC(0x40000, 0x50000, None, 1 << 20, 1 * 4 * 8)
    pc = SelectParams(block_q=64, block_k=64, list_mode=1).c()
    sel = lambda lists, p: L.rbs_select(ctypes.byref(q), 0x20000, 0x30000, 2, 8, ctypes.byref(p), 0x60000, 1 << 24,
                                        ctypes.byref(lists), None, None)
    assert sel(per_head, pc) == 1
    assert sel(group, pc) == 4  # past validation: no GPU here
    assert sel(group, SelectParams(block_q=64, block_k=64).c()) == 1  # per-head mode wants 32 rows
    assert sel(group, SelectParams(block_q=64, block_k=64, list_mode=2).c()) == 1
    # capacity of the per-head lists bounds the group unions: sum_g min(n, G x) <= G sum min(n, x)
    p1 = SelectParams(block_q=64, block_k=64, list_mode=1)
    assert L.rbs_select_capacity(1, 4, 8, 8, ctypes.byref(p1.c())) == L.rbs_select_capacity(
        1, 4, 8, 8, ctypes.byref(SelectParams(block_q=64, block_k=64).c()))
    k = _fake(Lq=512, H=2)
    o = _fake(Lq=512, H=4)
    f = L.bsa_prefill
    for lists in (group, per_head):
        assert f(ctypes.byref(q), ctypes.byref(k), ctypes.byref(k), ctypes.byref(lists), 64, 64, 0, 0.0, 1,
                 ctypes.byref(o), None, s) == 4  # both shapes pass validation
    odd = _abi.BlockListsC(0x40000, 0x50000, None, 1 << 20, 1 * 3 * 8)
    assert f(ctypes.byref(q), ctypes.byref(k), ctypes.byref(k), ctypes.byref(odd), 64, 64, 0, 0.0, 1,
             ctypes.byref(o), None, s) == 1


def test_rescue_weighted_validation(L):
    """bsa_prefill_rescue_weighted: the weight must be finite and >= 0, and
    any weight but 1 needs the lists' branch flags."""
    s = ctypes.c_void_p(0)
    q = _fake(Lq=256, H=4)
    k = _fake(Lq=256, H=2)
    o = _fake(Lq=256, H=4)
    flagged = _abi.BlockListsC(0x40000, 0x50000, 0x70000, 100, 1 * 4 * 2)
    bare = _abi.BlockListsC(0x40000, 0x50000, None, 100, 1 * 4 * 2)
    f = L.bsa_prefill_rescue_weighted
    call = lambda lists, w: f(ctypes.byref(q), ctypes.byref(k), ctypes.byref(k), ctypes.byref(lists), 128, 128, 0,
                              0.0, 1, w, ctypes.byref(o), None, s)
    for bad in (-1.0, float("nan"), float("inf")):
        assert call(flagged, bad) == 1, bad
    assert call(bare, 0.5) == 1  # no flags to tell the rescue blocks apart
    assert call(bare, 1.0) == 4  # weight 1 is bsa_prefill: past validation, no GPU here
    assert call(flagged, 0.0) == 4


def test_query_pool_validation(L):
    """query_pool TOKEN_MAX: a field value outside {0, 1} is rejected, and more
    key blocks than the per-token kernel holds are unsupported."""
    s = None
    q = _fake(Lq=512)
    rows = 1 * 2 * 8
    ok = _abi.BlockListsC(0x40000, 0x50000, None, 1 << 20, rows)
    sel = lambda p, nkb: L.rbs_select(ctypes.byref(q), 0x20000, 0x30000, 1, nkb, ctypes.byref(p), 0x60000, 1 << 26,
                                      ctypes.byref(ok), None, s)
    assert sel(SelectParams(block_q=64, block_k=64, query_pool=2).c(), 8) == 1
    assert sel(SelectParams(block_q=64, block_k=64, query_pool=1).c(), 8) == 4  # past validation
    assert sel(SelectParams(block_q=64, block_k=64, query_pool=1).c(), 4096) == 2
    # the per-token path's workspace includes the centroid parts
    p0 = SelectParams(block_q=64, block_k=64).c()
    p1 = SelectParams(block_q=64, block_k=64, query_pool=1).c()
    assert L.rbs_select_workspace_bytes(1, 2, 8, 1, 8, ctypes.byref(p1)) > 0
    assert L.rbs_select_workspace_bytes(1, 2, 8, 1, 8, ctypes.byref(p0)) > 0


def test_token_max_workspace_holds_the_key_matrix(L):
    """query_pool TOKEN_MAX: the full workspace adds both branches' key rows
    ([rows][2][nKB padded to 32] uint32) for the separate top-k kernel; a
    workspace one byte short still runs (the scoring kernel selects in
    place), one without room for the split centroids is refused."""
    p1 = SelectParams(block_q=64, block_k=64, query_pool=1).c()
    nkb = 64
    small = L.rbs_select_workspace_bytes(1, 2, 8, 1, nkb, ctypes.byref(p1))
    large = L.rbs_select_workspace_bytes(1, 2, 16, 1, nkb, ctypes.byref(p1))
    extra_rows = 1 * 2 * 8
    # at least the extra rows' key rows (2 x 4 B per block); the smaller
    # regions are rounded up to 256 bytes
    assert large - small >= extra_rows * 2 * nkb * 4
    q = _fake(Lq=512)
    rows = 1 * 2 * 8
    ok = _abi.BlockListsC(0x40000, 0x50000, None, 1 << 20, rows)
    sel = lambda ws: L.rbs_select(ctypes.byref(q), 0x20000, 0x30000, 1, 8, ctypes.byref(p1), 0x60000, ws,
                                  ctypes.byref(ok), None, None)
    full = L.rbs_select_workspace_bytes(1, 2, 8, 1, 8, ctypes.byref(p1))
    assert sel(full) == 4  # past validation: no GPU here
    assert sel(full - 1) == 4
    assert sel(256) == 3
