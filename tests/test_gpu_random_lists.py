"""GPU parity of block-sparse attention on random lists that exercise the
cases a fixed selection rarely produces: overlapping lists of neighbouring
heads, 3 q heads per KV head, an odd number of rows, empty rows between full
ones, MHA with 5 heads, KV-group lists (one list per KV head), rows of very
different lengths next to each other, and every row empty; each against the
fp64 oracle (outputs and log-sum-exps)."""

import numpy as np
import pytest
import torch

import block_sparse_long_rbs_b200 as rbs
from helpers import dev, lists_np, o_rows_close
from oracle import rbs_oracle as O
from workloads import make_mixture

pytestmark = pytest.mark.gpu


def _random_lists(rows, nqb, rng, p_keep, p_empty=0.0):
    """Causal lists: each visible block kept with probability p_keep, the
    diagonal always (unless the row is made empty)."""
    out = []
    for r in range(rows):
        i = r % nqb
        if rng.random() < p_empty:
            out.append([])
            continue
        keep = [j for j in range(i) if rng.random() < p_keep] + [i]
        out.append(keep)
    rp = np.concatenate([[0], np.cumsum([len(x) for x in out])]).astype(np.int32)
    ci = np.array(sum(out, []), dtype=np.int32)
    return rp, ci


def _check(inp, rp, ci, block=128):
    lists = rbs.BlockLists(torch.from_numpy(rp).cuda(), torch.from_numpy(ci if ci.size else np.zeros(1, np.int32)).cuda(),
                           None, rp.size - 1)
    out, lse = rbs.bsa_prefill(dev(inp["Q"]), dev(inp["K"]), dev(inp["V"]), lists, block, block, return_lse=True)
    torch.cuda.synchronize()
    assert rbs.rbs_get_device_error() == 0
    Oo, Lo = O.masked_attention(inp["Q"], inp["K"], inp["V"], rp.astype(np.int64), ci.astype(np.int64), block, block)
    Hq = inp["Q"].shape[2]
    nqb = -(-inp["Q"].shape[1] // block)
    if rp.size - 1 == inp["Q"].shape[0] * Hq * nqb:
        o_rows_close(out, Oo, range(rp.size - 1), Hq, nqb, block)
    else:  # KV-group lists: compare every q head's rows
        o_rows_close(out, Oo, range(inp["Q"].shape[0] * Hq * nqb), Hq, nqb, block)
    lg = lse.cpu().numpy()
    np.testing.assert_allclose(lg, Lo, atol=1e-3)


@pytest.mark.parametrize("Hq,Hkv,p_keep,p_empty,seed", [
    (8, 2, 0.4, 0.0, 701),   # neighbouring q heads of one KV head, overlapping lists
    (6, 2, 0.3, 0.0, 702),   # 3 q heads per KV head
    (3, 1, 0.5, 0.2, 703),   # odd rows per prompt, empty rows in between
    (5, 5, 0.6, 0.1, 704),   # MHA, 5 heads, odd total
])
def test_random_lists(cuda_ok, Hq, Hkv, p_keep, p_empty, seed):
    inp = make_mixture(L=2048 + 77, Hq=Hq, Hkv=Hkv, block=128, seed=seed)
    nqb = -(-inp["Q"].shape[1] // 128)
    rng = np.random.default_rng(seed)
    rp, ci = _random_lists(Hq * nqb, nqb, rng, p_keep, p_empty)
    _check(inp, rp, ci)


def test_rows_of_very_different_lengths(cuda_ok):
    # row lengths alternate between 1 and every visible block
    inp = make_mixture(L=4096, Hq=4, Hkv=1, block=128, seed=705)
    nqb = 32
    rows = []
    for h in range(4):
        for i in range(nqb):
            rows.append(list(range(i + 1)) if (h + i) % 2 else [i])
    rp = np.concatenate([[0], np.cumsum([len(x) for x in rows])]).astype(np.int32)
    ci = np.array(sum(rows, []), dtype=np.int32)
    _check(inp, rp, ci)


def test_random_kv_group_lists(cuda_ok):
    # one list per KV head, shared by its q heads
    inp = make_mixture(L=4096, Hq=8, Hkv=2, block=128, seed=706)
    nqb = 32
    rng = np.random.default_rng(706)
    rp, ci = _random_lists(2 * nqb, nqb, rng, 0.3)
    _check(inp, rp, ci)


def test_all_rows_empty(cuda_ok):
    inp = make_mixture(L=1024, Hq=4, Hkv=2, block=128, seed=707)
    rp = np.zeros(4 * 8 + 1, dtype=np.int32)
    lists = rbs.BlockLists(torch.from_numpy(rp).cuda(), torch.zeros(1, dtype=torch.int32, device="cuda"), None, 32)
    out, lse = rbs.bsa_prefill(dev(inp["Q"]), dev(inp["K"]), dev(inp["V"]), lists, 128, 128, return_lse=True)
    torch.cuda.synchronize()
    assert rbs.rbs_get_device_error() == 0
    assert torch.all(out == 0) and torch.all(torch.isneginf(lse))
