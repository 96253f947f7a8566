"""GPU parity of the two-row attention schedule (the kernel runs rows in
pairs and walks their lists as one stream, loading a key block both rows
list once: "QUILT: Rethinking Sparse-Attention Prefill through Shared Query
Execution", Abstract).  Random lists exercise the cases the merge must get
right: pairs of rows of the same KV head with overlapping lists, pairs that
straddle KV heads or query blocks (3 q heads per KV head), an odd number of
rows (a last pair with one row), pairs with one empty row, identical lists
(KV-group lists), and rows of very different lengths."""

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
    (8, 2, 0.4, 0.0, 701),   # pairs of q heads of one KV head, overlapping lists
    (6, 2, 0.3, 0.0, 702),   # 3 q heads per KV head: pairs straddle KV heads / query blocks
    (3, 1, 0.5, 0.2, 703),   # odd rows per prompt, empty rows inside pairs
    (5, 5, 0.6, 0.1, 704),   # MHA, 5 heads: pairs of consecutive query blocks, odd total
])
def test_pairs_random_lists(cuda_ok, Hq, Hkv, p_keep, p_empty, seed):
    inp = make_mixture(L=2048 + 77, Hq=Hq, Hkv=Hkv, block=128, seed=seed)
    nqb = -(-inp["Q"].shape[1] // 128)
    rng = np.random.default_rng(seed)
    rp, ci = _random_lists(Hq * nqb, nqb, rng, p_keep, p_empty)
    _check(inp, rp, ci)


def test_pairs_very_different_lengths(cuda_ok):
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


def test_pairs_kv_group_lists(cuda_ok):
    # one list per KV head: every pair of q heads shares its whole list
    inp = make_mixture(L=4096, Hq=8, Hkv=2, block=128, seed=706)
    nqb = 32
    rng = np.random.default_rng(706)
    rp, ci = _random_lists(2 * nqb, nqb, rng, 0.3)
    _check(inp, rp, ci)


def test_pairs_all_rows_empty(cuda_ok):
    inp = make_mixture(L=1024, Hq=4, Hkv=2, block=128, seed=707)
    rp = np.zeros(4 * 8 + 1, dtype=np.int32)
    lists = rbs.BlockLists(torch.from_numpy(rp).cuda(), torch.zeros(1, dtype=torch.int32, device="cuda"), None, 32)
    out, lse = rbs.bsa_prefill(dev(inp["Q"]), dev(inp["K"]), dev(inp["V"]), lists, 128, 128, return_lse=True)
    torch.cuda.synchronize()
    assert rbs.rbs_get_device_error() == 0
    assert torch.all(out == 0) and torch.all(torch.isneginf(lse))
