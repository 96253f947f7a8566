"""Shared test helpers: moving seeded inputs to the GPU and comparing the
GPU path's outputs with the oracle's."""

from __future__ import annotations

import numpy as np
import torch

from oracle import rbs_oracle as O

# Tolerances (what the attention and selection paths are held to)
TOL_STATS_REL = 1e-3  # centroid (relative L2 per vector) and radius (relative)
TOL_O_ABS = 2e-2  # attention output, max abs, oracle run on the GPU's lists
TOL_NEAR_TAU = 1e-3  # a block whose score is within 1e-3*max(1,|tau|) of its branch threshold


def dev(bits: np.ndarray) -> torch.Tensor:
    """bf16 bit patterns (uint16 numpy) -> bf16 CUDA tensor with the same bytes."""
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).cuda()


def host_bits(t: torch.Tensor) -> np.ndarray:
    return t.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16)


def lists_np(lists):
    rp = lists.row_ptr.cpu().numpy().astype(np.int64)
    nnz = int(rp[-1])
    ci = lists.col_idx[:nnz].cpu().numpy().astype(np.int64)
    fl = lists.flags[:nnz].cpu().numpy() if lists.flags is not None else None
    return rp, ci, fl


def dense_masks(rp, ci, fl, nkb):
    rows = rp.size - 1
    union = np.zeros((rows, nkb), dtype=bool)
    cen = np.zeros((rows, nkb), dtype=bool)
    res = np.zeros((rows, nkb), dtype=bool)
    r_of = np.repeat(np.arange(rows), np.diff(rp))
    union[r_of, ci] = True
    if fl is not None:
        cen[r_of, ci] = (fl & O.FLAG_CENTROID) > 0
        res[r_of, ci] = (fl & O.FLAG_RESCUE) > 0
    return union, cen, res


def compare_selection(gpu_lists, ora: dict, Hq: int, nqb: int, nkb: int, exact_k: bool = True) -> dict:
    """Per-branch comparison with the near-threshold rule; returns counts, raises on a real mismatch.

    exact_k: each GPU branch keeps exactly the oracle's k_i (top-k mode); in
    the max-relative mode the count follows the excused blocks instead."""
    grp, gci, gfl = lists_np(gpu_lists)
    assert np.all(np.diff(grp) >= 0)
    for r in range(grp.size - 1):  # ascending, in range
        row = gci[grp[r]:grp[r + 1]]
        assert np.all(np.diff(row) > 0) and (row.size == 0 or (row[0] >= 0 and row[-1] < nkb))
    assert np.all(gfl != 0)
    gu, gc, gr = dense_masks(grp, gci, gfl, nkb)
    ou, oc, orr = dense_masks(ora["row_ptr"], ora["col_idx"], ora["flags"], nkb)
    rows = grp.size - 1
    excused = {"centroid": 0, "rescue": 0}
    for name, gm, om, bi in (("centroid", gc, oc, 0), ("rescue", gr, orr, 1)):
        diff_r, diff_j = np.nonzero(gm != om)
        for r, j in zip(diff_r, diff_j):
            b, rem = divmod(int(r), Hq * nqb)
            hq, i = divmod(rem, nqb)
            s = ora["scores"][(b, hq)][bi][i, j]
            tau = ora["tau"][b, hq, i, bi]
            if abs(s - tau) > TOL_NEAR_TAU * max(1.0, abs(tau)):
                raise AssertionError(f"{name} branch: row {r} (b={b}, h={hq}, i={i}) block {j}: gpu={gm[r, j]} "
                                     f"oracle={om[r, j]} score={s:.6f} tau={tau:.6f}")
            excused[name] += 1
        # each GPU branch keeps exactly k_i blocks
        if exact_k:
            assert np.array_equal(gm.sum(axis=1), ora["k"].reshape(rows, 2)[:, bi])
    # union = branches + forced: GPU entries flagged forced must be forced in the oracle too
    gforced = np.zeros_like(gu)
    r_of = np.repeat(np.arange(rows), np.diff(grp))
    gforced[r_of, gci] = (gfl & O.FLAG_FORCED) > 0
    oforced = np.zeros_like(ou)
    r_of_o = np.repeat(np.arange(rows), np.diff(ora["row_ptr"]))
    oforced[r_of_o, ora["col_idx"]] = (ora["flags"] & O.FLAG_FORCED) > 0
    assert np.array_equal(gforced, oforced)
    assert np.array_equal(gu, gc | gr | gforced)
    excused["rows"] = rows
    excused["nnz_gpu"] = int(grp[-1])
    excused["nnz_oracle"] = int(ora["row_ptr"][-1])
    return excused


def o_rows_close(O_gpu: torch.Tensor, O_ref: np.ndarray, rows, Hq: int, nqb: int, block_q: int,
                 tol: float = TOL_O_ABS) -> float:
    """Max abs difference over the query tokens of the given rows; asserts <= tol."""
    og = O_gpu.float().cpu().numpy()
    worst = 0.0
    for row in rows:
        b, rem = divmod(int(row), Hq * nqb)
        hq, i = divmod(rem, nqb)
        sl = slice(i * block_q, (i + 1) * block_q)
        a, r = og[b, sl, hq], O_ref[b, sl, hq]
        # a NaN on either side is a failure, not a silently skipped comparison
        assert np.all(np.isfinite(a)) and np.all(np.isfinite(r)), f"non-finite output in row {row}"
        worst = max(worst, float(np.abs(a - r).max()))
    assert worst <= tol, f"max |O_gpu - O_oracle| = {worst}"
    return worst
