"""The Python binding's argument checks (no GPU): buffers the kernels would
write or read past their end, or host tensors where device pointers are
needed, are refused before anything reaches the C ABI."""

import pytest
import torch

import block_sparse_long_rbs_b200 as rbs


def test_lists_refuse_host_and_short_buffers():
    rp = torch.zeros(9, dtype=torch.int32)
    ci = torch.zeros(4, dtype=torch.int32)
    with pytest.raises(TypeError, match="CUDA"):
        rbs.BlockLists(rp, ci, None, 8).c()
    with pytest.raises(ValueError, match="lists.row_ptr"):
        rbs.BlockLists(rp[:8], ci, None, 8).c()  # row_ptr needs num_rows + 1 entries
    with pytest.raises(ValueError, match="lists.flags"):
        rbs.BlockLists(rp, ci, torch.zeros(3, dtype=torch.uint8), 8).c()  # flags shorter than col_idx


def test_select_refuses_mismatched_stats_before_any_call():
    Q = torch.zeros(1, 512, 4, 128, dtype=torch.bfloat16)
    p = rbs.SelectParams(block_q=128, block_k=128)
    C = torch.zeros(1, 2, 4, 128)
    R = torch.zeros(1, 2, 4)
    with pytest.raises(ValueError, match="centroids"):
        rbs.rbs_select(Q, torch.zeros(2, 2, 4, 128), R, p)  # batch differs from Q's
    with pytest.raises(ValueError, match="centroids"):
        rbs.rbs_select(Q, torch.zeros(1, 2, 4, 64), R, p)  # head_dim differs from Q's
    with pytest.raises(ValueError, match="radii"):
        rbs.rbs_select(Q, C, torch.zeros(1, 2, 5), p)
    with pytest.raises(ValueError, match="beta_out"):
        rbs.rbs_select(Q, C, R, p, beta_out=torch.zeros(1, 2, 3))
    with pytest.raises(TypeError, match="centroids"):
        rbs.rbs_select(Q, C, R, p)  # shapes right, but host tensors


def test_tensors_of_one_call_must_share_a_device():
    # the library launches on the current device: a tensor on another GPU is
    # refused before its pointer can reach a kernel (fake device attributes:
    # no GPU is needed to check the rule)
    from types import SimpleNamespace
    d0, d1 = torch.device("cuda", 0), torch.device("cuda", 1)
    Q = SimpleNamespace(device=d0)
    assert rbs._one_device("Q", Q, K=SimpleNamespace(device=d0), lse=None) == d0
    with pytest.raises(ValueError, match="K is on cuda:1 but Q is on cuda:0"):
        rbs._one_device("Q", Q, K=SimpleNamespace(device=d1))
    lists = SimpleNamespace(row_ptr=SimpleNamespace(device=d0), col_idx=SimpleNamespace(device=d1), flags=None)
    with pytest.raises(ValueError, match="lists.col_idx"):
        rbs._one_device("Q", Q, **rbs._lists_tensors(lists))
