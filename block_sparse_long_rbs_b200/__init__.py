"""Block-sparse prefill attention with radius-bounded block selection (RBS)
and the Block-attention mask, on NVIDIA B200 (sm_100a).

A thin binding over the C ABI of librbs (include/rbs.h): argument
marshalling only.  Torch tensors supply device memory and the current CUDA
stream; every step of the computation runs in the library's CUDA kernels.
Functions carry the same names as the C entry points.
"""

from __future__ import annotations

import ctypes
import dataclasses
import math

import torch

from ._abi import (  # noqa: F401
    DEVERR_BLOCK_INDEX,
    DEVERR_NONCAUSAL,
    DEVERR_ROW_PTR,
    DEVERR_TIMEOUT,
    MAX_KV_BLOCKS,
    BlockListsC,
    Bf16Tensor,
    RbsError,
    SelectParamsC,
    check,
    lib,
)

__all__ = [
    "SelectParams", "BlockLists", "rbs_block_stats", "rbs_block_beta", "rbs_pool_queries", "rbs_select",
    "rbs_select_capacity", "rbs_select_workspace_bytes", "rbs_lists_causal_full", "rbs_lists_block_attention",
    "bsa_prefill", "bsa_prefill_rescue_weighted", "bsa_prefill_segments", "rope_reencode", "rbs_get_device_error",
    "RbsError",
]


@dataclasses.dataclass
class SelectParams:
    """Selection parameters (field meanings and defaults as in include/rbs.h)."""

    block_q: int = 128
    block_k: int = 128
    rho_centroid: float = 0.05
    rho_rescue: float = 0.05
    beta_mode: int = 0
    beta_const: float = 1.0
    beta_p_lo: float = 0.0
    beta_p_hi: float = 1.0
    force_diag: int = 1
    force_sink: int = 0
    causal: int = 1
    q_block_offset: int = 0
    threshold_mode: int = 0  # 0 = top-k fraction, 1 = within delta of the row maximum
    delta_centroid: float = 0.0
    delta_rescue: float = 0.0
    list_mode: int = 0  # 0 = one list per q head, 1 = one per KV head (union of its q heads)
    query_pool: int = 0  # 0 = mean query of the block, 1 = best query token of the block

    def c(self) -> SelectParamsC:
        return SelectParamsC(*[getattr(self, f.name) for f in dataclasses.fields(self)])


@dataclasses.dataclass
class BlockLists:
    """CSR key-block lists on the device: one row per (batch, q head, query block)."""

    row_ptr: torch.Tensor  # int32 [num_rows + 1]
    col_idx: torch.Tensor  # int32 [capacity]
    flags: torch.Tensor | None  # uint8 [capacity]
    num_rows: int

    def c(self) -> BlockListsC:
        # the kernels write row_ptr[0 .. num_rows] and col_idx / flags up to
        # the capacity: every buffer must be a contiguous CUDA tensor that long
        if self.row_ptr.numel() < self.num_rows + 1:
            raise ValueError(f"lists.row_ptr: {self.row_ptr.numel()} entries for {self.num_rows} rows")
        if self.flags is not None and self.flags.numel() < self.col_idx.numel():
            raise ValueError(f"lists.flags: {self.flags.numel()} entries, capacity {self.col_idx.numel()}")
        _dev(self.row_ptr, "lists.row_ptr", torch.int32)
        _dev(self.col_idx, "lists.col_idx", torch.int32)
        if self.flags is not None:
            _dev(self.flags, "lists.flags", torch.uint8)
        return BlockListsC(self.row_ptr.data_ptr(), self.col_idx.data_ptr(),
                           self.flags.data_ptr() if self.flags is not None else None,
                           self.col_idx.numel(), self.num_rows)

    def nnz(self) -> int:
        return int(self.row_ptr[-1].item())

    @staticmethod
    def empty(num_rows: int, capacity: int, device, flags: bool = True) -> "BlockLists":
        return BlockLists(torch.empty(num_rows + 1, dtype=torch.int32, device=device),
                          torch.empty(max(1, capacity), dtype=torch.int32, device=device),
                          torch.empty(max(1, capacity), dtype=torch.uint8, device=device) if flags else None,
                          num_rows)


def _dev(x, name: str, dtype: torch.dtype) -> int:
    """Check a contiguous CUDA tensor of the given dtype and return its
    device pointer."""
    if not isinstance(x, torch.Tensor):
        raise TypeError(f"{name}: expected a torch.Tensor")
    if not x.is_cuda or x.dtype != dtype or not x.is_contiguous():
        raise TypeError(f"{name}: expected a contiguous {dtype} CUDA tensor")
    return x.data_ptr()


def _stream() -> ctypes.c_void_p:
    return ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)


def _one_device(ref_name: str, ref, **others) -> torch.device:
    """The device every tensor of one call must live on (ref's).  The library
    launches on the current device and its current stream, so a tensor on
    another GPU would hand a kernel a pointer it cannot use: refuse it here.
    None entries (optional arguments) are skipped."""
    dev = ref.device
    for name, x in others.items():
        if x is not None and x.device != dev:
            raise ValueError(f"{name} is on {x.device} but {ref_name} is on {dev}: "
                             "every tensor of a call must be on one device")
    return dev


def _lists_tensors(lists) -> dict:
    return {"lists.row_ptr": lists.row_ptr, "lists.col_idx": lists.col_idx, "lists.flags": lists.flags}


def _t(x: torch.Tensor, name: str) -> Bf16Tensor:
    """Describe a [B, L, H, 128] bf16 CUDA tensor (head_dim contiguous) for the C ABI."""
    if not isinstance(x, torch.Tensor) or not x.is_cuda:
        raise TypeError(f"{name}: expected a CUDA tensor")
    if x.dtype != torch.bfloat16 or x.dim() != 4 or x.stride(3) != 1:
        raise TypeError(f"{name}: expected bf16 [B, L, H, 128] with a contiguous last dimension")
    B, L, H, D = x.shape
    return Bf16Tensor(x.data_ptr(), B, L, H, D, x.stride(0), x.stride(1), x.stride(2))


def _f32(x: torch.Tensor, name: str) -> int:
    if not x.is_cuda or x.dtype != torch.float32 or not x.is_contiguous():
        raise TypeError(f"{name}: expected a contiguous float32 CUDA tensor")
    return x.data_ptr()


def rbs_block_stats(K: torch.Tensor, block_k: int):
    """Centroids [B, Hkv, nKB, 128] and radii [B, Hkv, nKB] (fp32) of every key block."""
    B, L, H, D = K.shape
    nkb = -(-L // block_k)  # a last, partial block holds the remaining keys
    C = torch.empty(B, H, nkb, D, dtype=torch.float32, device=K.device)
    R = torch.empty(B, H, nkb, dtype=torch.float32, device=K.device)
    tK = _t(K, "K")
    with torch.cuda.device(K.device):
        check(lib().rbs_block_stats(ctypes.byref(tK), block_k, C.data_ptr(), R.data_ptr(), _stream()),
              "rbs_block_stats")
    return C, R


def rbs_block_beta(radii: torch.Tensor, params: SelectParams):
    """beta [B, Hkv, nKB] and the (R_lo, R_hi) range [B, Hkv, 2] from the radii."""
    B, H, n = radii.shape
    beta = torch.empty_like(radii)
    rng = torch.empty(B, H, 2, dtype=torch.float32, device=radii.device)
    p = params.c()
    r_ptr = _f32(radii, "radii")
    with torch.cuda.device(radii.device):
        check(lib().rbs_block_beta(r_ptr, B, H, n, ctypes.byref(p), beta.data_ptr(), rng.data_ptr(), _stream()),
              "rbs_block_beta")
    return beta, rng


def rbs_pool_queries(Q: torch.Tensor, block_q: int):
    """qbar [B, Hq, nQB, 128] and qnorm [B, Hq, nQB] (fp32)."""
    B, L, H, D = Q.shape
    nqb = -(-L // block_q)
    qbar = torch.empty(B, H, nqb, D, dtype=torch.float32, device=Q.device)
    qnorm = torch.empty(B, H, nqb, dtype=torch.float32, device=Q.device)
    tQ = _t(Q, "Q")
    with torch.cuda.device(Q.device):
        check(lib().rbs_pool_queries(ctypes.byref(tQ), block_q, qbar.data_ptr(), qnorm.data_ptr(), _stream()),
              "rbs_pool_queries")
    return qbar, qnorm


def rbs_select_capacity(batch: int, heads_q: int, num_q_blocks: int, num_kv_blocks: int, params: SelectParams) -> int:
    p = params.c()
    return int(lib().rbs_select_capacity(batch, heads_q, num_q_blocks, num_kv_blocks, ctypes.byref(p)))


def rbs_select_workspace_bytes(batch: int, heads_q: int, num_q_blocks: int, kv_heads: int, num_kv_blocks: int,
                               params: SelectParams) -> int:
    p = params.c()
    return int(lib().rbs_select_workspace_bytes(batch, heads_q, num_q_blocks, kv_heads, num_kv_blocks,
                                                ctypes.byref(p)))


def rbs_select(Q: torch.Tensor, centroids: torch.Tensor, radii: torch.Tensor, params: SelectParams,
               workspace: torch.Tensor | None = None, out: BlockLists | None = None, beta_out: torch.Tensor | None = None,
               flags: bool = True) -> BlockLists:
    """Two-branch selection -> CSR key-block lists, rows = (batch, q head, query block), or
    (batch, KV head, query block) when params.list_mode == 1."""
    B, L, Hq, D = Q.shape
    if centroids.dim() != 4:
        raise ValueError(f"centroids: expected [B, Hkv, nKB, {D}], got {tuple(centroids.shape)}")
    Hkv, nkb = centroids.shape[1], centroids.shape[2]
    # every shape first, then where the tensors live
    for x, name, shape in ((centroids, "centroids", (B, Hkv, nkb, D)), (radii, "radii", (B, Hkv, nkb)),
                           (beta_out, "beta_out", (B, Hkv, nkb))):
        if x is not None and tuple(x.shape) != shape:
            raise ValueError(f"{name}: expected shape {shape}, got {tuple(x.shape)}")
    c_ptr = _dev(centroids, "centroids", torch.float32)
    r_ptr = _dev(radii, "radii", torch.float32)
    b_ptr = _dev(beta_out, "beta_out", torch.float32) if beta_out is not None else None
    nqb = -(-L // params.block_q)
    rows = B * (Hkv if params.list_mode == 1 else Hq) * nqb
    if out is None:
        out = BlockLists.empty(rows, rbs_select_capacity(B, Hq, nqb, nkb, params), Q.device, flags)
    if workspace is None:
        workspace = torch.empty(rbs_select_workspace_bytes(B, Hq, nqb, Hkv, nkb, params), dtype=torch.uint8,
                                device=Q.device)
    ws_ptr = _dev(workspace, "workspace", torch.uint8)
    p = params.c()
    lc = out.c()
    tQ = _t(Q, "Q")
    dev = _one_device("Q", Q, centroids=centroids, radii=radii, beta_out=beta_out, workspace=workspace,
                      **_lists_tensors(out))
    with torch.cuda.device(dev):
        check(lib().rbs_select(ctypes.byref(tQ), c_ptr, r_ptr, Hkv, nkb, ctypes.byref(p), ws_ptr,
                               workspace.numel(), ctypes.byref(lc), b_ptr, _stream()), "rbs_select")
    return out


def rbs_lists_causal_full(batch: int, heads_q: int, num_q_blocks: int, q_block_offset: int = 0, device="cuda",
                          flags: bool = False) -> BlockLists:
    """Every causally visible block for every row (the dense reference point)."""
    nnz = int(lib().rbs_lists_causal_full_nnz(batch, heads_q, num_q_blocks, q_block_offset))
    out = BlockLists.empty(batch * heads_q * num_q_blocks, nnz, device, flags)
    lc = out.c()
    with torch.cuda.device(out.row_ptr.device):
        check(lib().rbs_lists_causal_full(batch, heads_q, num_q_blocks, q_block_offset, ctypes.byref(lc), _stream()),
              "rbs_lists_causal_full")
    return out


def rbs_lists_block_attention(seg_start, final_start: int, block: int, batch: int, heads_q: int, q_first_block: int,
                              q_num_blocks: int, device="cuda", flags: bool = False) -> BlockLists:
    """Block-attention mask lists (passages self-attend, the final block sees all)."""
    seg = (ctypes.c_int32 * len(seg_start))(*[int(s) for s in seg_start])
    nnz = int(lib().rbs_lists_block_attention_nnz(seg, len(seg_start), final_start, block, batch, heads_q,
                                                  q_first_block, q_num_blocks))
    if nnz < 0:
        raise RbsError(1, "rbs_lists_block_attention_nnz", lib().rbs_last_error().decode())
    out = BlockLists.empty(batch * heads_q * q_num_blocks, nnz, device, flags)
    lc = out.c()
    with torch.cuda.device(out.row_ptr.device):
        check(lib().rbs_lists_block_attention(seg, len(seg_start), final_start, block, batch, heads_q, q_first_block,
                                              q_num_blocks, ctypes.byref(lc), _stream()), "rbs_lists_block_attention")
    return out


def bsa_prefill(Q: torch.Tensor, K: torch.Tensor, V: torch.Tensor, lists: BlockLists, block_q: int = 128,
                block_k: int = 128, q_offset: int = 0, softmax_scale: float | None = None, causal: bool = True,
                out: torch.Tensor | None = None, return_lse: bool = False):
    """Exact softmax attention of every query block over its listed key blocks."""
    if out is None:
        out = torch.empty_like(Q)
    lse = None
    if return_lse:
        lse = torch.empty(Q.shape[0], Q.shape[2], Q.shape[1], dtype=torch.float32, device=Q.device)
    scale = softmax_scale if softmax_scale is not None else 1.0 / math.sqrt(Q.shape[-1])
    lc = lists.c()
    tQ, tK, tV, tO = _t(Q, "Q"), _t(K, "K"), _t(V, "V"), _t(out, "O")
    dev = _one_device("Q", Q, K=K, V=V, out=out, lse=lse, **_lists_tensors(lists))
    with torch.cuda.device(dev):
        check(lib().bsa_prefill(ctypes.byref(tQ), ctypes.byref(tK), ctypes.byref(tV), ctypes.byref(lc), block_q,
                                block_k, q_offset, scale, 1 if causal else 0, ctypes.byref(tO),
                                lse.data_ptr() if lse is not None else None, _stream()), "bsa_prefill")
    return (out, lse) if return_lse else out


def bsa_prefill_rescue_weighted(Q: torch.Tensor, K: torch.Tensor, V: torch.Tensor, lists: BlockLists,
                                rescue_weight: float, block_q: int = 128, block_k: int = 128, q_offset: int = 0,
                                softmax_scale: float | None = None, causal: bool = True,
                                out: torch.Tensor | None = None, return_lse: bool = False):
    """bsa_prefill with the rescue-only blocks' softmax mass scaled by rescue_weight
    (the lists' flags say which entries those are)."""
    if out is None:
        out = torch.empty_like(Q)
    lse = None
    if return_lse:
        lse = torch.empty(Q.shape[0], Q.shape[2], Q.shape[1], dtype=torch.float32, device=Q.device)
    scale = softmax_scale if softmax_scale is not None else 1.0 / math.sqrt(Q.shape[-1])
    lc = lists.c()
    tQ, tK, tV, tO = _t(Q, "Q"), _t(K, "K"), _t(V, "V"), _t(out, "O")
    dev = _one_device("Q", Q, K=K, V=V, out=out, lse=lse, **_lists_tensors(lists))
    with torch.cuda.device(dev):
        check(lib().bsa_prefill_rescue_weighted(
            ctypes.byref(tQ), ctypes.byref(tK), ctypes.byref(tV), ctypes.byref(lc), block_q, block_k, q_offset, scale,
            1 if causal else 0, float(rescue_weight), ctypes.byref(tO), lse.data_ptr() if lse is not None else None,
            _stream()), "bsa_prefill_rescue_weighted")
    return (out, lse) if return_lse else out


def bsa_prefill_segments(Q: torch.Tensor, K: torch.Tensor, V: torch.Tensor, lists: BlockLists, seg_start,
                         final_start: int, block_q: int = 128, block_k: int = 128, q_offset: int = 0,
                         softmax_scale: float | None = None, out: torch.Tensor | None = None,
                         return_lse: bool = False):
    """bsa_prefill with the Block-attention mask applied token by token: a query
    token of a passage sees only its own passage's earlier keys, a token of the
    final block every earlier key (passage starts may be any token offsets)."""
    if out is None:
        out = torch.empty_like(Q)
    lse = None
    if return_lse:
        lse = torch.empty(Q.shape[0], Q.shape[2], Q.shape[1], dtype=torch.float32, device=Q.device)
    scale = softmax_scale if softmax_scale is not None else 1.0 / math.sqrt(Q.shape[-1])
    seg = (ctypes.c_int32 * len(seg_start))(*[int(s) for s in seg_start])
    lc = lists.c()
    tQ, tK, tV, tO = _t(Q, "Q"), _t(K, "K"), _t(V, "V"), _t(out, "O")
    dev = _one_device("Q", Q, K=K, V=V, out=out, lse=lse, **_lists_tensors(lists))
    with torch.cuda.device(dev):
        check(lib().bsa_prefill_segments(ctypes.byref(tQ), ctypes.byref(tK), ctypes.byref(tV), ctypes.byref(lc),
                                         block_q, block_k, q_offset, seg, len(seg_start), int(final_start), scale,
                                         ctypes.byref(tO), lse.data_ptr() if lse is not None else None, _stream()),
              "bsa_prefill_segments")
    return (out, lse) if return_lse else out


def rope_reencode(x: torch.Tensor, old_pos: torch.Tensor, new_pos: torch.Tensor, theta: float, rope_style: int = 0,
                  out: torch.Tensor | None = None) -> torch.Tensor:
    """Move RoPE-encoded vectors from old_pos to new_pos (out may be x for in place)."""
    if out is None:
        out = torch.empty_like(x)
    for name, p in (("old_pos", old_pos), ("new_pos", new_pos)):
        if not p.is_cuda or p.dtype != torch.int32 or p.numel() != x.shape[1]:
            raise TypeError(f"{name}: expected int32 CUDA tensor of length {x.shape[1]}")
    tx, to = _t(x, "x"), _t(out, "out")
    dev = _one_device("x", x, out=out, old_pos=old_pos, new_pos=new_pos)
    with torch.cuda.device(dev):
        check(lib().rope_reencode(ctypes.byref(tx), ctypes.byref(to), old_pos.data_ptr(), new_pos.data_ptr(), theta,
                                  rope_style, _stream()), "rope_reencode")
    return out


def rbs_get_device_error() -> int:
    """Read and clear the library's device error word (synchronises the current stream)."""
    code = ctypes.c_int32(0)
    st = lib().rbs_get_device_error(ctypes.byref(code), _stream())
    if st not in (0, 5):
        check(st, "rbs_get_device_error")
    return int(code.value)
