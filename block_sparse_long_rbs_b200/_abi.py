"""ctypes declarations of the librbs C ABI (include/rbs.h).

Loading needs no GPU; compute calls do.  The library must have been built
in-tree (``python -m block_sparse_long_rbs_b200.build``); a missing library
raises immediately -- there is no fallback path.
"""

from __future__ import annotations

import ctypes
import os

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "librbs.so")

RBS_OK = 0
STATUS_NAMES = {0: "RBS_OK", 1: "RBS_ERR_INVALID_ARG", 2: "RBS_ERR_UNSUPPORTED", 3: "RBS_ERR_CAPACITY",
                4: "RBS_ERR_CUDA", 5: "RBS_ERR_DEVICE"}
DEVERR_BLOCK_INDEX, DEVERR_ROW_PTR, DEVERR_TIMEOUT, DEVERR_NONCAUSAL = 0x1, 0x2, 0x4, 0x8
MAX_SEGMENTS = 512
MAX_KV_BLOCKS = 4096
NOALLOC_SCRATCH_BYTES = 32 << 20


class Bf16Tensor(ctypes.Structure):
    _fields_ = [("data", ctypes.c_void_p), ("batch", ctypes.c_int64), ("seqlen", ctypes.c_int64),
                ("heads", ctypes.c_int64), ("head_dim", ctypes.c_int64), ("stride_b", ctypes.c_int64),
                ("stride_s", ctypes.c_int64), ("stride_h", ctypes.c_int64)]


class SelectParamsC(ctypes.Structure):
    _fields_ = [("block_q", ctypes.c_int32), ("block_k", ctypes.c_int32), ("rho_centroid", ctypes.c_float),
                ("rho_rescue", ctypes.c_float), ("beta_mode", ctypes.c_int32), ("beta_const", ctypes.c_float),
                ("beta_p_lo", ctypes.c_float), ("beta_p_hi", ctypes.c_float), ("force_diag", ctypes.c_int32),
                ("force_sink", ctypes.c_int32), ("causal", ctypes.c_int32), ("q_block_offset", ctypes.c_int32),
                ("threshold_mode", ctypes.c_int32), ("delta_centroid", ctypes.c_float), ("delta_rescue", ctypes.c_float),
                ("list_mode", ctypes.c_int32), ("query_pool", ctypes.c_int32)]


class BlockListsC(ctypes.Structure):
    _fields_ = [("row_ptr", ctypes.c_void_p), ("col_idx", ctypes.c_void_p), ("flags", ctypes.c_void_p),
                ("capacity", ctypes.c_int64), ("num_rows", ctypes.c_int32)]


P = ctypes.POINTER
vp = ctypes.c_void_p
i32, i64, f32, sz = ctypes.c_int32, ctypes.c_int64, ctypes.c_float, ctypes.c_size_t

# name -> (restype, argtypes): every entry point include/rbs.h declares
SIGNATURES = {
    "rbs_abi_version": (i32, []),
    "rbs_status_string": (ctypes.c_char_p, [ctypes.c_int]),
    "rbs_last_error": (ctypes.c_char_p, []),
    "rbs_select_params_default": (None, [P(SelectParamsC)]),
    "rbs_get_device_error": (ctypes.c_int, [P(i32), vp]),
    "rbs_block_stats": (ctypes.c_int, [P(Bf16Tensor), i32, vp, vp, vp]),
    "rbs_block_beta": (ctypes.c_int, [vp, i64, i64, i64, P(SelectParamsC), vp, vp, vp]),
    "rbs_pool_queries": (ctypes.c_int, [P(Bf16Tensor), i32, vp, vp, vp]),
    "rbs_select_capacity": (i64, [i64, i64, i64, i64, P(SelectParamsC)]),
    "rbs_select_workspace_bytes": (sz, [i64, i64, i64, i64, i64, P(SelectParamsC)]),
    "rbs_select": (ctypes.c_int, [P(Bf16Tensor), vp, vp, i32, i64, P(SelectParamsC), vp, sz, P(BlockListsC), vp, vp]),
    "rbs_select_noalloc": (ctypes.c_int, [P(Bf16Tensor), vp, vp, i32, i64, P(SelectParamsC), P(BlockListsC), vp, vp]),
    "rbs_lists_causal_full_nnz": (i64, [i32, i32, i32, i32]),
    "rbs_lists_causal_full": (ctypes.c_int, [i32, i32, i32, i32, P(BlockListsC), vp]),
    "rbs_lists_block_attention_nnz": (i64, [P(i32), i32, i32, i32, i32, i32, i32, i32]),
    "rbs_lists_block_attention": (ctypes.c_int, [P(i32), i32, i32, i32, i32, i32, i32, i32, P(BlockListsC), vp]),
    "bsa_prefill": (ctypes.c_int, [P(Bf16Tensor), P(Bf16Tensor), P(Bf16Tensor), P(BlockListsC), i32, i32, i64, f32,
                                   i32, P(Bf16Tensor), vp, vp]),
    "bsa_prefill_rescue_weighted": (ctypes.c_int, [P(Bf16Tensor), P(Bf16Tensor), P(Bf16Tensor), P(BlockListsC), i32,
                                                   i32, i64, f32, i32, f32, P(Bf16Tensor), vp, vp]),
    "bsa_prefill_segments": (ctypes.c_int, [P(Bf16Tensor), P(Bf16Tensor), P(Bf16Tensor), P(BlockListsC), i32, i32,
                                            i64, P(i32), i32, i32, f32, P(Bf16Tensor), vp, vp]),
    "rope_reencode": (ctypes.c_int, [P(Bf16Tensor), P(Bf16Tensor), vp, vp, f32, i32, vp]),
    "rbs_testing_bsa_prefill_stalled": (ctypes.c_int, [P(Bf16Tensor), P(Bf16Tensor), P(Bf16Tensor), P(BlockListsC),
                                                       i32, i32, ctypes.c_uint64, i32, P(Bf16Tensor), vp]),
    "rbs_testing_exp2": (ctypes.c_int, [vp, vp, i64, vp]),
}


class RbsError(RuntimeError):
    def __init__(self, status: int, where: str, detail: str):
        self.status = status
        super().__init__(f"{where}: {STATUS_NAMES.get(status, status)}: {detail}")


ABI_VERSION = 5  # RBS_ABI_VERSION of include/rbs.h that these structures match
_lib = None


def lib() -> ctypes.CDLL:
    """The loaded librbs.so with every signature set (raises if it is not built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(f"librbs.so not built at {LIB_PATH}; run python -m block_sparse_long_rbs_b200.build")
        L = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in SIGNATURES.items():
            fn = getattr(L, name)
            fn.restype = res
            fn.argtypes = args
        if L.rbs_abi_version() != ABI_VERSION:
            raise ImportError(f"{LIB_PATH} has ABI version {L.rbs_abi_version()}, this binding expects {ABI_VERSION}; "
                              "rebuild it with python -m block_sparse_long_rbs_b200.build")
        _lib = L
    return _lib


def check(status: int, where: str) -> None:
    if status != RBS_OK:
        raise RbsError(status, where, lib().rbs_last_error().decode())
