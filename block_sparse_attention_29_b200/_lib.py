"""ctypes binding of libsparse_attn.so (the C ABI in include/sparse_attn.h).

Argument marshalling only: every step of the computation runs in the library's
CUDA kernels.  Loading fails loudly (RuntimeError) when the library has not
been built; there is no fallback implementation.
"""
from __future__ import annotations

import ctypes
import os

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libsparse_attn.so")

SA_OK = 0
SA_ERR_INVALID_ARG = 1
SA_ERR_UNSUPPORTED = 2
SA_ERR_CUDA = 3
SA_ERR_NO_MEMORY = 4
SA_ERR_TIMEOUT = 5
SA_ERR_DEVICE_INDEX = 6

# Every function the header declares (tests check the library exports them all).
EXPORTS = (
    "sparse_attn_plan_create", "sparse_attn_plan_create_ex", "sparse_attn_plan_create_opts",
    "sparse_attn_plan_info",
    "sparse_attn_plan_destroy",
    "sparse_attn_prefill_plan", "sparse_attn_prefill", "sparse_attn_block_stats",
    "sparse_attn_calibrate", "sparse_attn_gather", "sparse_attn_decode_window",
    "sparse_attn_window_slot", "sparse_attn_compile_pattern", "sparse_attn_work_order",
    "sparse_attn_check_device_error", "sparse_attn_last_error", "sparse_attn_prefill_noalloc",
    "sparse_attn_decode_topk", "sparse_attn_decode_topk_workspace",
)


class SaPattern(ctypes.Structure):
    """sa_pattern_t."""
    _fields_ = [("causal", ctypes.c_int32), ("window", ctypes.c_int32),
                ("n_global", ctypes.c_int32), ("block_local", ctypes.c_int32),
                ("block_q", ctypes.c_int32), ("block_k", ctypes.c_int32),
                ("random_block", ctypes.c_int32), ("n_random", ctypes.c_int32),
                ("random_table", ctypes.c_void_p), ("thresholds", ctypes.c_void_p),
                ("scale", ctypes.c_float), ("dilation", ctypes.c_int32),
                ("skipped_in_denominator", ctypes.c_int32), ("row_level_skip", ctypes.c_int32)]


class SaPlanInfo(ctypes.Structure):
    """sa_plan_info_t."""
    _fields_ = [("T_q", ctypes.c_int32), ("n_kb", ctypes.c_int32),
                ("n_units", ctypes.c_int64), ("blocks", ctypes.c_int64),
                ("blocks_full", ctypes.c_int64), ("blocks_desc", ctypes.c_int64),
                ("pairs", ctypes.c_int64), ("compile_ms", ctypes.c_double),
                ("split_tiles", ctypes.c_int64), ("queue_units", ctypes.c_int64),
                ("workspace_bytes", ctypes.c_int64)]


class SaPlanOptions(ctypes.Structure):
    """sa_plan_options_t."""
    _fields_ = [("kernel", ctypes.c_int32), ("max_unit_blocks", ctypes.c_int32)]


class SparseAttnError(RuntimeError):
    def __init__(self, code: int, msg: str):
        super().__init__(f"sparse_attn error {code}: {msg}")
        self.code = code


_lib = None


def lib():
    """The loaded library (raises RuntimeError when it is missing)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is missing: build it with "
                               "`python -m block_sparse_attention_29_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        vp, i32, i64, f32, f64 = (ctypes.c_void_p, ctypes.c_int, ctypes.c_int64,
                                  ctypes.c_float, ctypes.c_double)
        P = ctypes.POINTER(SaPattern)
        L.sparse_attn_plan_create.argtypes = [P, i32, i32, i32, i32, i32, ctypes.POINTER(vp)]
        L.sparse_attn_plan_create_ex.argtypes = [P, i32, i32, i32, i32, i32, i32,
                                                 ctypes.POINTER(vp)]
        L.sparse_attn_plan_create_opts.argtypes = [P, i32, i32, i32, i32, i32,
                                                   ctypes.POINTER(SaPlanOptions),
                                                   ctypes.POINTER(vp)]
        L.sparse_attn_plan_info.argtypes = [vp, ctypes.POINTER(SaPlanInfo)]
        L.sparse_attn_plan_destroy.argtypes = [vp]
        L.sparse_attn_plan_destroy.restype = None
        L.sparse_attn_prefill_plan.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, vp, vp]
        L.sparse_attn_prefill.argtypes = [vp, vp, vp, vp, i32, i32, i32, i32, i32, P, vp, vp, vp]
        L.sparse_attn_prefill_noalloc.argtypes = [vp, vp, vp, vp, i32, i32, i32, i32, i32, P, vp,
                                                  vp]
        L.sparse_attn_block_stats.argtypes = [vp, vp, vp, vp, vp, vp]
        L.sparse_attn_calibrate.argtypes = [vp, vp, f64, vp, vp]
        L.sparse_attn_decode_window.argtypes = [vp, vp, vp, vp, vp, i32, i32, i32, i32, P, vp, vp]
        L.sparse_attn_window_slot.argtypes = [i64, i32, i32]
        L.sparse_attn_decode_topk.argtypes = [vp, vp, vp, vp, vp, i32, i32, i32, i32, i32, i32,
                                              f32, vp, vp, vp, vp, ctypes.c_size_t, vp]
        L.sparse_attn_decode_topk_workspace.argtypes = [i32, i32, i32, i32]
        L.sparse_attn_gather.argtypes = [vp, vp, vp, vp, vp, vp, i32, i32, i32, i32, i32, i32,
                                         i32, f32, vp, vp]
        L.sparse_attn_work_order.argtypes = [P, i32, i32, i32, i32, i32, i32, vp, vp, vp, vp,
                                             vp, vp]
        L.sparse_attn_compile_pattern.argtypes = [P, i32, i32, i32, i32,
                                                  ctypes.POINTER(ctypes.c_int),
                                                  ctypes.POINTER(ctypes.c_int),
                                                  ctypes.POINTER(i64), vp, vp, vp, vp]
        L.sparse_attn_check_device_error.argtypes = [vp]
        L.sparse_attn_last_error.argtypes = []
        L.sparse_attn_last_error.restype = ctypes.c_char_p
        for name in EXPORTS:
            if name not in ("sparse_attn_plan_destroy", "sparse_attn_last_error"):
                getattr(L, name).restype = ctypes.c_int
        L.sparse_attn_window_slot.restype = i64
        L.sparse_attn_decode_topk_workspace.restype = ctypes.c_size_t
        _lib = L
    return _lib


def check(rc: int) -> None:
    if rc != SA_OK:
        raise SparseAttnError(rc, lib().sparse_attn_last_error().decode(errors="replace"))
