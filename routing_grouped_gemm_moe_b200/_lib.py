"""ctypes view of ``libmoe_b200.so`` (the C ABI declared in include/moe_b200.h).

Loading fails loudly when the library has not been built; there is no
fallback implementation.
"""
from __future__ import annotations

import ctypes as C
import os

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libmoe_b200.so")

MOE_OK = 0
STATUS_NAMES = {0: "MOE_OK", 1: "MOE_ERR_INVALID_ARG", 2: "MOE_ERR_UNSUPPORTED",
                3: "MOE_ERR_CUDA", 4: "MOE_ERR_DEVICE_TIMEOUT", 5: "MOE_ERR_DEVICE_BOUNDS"}

DTYPE_BF16, DTYPE_MXFP8 = 0, 1
GG_RAGGED_M, GG_RAGGED_K = 0, 1
EPI_NONE, EPI_SWIGLU, EPI_SWIGLU_BWD = 0, 1, 2
ROUTER_LOGITS, ROUTER_PROJ = 0, 1

vp = C.c_void_p
i32 = C.c_int
i64 = C.c_int64
sz = C.c_size_t


class GGArgs(C.Structure):
    _fields_ = [("mode", i32), ("dtype", i32), ("epilogue", i32), ("E", i32),
                ("M_total", i64), ("M", i32), ("N", i32), ("K", i32),
                ("offsets", vp), ("a", vp), ("b", vp), ("b_mn_major", i32),
                ("c", vp), ("aux", vp), ("gu", vp), ("a_scales", vp), ("b_scales", vp),
                ("workspace", vp), ("workspace_bytes", sz), ("status", vp),
                ("q_row_codes", vp), ("q_row_scales", vp), ("q_col_codes", vp),
                ("q_col_scales", vp)]


FWD_STAGES, BWD_STAGES = 5, 8
MX_GEMM1, MX_GEMM2, MX_DA, MX_DW2, MX_DX, MX_DW13 = 1, 2, 4, 8, 16, 32


class LayerDesc(C.Structure):
    _fields_ = [("T", i32), ("d", i32), ("E", i32), ("k", i32), ("f", i32),
                ("dtype", i32), ("router_mode", i32), ("recompute", i32), ("mx_gemms", i32),
                ("mx_keep_weights", i32),
                ("stage_events", C.POINTER(vp))]


class LayerParams(C.Structure):
    _fields_ = [("x", vp), ("logits", vp), ("w_r", vp), ("w13", vp), ("w2", vp)]


class LayerSaved(C.Structure):
    _fields_ = [("logits", vp), ("topk_idx", vp), ("topk_w", vp), ("counts", vp),
                ("offsets", vp), ("dest_pos", vp), ("src_token", vp), ("x_perm", vp),
                ("gu", vp), ("a", vp), ("y_perm", vp)]


class LayerGrads(C.Structure):
    _fields_ = [("dx", vp), ("dw13", vp), ("dw2", vp), ("dw_r", vp), ("d_logits", vp)]


# name -> (restype, argtypes)
SIGNATURES = {
    "moe_status_string": (C.c_char_p, [i32]),
    "moe_version": (i32, []),
    "moe_kernel_launches": (C.c_uint64, []),
    "moe_read_device_status": (i32, [vp, i32, C.POINTER(C.c_int32), vp]),
    "moe_selftest_bounded_wait": (i32, [vp, C.c_uint64, vp, vp]),
    "moe_router_topk": (i32, [vp, i32, i32, i32, vp, vp, vp]),
    "moe_router_topk_proj": (i32, [vp, vp, i32, i32, i32, i32, vp, vp, vp, vp]),
    "moe_router_bwd": (i32, [vp, vp, vp, i32, i32, i32, vp, vp]),
    "moe_router_proj_bwd": (i32, [vp, vp, i32, i32, i32, vp, vp]),
    "moe_router_balance_workspace_bytes": (sz, [i32, i32]),
    "moe_router_balance": (i32, [vp, vp, i32, i32, i32, vp, vp, vp, sz, vp]),
    "moe_router_balance_bwd": (i32, [vp, vp, i32, i32, i32, C.c_float, vp, vp]),
    "moe_permute_workspace_bytes": (sz, [i32, i32]),
    "moe_permute_rows": (i32, [vp, vp, i32, i32, i32, i32, vp, vp, vp, vp, vp, vp, sz, vp]),
    "moe_permute_rows_noalloc": (i32, [vp, vp, i32, i32, i32, i32, vp, vp, vp, vp, vp, vp]),
    "moe_permute_rows_mxfp8": (i32, [vp, vp, i32, i32, i32, i32, vp, vp, vp, vp, vp, vp, vp, vp, sz, vp]),
    "moe_grouped_gemm": (i32, [C.POINTER(GGArgs), vp]),
    "moe_grouped_gemm_workspace_bytes": (sz, [C.POINTER(GGArgs)]),
    "moe_swiglu": (i32, [vp, vp, i64, i32, vp]),
    "moe_swiglu_bwd": (i32, [vp, vp, vp, i64, i32, vp]),
    "moe_unpermute_combine": (i32, [vp, vp, vp, i32, i32, i32, vp, vp]),
    "moe_unpermute_combine_bwd": (i32, [vp, vp, vp, vp, i32, i32, i32, vp, vp, vp]),
    "moe_unpermute_sum": (i32, [vp, vp, i32, i32, i32, vp, vp, i32, vp, vp]),
    "mxfp8_quantize": (i32, [vp, i64, i64, i32, vp, i32, vp, vp, vp, vp]),
    "mxfp8_quantize_rowcol": (i32, [vp, i64, i64, vp, i32, vp, vp, vp, vp, vp]),
    "moe_layer_workspace_bytes": (sz, [C.POINTER(LayerDesc)]),
    "moe_layer_fwd": (i32, [C.POINTER(LayerDesc), C.POINTER(LayerParams), C.POINTER(LayerSaved),
                            vp, vp, sz, vp]),
    "moe_layer_bwd": (i32, [C.POINTER(LayerDesc), C.POINTER(LayerParams), C.POINTER(LayerSaved),
                            vp, C.POINTER(LayerGrads), vp, sz, vp]),
}

_lib = None


class MoeError(RuntimeError):
    def __init__(self, fn: str, status: int):
        super().__init__(f"{fn} returned {STATUS_NAMES.get(status, status)}")
        self.status = status


def lib() -> C.CDLL:
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is missing: build it with "
                               "`python -m routing_grouped_gemm_moe_b200.build`")
        L = C.CDLL(LIB_PATH)
        for name, (res, args) in SIGNATURES.items():
            fn = getattr(L, name)
            fn.restype = res
            fn.argtypes = args
        _lib = L
    return _lib


def call(name: str, *args) -> None:
    st = getattr(lib(), name)(*args)
    if st != MOE_OK:
        raise MoeError(name, st)
