"""ctypes loader for the in-tree C-ABI library ``libfp4moe.so`` (include/fp4moe.h).

Argument marshalling only: every step of the layer runs in the library's CUDA
kernels. There is no fallback: if the library is missing, loading raises.
"""
from __future__ import annotations

import ctypes
import os

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libfp4moe.so")

FP4_MXFP4, FP4_NVFP4, FP4_CB4, FP4_V2A, FP4_DENSE_BF16 = 1, 2, 3, 4, 5
FP4_F32, FP4_BF16 = 0, 1
FORMATS = {"mxfp4": FP4_MXFP4, "nvfp4": FP4_NVFP4, "cb4": FP4_CB4, "v2a": FP4_V2A}
BLOCK = {FP4_MXFP4: 32, FP4_NVFP4: 16}

STATUS = {
    0: "FP4_OK", 1: "FP4_ERR_INVALID_ARG", 2: "FP4_ERR_EMPTY_SHAPE", 3: "FP4_ERR_SHAPE_OVERFLOW",
    4: "FP4_ERR_ALIGNMENT", 5: "FP4_ERR_UNSUPPORTED", 6: "FP4_ERR_WORKSPACE", 7: "FP4_ERR_CUDA",
    8: "FP4_ERR_TIMEOUT",
}

# Every function the header declares, with its C signature.
_vp, _i32, _i64, _sz, _f32 = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64, ctypes.c_size_t, ctypes.c_float
_cint = ctypes.c_int


class MoEWeightsC(ctypes.Structure):
    _fields_ = [
        ("fmt", _cint), ("num_experts", _i32), ("hidden", _i32), ("inter", _i32), ("swiglu_limit", _f32),
        ("gu_codes", _vp), ("gu_scales", _vp), ("gu_tscale", _vp),
        ("dn_codes", _vp), ("dn_scales", _vp), ("dn_tscale", _vp),
        ("gu_cb", _vp), ("gu_rowptr", _vp), ("gu_col", _vp), ("gu_val", _vp),
        ("dn_cb", _vp), ("dn_rowptr", _vp), ("dn_col", _vp), ("dn_val", _vp),
        ("kernel_variant", _i32),
        ("gu_mma_scales", _vp), ("dn_mma_scales", _vp),
        ("expert_begin", _i32), ("local_experts", _i32),
        ("expert_format", _vp), ("gu_offset", _vp), ("gu_scale_offset", _vp), ("dn_offset", _vp),
        ("dn_scale_offset", _vp), ("gu_bytes", _i64), ("gu_scale_bytes", _i64), ("dn_bytes", _i64),
        ("dn_scale_bytes", _i64),
    ]


class RouteOutC(ctypes.Structure):
    _fields_ = [("logits", _vp), ("topk_ids", _vp), ("topk_w", _vp), ("counts", _vp), ("offsets", _vp),
                ("perm", _vp), ("inv", _vp)]


class KernelStatsC(ctypes.Structure):
    _fields_ = [("gate_up_ns", ctypes.c_uint64), ("gate_up_launches", ctypes.c_uint64),
                ("down_ns", ctypes.c_uint64), ("down_launches", ctypes.c_uint64)]


SIGNATURES = {
    "fp4_status_string": (ctypes.c_char_p, [_cint]),
    "fp4_last_error_string": (ctypes.c_char_p, []),
    "fp4_version": (ctypes.c_char_p, []),
    "fp4_launch_count": (ctypes.c_ulonglong, []),
    "fp4_selftest_wait_timeout": (_cint, [_vp, _i64, _vp]),
    "fp4_pack": (_cint, [_cint, _vp, _cint, _i64, _i64, _i64, _vp, _vp, _vp, _vp]),
    "fp4_mma_scales": (_cint, [_vp, _i64, _i64, _i64, _vp, _vp]),
    "fp4_nvfp4_mma_scales": (_cint, [_vp, _i64, _i64, _i64, _vp, _vp]),
    "fp4_cb4_row_ptr": (_cint, [_vp, _cint, _i64, _i64, ctypes.c_double, ctypes.c_double, _vp, _vp]),
    "fp4_pack_cb4": (_cint, [_vp, _cint, _i64, _i64, ctypes.c_double, ctypes.c_double, _vp, _vp, _vp, _vp, _vp,
                             _vp]),
    "fp4_pack_v2a_workspace_size": (_sz, [_i64, _i64, _i64, _i32]),
    "fp4_pack_v2a": (_cint, [_vp, _cint, _i64, _i64, _i64, _i32, ctypes.c_double, ctypes.c_double, _vp, _vp, _vp,
                             _vp, _vp, _vp, _vp, _sz, _vp]),
    "fp4_unpack_v2a": (_cint, [_vp, _vp, _vp, _i64, _i64, _i64, _i32, _vp, _vp]),
    "fp4_unpack": (_cint, [_cint, _vp, _vp, _vp, _i64, _i64, _i64, _vp, _cint, _vp]),
    "moe_route": (_cint, [_vp, _vp, _vp, _i32, _i32, _i32, _i32, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp]),
    "moe_fp4_workspace_size": (_sz, [ctypes.POINTER(MoEWeightsC), _i32, _i32]),
    "moe_fp4_forward": (_cint, [ctypes.POINTER(MoEWeightsC), _vp, _vp, _vp, _i32, _i32, _vp,
                                ctypes.POINTER(RouteOutC), _vp, _sz, _vp]),
    "moe_fp4_forward_partial": (_cint, [ctypes.POINTER(MoEWeightsC), _vp, _vp, _vp, _i32, _i32, _vp,
                                        ctypes.POINTER(RouteOutC), _vp, _sz, _vp]),
    "fp4_f32_to_bf16": (_cint, [_vp, _i64, _vp, _vp]),
    "fp4_linear_workspace_size": (_sz, [_i32, _i64]),
    "fp4_linear": (_cint, [_cint, _vp, _i32, _i64, _vp, _vp, _vp, _i64, _vp, _vp, _sz, _vp]),
    "fp4_workspace_status": (_cint, [_vp, _vp]),
    "moe_fp4_noalloc_capacity": (_sz, []),
    "moe_fp4_forward_noalloc": (_cint, [ctypes.POINTER(MoEWeightsC), _vp, _vp, _vp, _i32, _i32, _vp, _vp]),
    "moe_fp4_noalloc_status": (_cint, [_vp]),
    "moe_fp4_expert_kernels": (_i32, [ctypes.POINTER(MoEWeightsC), _i32, _i32]),
    "fp4_workspace_kernel_stats": (_cint, [_vp, _cint, ctypes.POINTER(KernelStatsC), _vp]),
}

_lib = None


class FP4Error(RuntimeError):
    def __init__(self, fn, code, detail=""):
        self.code = code
        self.name = STATUS.get(code, str(code))
        super().__init__(f"{fn} -> {self.name}" + (f": {detail}" if detail else ""))


def load():
    """Load libfp4moe.so (raises if it has not been built)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise RuntimeError(f"{LIB_PATH} is missing: build it with `python -m fp4_block_scaled_moe_b200.build`")
    lib = ctypes.CDLL(LIB_PATH)
    for name, (res, args) in SIGNATURES.items():
        f = getattr(lib, name)
        f.restype = res
        f.argtypes = args
    _lib = lib
    return lib


def check(fn, code):
    if code != 0:
        detail = ""
        if code == 7:
            detail = load().fp4_last_error_string().decode()
        raise FP4Error(fn, code, detail)
