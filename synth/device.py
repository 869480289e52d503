"""Device-side twin of synth.draws.expert_weights (libfp4synth.so, C ABI).

Input generation only: draws the same Student-t(4) / planted-outlier weights
as the host recipe, bit for bit, directly into a CUDA float32 tensor.
"""
from __future__ import annotations

import ctypes
import os

import numpy as np

from .draws import t4_scale

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libfp4synth.so")
_lib = None


def _load():
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is missing: build with `python -m fp4_block_scaled_moe_b200.build`")
        lib = ctypes.CDLL(LIB_PATH)
        lib.synth_t4_weights.restype = ctypes.c_int
        lib.synth_t4_weights.argtypes = [ctypes.c_void_p, ctypes.c_int64, ctypes.c_int64, ctypes.c_uint32,
                                         ctypes.c_uint32, ctypes.c_float, ctypes.c_int, ctypes.c_float,
                                         ctypes.c_float, ctypes.c_float, ctypes.c_float, ctypes.c_void_p]
        _lib = lib
    return _lib


def expert_weights_into(out, seed: int, tensor_id: int, start_row: int = 0, sigma: float = 0.02,
                        outliers=None, stream=None):
    """Fill ``out`` (CUDA float32, [rows, K] contiguous) with rows starting at start_row."""
    import torch
    assert out.is_cuda and out.dtype == torch.float32 and out.is_contiguous()
    k = out.shape[-1]
    start = start_row * k
    count = out.numel()
    if outliers is None:
        wo, frac, lo, span = 0, 0.0, 0.0, 0.0
    else:
        frac, lo_s, hi_s = outliers
        wo, frac, lo, span = 1, float(np.float32(frac)), float(np.float32(lo_s)), float(np.float32(hi_s - lo_s))
    st = torch.cuda.current_stream(out.device).cuda_stream if stream is None else stream
    rc = _load().synth_t4_weights(ctypes.c_void_p(out.data_ptr()), start, count, seed, tensor_id,
                                  float(t4_scale(sigma)), wo, frac, lo, span, float(np.float32(sigma)),
                                  ctypes.c_void_p(st))
    if rc != 0:
        raise RuntimeError(f"synth_t4_weights failed: cudaError {rc}")
    return out
