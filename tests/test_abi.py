"""The C-ABI library loads, exports every declared symbol, and refuses bad shapes by
name before touching the device (CPU only; no kernel is launched here)."""
import ctypes
import os
import re

import pytest

from fp4_block_scaled_moe_b200 import _lib as L

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HDR = os.path.join(ROOT, "include", "fp4moe.h")
P = ctypes.c_void_p(0x10000)      # aligned dummy device pointer: never dereferenced on refusal
PMIS = ctypes.c_void_p(0x10008)   # misaligned


def declared():
    src = open(HDR).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    src = "\n".join(l for l in src.splitlines() if not l.lstrip().startswith("#"))
    return sorted(set(re.findall(r"\b([a-z][a-z0-9_]+)\s*\(", src)))


def test_exports_every_declared_symbol():
    lib = L.load()
    names = declared()
    assert set(L.SIGNATURES) == set(names), (set(L.SIGNATURES) ^ set(names))
    for n in names:
        assert hasattr(lib, n)
    assert lib.fp4_version() == b"0.1.0"
    assert lib.fp4_status_string(3) == b"FP4_ERR_SHAPE_OVERFLOW"


def _pack(fmt, batch, n, k, w=P, codes=P, scales=P, ts=P):
    return L.load().fp4_pack(fmt, w, 0, batch, n, k, codes, scales, ts, None)


def test_pack_named_refusals():
    assert _pack(L.FP4_MXFP4, 1, 0, 32) == 2                 # EmptyShape
    assert _pack(L.FP4_MXFP4, 0, 4, 32) == 2
    assert _pack(L.FP4_MXFP4, -1, 4, 32) == 2
    assert _pack(L.FP4_MXFP4, 1 << 40, 1 << 20, 64) == 3     # ShapeOverflow
    assert _pack(L.FP4_MXFP4, 1, 4, 48) == 4                 # K not a multiple of 32
    assert _pack(L.FP4_NVFP4, 1, 4, 24) == 4
    assert _pack(L.FP4_MXFP4, 1, 4, 32, w=PMIS) == 4         # misaligned
    assert _pack(L.FP4_NVFP4, 1, 4, 32, ts=None) == 1        # NVFP4 needs the tensor scale
    assert _pack(L.FP4_CB4, 1, 4, 128) == 5
    assert _pack(9, 1, 4, 32) == 5
    assert L.load().fp4_unpack(L.FP4_MXFP4, P, P, None, 1, 4, 0, P, 0, None) == 2


def test_route_named_refusals():
    lib = L.load()
    r = lambda T, H, E, k, lg=None: lib.moe_route(P, P, None, T, H, E, k, lg, P, P, P, P, P, P, P, None)
    assert r(0, 64, 8, 2) == 2
    assert r(4, 64, 8, 0) == 2
    assert r(4, 64, 8, 9) == 1        # k > E
    assert r(4, 64, 64, 33) == 1      # k > 32
    assert r(4, 64, 2048, 8) == 1     # E > 1024
    assert r(4, 60, 8, 2) == 4        # H % 8
    assert r(1 << 30, 64, 8, 8) == 3  # T k overflows int32


def _weights(fmt=L.FP4_MXFP4, E=8, H=512, I=256, lim=7.0):
    s = L.MoEWeightsC()
    s.fmt, s.num_experts, s.hidden, s.inter, s.swiglu_limit = fmt, E, H, I, lim
    for f in ("gu_codes", "gu_scales", "dn_codes", "dn_scales", "gu_tscale", "dn_tscale"):
        setattr(s, f, 0x10000)
    return s


def test_forward_named_refusals():
    lib = L.load()

    def fwd(w, T=4, k=2, ws=P, nbytes=1 << 40):
        return lib.moe_fp4_forward(ctypes.byref(w), P, P, None, T, k, P, None, ws, nbytes, None)

    assert fwd(_weights(E=0)) == 2
    assert fwd(_weights(), T=0) == 2
    assert fwd(_weights(H=500)) == 4
    assert fwd(_weights(H=544)) == 5           # multiple of 32 but not of 256: not run by this build
    assert fwd(_weights(lim=float("inf"))) == 1
    assert fwd(_weights(lim=-1.0)) == 1
    assert fwd(_weights(), k=9) == 1
    assert fwd(_weights(fmt=L.FP4_CB4)) == 1           # CB4 without codebooks / CSR
    cb = _weights(fmt=L.FP4_CB4)
    cb.gu_cb = cb.dn_cb = cb.gu_rowptr = cb.dn_rowptr = 0x10000
    cb.kernel_variant = 2
    assert fwd(cb) == 5                                 # CB4 runs on the CUDA-core kernels only
    assert fwd(_weights(E=1 << 20, H=1 << 16, I=1 << 16)) == 3
    assert fwd(_weights(), ws=None) == 6
    bad = _weights()
    bad.kernel_variant = 7
    assert fwd(bad) == 1                       # unknown kernel variant
    nv1, nv2 = _weights(fmt=L.FP4_NVFP4), _weights(fmt=L.FP4_NVFP4)
    nv1.kernel_variant, nv2.kernel_variant = 1, 2
    # NVFP4 on the tensor cores keeps slot-ordered f16 rows of x in the workspace
    assert lib.moe_fp4_workspace_size(ctypes.byref(nv2), 4, 2) > lib.moe_fp4_workspace_size(ctypes.byref(nv1), 4, 2)
    assert lib.moe_fp4_expert_kernels(ctypes.byref(nv2), 4, 2) == 2
    assert lib.moe_fp4_expert_kernels(ctypes.byref(nv1), 4, 2) == 1
    assert lib.moe_fp4_expert_kernels(ctypes.byref(_weights(E=0)), 4, 2) == 0
    small_w, big_w = _weights(), _weights()
    small_w.kernel_variant, big_w.kernel_variant = 1, 2
    # the tensor-core variant keeps x and h as two-term E4M3 rows in the workspace
    assert lib.moe_fp4_workspace_size(ctypes.byref(big_w), 4, 2) != lib.moe_fp4_workspace_size(
        ctypes.byref(small_w), 4, 2)
    assert fwd(_weights(), nbytes=100) == 6
    w = _weights()
    assert lib.moe_fp4_workspace_size(ctypes.byref(w), 4, 2) > 0
    assert lib.moe_fp4_workspace_size(ctypes.byref(_weights(E=0)), 4, 2) == 0


def test_mma_scales_refusals():
    lib = L.load()
    ms = lambda rows, k, pair=0, src=P, dst=P: lib.fp4_mma_scales(src, rows, k, pair, dst, None)
    assert ms(0, 256) == 2
    assert ms(100, 256) == 5                  # rows not a multiple of 128
    assert ms(128, 200) == 5                  # k not a multiple of 128
    assert ms(3 * 96, 256, pair=96) == 5      # I not a multiple of 64
    assert ms(3 * 128, 256, pair=128) == 5    # rows not a multiple of 2I
    assert ms(128, 256, pair=-1) == 1
    assert ms(128, 256, src=None) == 1
    assert ms(128, 256, dst=ctypes.c_void_p(0x10008)) == 4


def test_nvfp4_mma_scales_refusals():
    lib = L.load()
    ms = lambda rows, k, pair=0, src=P, dst=P: lib.fp4_nvfp4_mma_scales(src, rows, k, pair, dst, None)
    assert ms(0, 256) == 2
    assert ms(100, 256) == 5                  # rows not a multiple of 128
    assert ms(128, 96) == 5                   # k not a multiple of 64
    assert ms(3 * 96, 256, pair=96) == 5      # I not a multiple of 64
    assert ms(128, 256, pair=-1) == 1
    assert ms(128, 256, src=None) == 1
    assert ms(128, 256, dst=ctypes.c_void_p(0x10008)) == 4


def test_v2a_pack_refusals():
    lib = L.load()
    ws = lambda b, r, k, n: lib.fp4_pack_v2a_workspace_size(b, r, k, n)
    assert ws(2, 64, 256, 4) > 0 and ws(2, 64, 256, 2) > 0
    assert ws(2, 64, 256, 3) == 0                   # only 2- and 4-bit codes pack a 128-group evenly
    assert ws(2, 16, 256, 4) == 0                   # fewer rows than library entries
    assert ws(2, 64, 200, 4) == 0                   # k not a multiple of 128
    pk = lambda b, r, k, n, thr=0.12, w=P, wsz=1 << 30: lib.fp4_pack_v2a(
        w, 0, b, r, k, n, thr, 0.0, P, P, P, P, P, P, P, wsz, None)
    assert pk(0, 64, 256, 4) == 2
    assert pk(1, 64, 200, 4) == 4
    assert pk(1, 64, 256, 3) == 1
    assert pk(1, 16, 256, 4) == 5
    assert pk(1, 64, 256, 4, thr=-1.0) == 1
    assert pk(1, 64, 256, 4, w=PMIS) == 4
    assert pk(1, 64, 256, 4, wsz=16) == 6


def test_cb4_pack_refusals():
    lib = L.load()
    rp = lambda rows, k, thr=0.12, mu=0.0, w=P, dt=L.FP4_F32: lib.fp4_cb4_row_ptr(w, dt, rows, k, thr, mu, P, None)
    assert rp(0, 128) == 2
    assert rp(4, 100) == 4                    # k not a multiple of 128
    assert rp(1 << 24, 1 << 8) == 3           # rows * k >= 2^31
    assert rp(4, 128, thr=-1.0) == 1
    assert rp(4, 128, thr=float("nan")) == 1
    assert rp(4, 128, mu=float("inf")) == 1
    assert rp(4, 128, w=None) == 1
    assert rp(4, 128, dt=7) == 1
    pk = lambda **kw: lib.fp4_pack_cb4(kw.get("w", P), L.FP4_F32, 4, 128, 0.12, 0.0, kw.get("rp", P),
                                       kw.get("idx", P), kw.get("cb", P), P, P, None)
    assert pk(rp=None) == 1
    assert pk(idx=ctypes.c_void_p(0x10004)) == 4
    assert pk(cb=None) == 1


def test_selftest_refusals():
    lib = L.load()
    assert lib.fp4_selftest_wait_timeout(None, 0, None) == 1
    assert lib.fp4_selftest_wait_timeout(P, 0, None) == 1
    assert lib.fp4_selftest_wait_timeout(P, 3_000_000_000, None) == 1


def test_linear_named_refusals():
    lib = L.load()
    lin = lambda fmt, T, K, N, ws=P: lib.fp4_linear(fmt, P, T, K, P, P, P, N, P, ws, 1 << 40, None)
    assert lin(L.FP4_MXFP4, 0, 256, 64) == 2
    assert lin(L.FP4_MXFP4, 4, 48, 64) == 4
    assert lin(L.FP4_MXFP4, 4, 256, 65) == 5
    assert lin(L.FP4_MXFP4, 4, 1 << 40, 64) == 3
    assert lin(L.FP4_MXFP4, 4, 256, 64, ws=None) == 6


def test_automatic_expert_kernels_follow_the_measured_crossovers():
    """kernel_variant 0: MXFP4 takes the tensor cores from 4 routed pairs per expert (or
    with prepared scale atoms), NVFP4 from 64 (below, the GEMV with 16-token units is
    faster than widening the weights on chip)."""
    lib = L.load()
    ek = lambda w, T, k: lib.moe_fp4_expert_kernels(ctypes.byref(w), T, k)   # noqa: E731
    nv, mx = _weights(fmt=L.FP4_NVFP4, E=8), _weights(fmt=L.FP4_MXFP4, E=8)
    assert ek(nv, 63, 8) == 1 and ek(nv, 64, 8) == 2
    assert ek(mx, 3, 8) == 1 and ek(mx, 4, 8) == 2
    mx.gu_mma_scales = mx.dn_mma_scales = 0x10000
    assert ek(mx, 1, 8) == 2
