"""Python binding of the fp4moe C ABI (same names as include/fp4moe.h).

PyTorch supplies device memory and the current stream; every computation runs
in the library's CUDA kernels. Tensors must be CUDA, contiguous, and of the
dtype each function states.
"""
from __future__ import annotations

import ctypes
from dataclasses import dataclass

import torch

from . import _lib as L


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(device=None):
    return ctypes.c_void_p(torch.cuda.current_stream(device).cuda_stream)


def _need(t, name, dtype=None, cuda=True):
    if t is None:
        raise ValueError(f"{name} is required")
    if cuda and not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if dtype is not None and t.dtype != dtype:
        raise ValueError(f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")


def fmt_code(fmt):
    return L.FORMATS[fmt] if isinstance(fmt, str) else int(fmt)


def fp4_pack(w: torch.Tensor, fmt="mxfp4"):
    """Quantise w [..., n, k] (float32 or bf16). Returns (codes, scales, tensor_scale or None)."""
    lib = L.load()
    f = fmt_code(fmt)
    _need(w, "w")
    if w.dtype not in (torch.float32, torch.bfloat16):
        raise ValueError("w must be float32 or bfloat16")
    *lead, n, k = w.shape
    batch = 1
    for d in lead:
        batch *= d
    B = L.BLOCK.get(f, 32)
    codes = torch.empty((*lead, n, max(k // 2, 1)), dtype=torch.uint8, device=w.device)
    scales = torch.empty((*lead, n, max(k // B, 1)), dtype=torch.uint8, device=w.device)
    ts = torch.empty(tuple(lead) if lead else (1,), dtype=torch.float32, device=w.device) if f == L.FP4_NVFP4 else None
    dt = L.FP4_F32 if w.dtype == torch.float32 else L.FP4_BF16
    L.check("fp4_pack", lib.fp4_pack(f, _ptr(w), dt, batch, n, k, _ptr(codes), _ptr(scales), _ptr(ts),
                                     _stream(w.device)))
    return codes, scales, ts


def fp4_mma_scales(scales: torch.Tensor, pair: int = 0) -> torch.Tensor:
    """MXFP4 scales [..., rows, k/32] re-laid as tensor-core scale atoms (flat uint8);
    pair = I for gate_up weights (tiles of 64 gate + 64 up rows), 0 for down weights."""
    _need(scales, "scales", torch.uint8)
    k = scales.shape[-1] * 32
    rows = scales.numel() // scales.shape[-1]
    out = torch.empty(scales.numel(), dtype=torch.uint8, device=scales.device)
    L.check("fp4_mma_scales", L.load().fp4_mma_scales(_ptr(scales), rows, k, pair, _ptr(out), _stream(scales.device)))
    return out


def fp4_nvfp4_mma_scales(scales: torch.Tensor, pair: int = 0) -> torch.Tensor:
    """NVFP4 scales [..., rows, k/16] re-laid as the tensor-core kernels' 512-byte atoms
    (flat uint8); pair = I for gate_up weights, 0 for down weights."""
    _need(scales, "scales", torch.uint8)
    k = scales.shape[-1] * 16
    rows = scales.numel() // scales.shape[-1]
    out = torch.empty(scales.numel(), dtype=torch.uint8, device=scales.device)
    L.check("fp4_nvfp4_mma_scales", L.load().fp4_nvfp4_mma_scales(_ptr(scales), rows, k, pair, _ptr(out),
                                                                   _stream(scales.device)))
    return out


def prepare_mma_scales(weights: "MoEWeights") -> "MoEWeights":
    """Attach re-laid gate_up / down scales to MXFP4 or NVFP4 weights for the tensor-core
    kernels (a one-time preparation; without it each call re-lays them)."""
    relay = fp4_mma_scales if weights.fmt == "mxfp4" else fp4_nvfp4_mma_scales
    if weights.fmt not in ("mxfp4", "nvfp4"):
        raise ValueError("tensor-core scale atoms exist for MXFP4 and NVFP4 weights only")
    weights.gu_mma_scales = relay(weights.gu_scales, pair=weights.I)
    weights.dn_mma_scales = relay(weights.dn_scales)
    return weights


def fp4_pack_cb4(w: torch.Tensor, threshold: float, mu: float = 0.0):
    """CB4 pack of w [rows, k] (float32 or bf16): returns dict(idx, cb, row_ptr, col, val)
    (see fp4_cb4_row_ptr / fp4_pack_cb4 in include/fp4moe.h)."""
    lib = L.load()
    _need(w, "w")
    if w.dtype not in (torch.float32, torch.bfloat16):
        raise ValueError("w must be float32 or bfloat16")
    w2 = w.reshape(-1, w.shape[-1])
    rows, k = w2.shape
    dt = L.FP4_F32 if w.dtype == torch.float32 else L.FP4_BF16
    dev = w.device
    row_ptr = torch.empty(rows + 1, dtype=torch.int32, device=dev)
    L.check("fp4_cb4_row_ptr", lib.fp4_cb4_row_ptr(_ptr(w2), dt, rows, k, float(threshold), float(mu), _ptr(row_ptr),
                                                   _stream(dev)))
    nnz = int(row_ptr[-1].item())
    idx = torch.empty((rows, k // 2), dtype=torch.uint8, device=dev)
    cb = torch.empty((rows, k // 128, 16), dtype=torch.int16, device=dev)
    col = torch.empty(max(nnz, 1), dtype=torch.int32, device=dev)
    val = torch.empty(max(nnz, 1), dtype=torch.int16, device=dev)
    L.check("fp4_pack_cb4", lib.fp4_pack_cb4(_ptr(w2), dt, rows, k, float(threshold), float(mu), _ptr(row_ptr),
                                             _ptr(idx), _ptr(cb), _ptr(col), _ptr(val), _stream(dev)))
    return {"idx": idx, "cb": cb, "row_ptr": row_ptr, "col": col[:nnz], "val": val[:nnz]}


def fp4_pack_v2a(w: torch.Tensor, n_bits: int, threshold: float, mu: float = 0.0):
    """V2a pack of w [rows, k] or [batch, rows, k] (float32 or bf16), one 32-codebook
    library per matrix: returns dict(codes, groups, lib, row_ptr, col, val) (see
    fp4_pack_v2a in include/fp4moe.h); groups are int64 records [batch * rows, k / 128]."""
    lib_ = L.load()
    _need(w, "w")
    if w.dtype not in (torch.float32, torch.bfloat16):
        raise ValueError("w must be float32 or bfloat16")
    w3 = w.reshape(-1, w.shape[-2], w.shape[-1]) if w.dim() >= 2 else w
    batch, rows, k = w3.shape
    dt = L.FP4_F32 if w.dtype == torch.float32 else L.FP4_BF16
    dev = w.device
    R = batch * rows
    row_ptr = torch.empty(R + 1, dtype=torch.int32, device=dev)
    L.check("fp4_cb4_row_ptr", lib_.fp4_cb4_row_ptr(_ptr(w3), dt, R, k, float(threshold), float(mu), _ptr(row_ptr),
                                                    _stream(dev)))
    nnz = int(row_ptr[-1].item())
    codes = torch.empty((R, k * n_bits // 8), dtype=torch.uint8, device=dev)
    groups = torch.empty((R, k // 128), dtype=torch.int64, device=dev)
    lib = torch.empty((batch, 32, 1 << n_bits), dtype=torch.int16, device=dev)
    col = torch.empty(max(nnz, 1), dtype=torch.int32, device=dev)
    val = torch.empty(max(nnz, 1), dtype=torch.int16, device=dev)
    need = int(lib_.fp4_pack_v2a_workspace_size(batch, rows, k, n_bits))
    if need == 0:
        raise L.FP4Error("fp4_pack_v2a_workspace_size", 5, "unsupported shape")
    ws = alloc_workspace(need, dev)
    L.check("fp4_pack_v2a", lib_.fp4_pack_v2a(_ptr(w3), dt, batch, rows, k, n_bits, float(threshold), float(mu),
                                              _ptr(row_ptr), _ptr(codes), _ptr(groups), _ptr(lib), _ptr(col),
                                              _ptr(val), _ptr(ws), ws.numel(), _stream(dev)))
    return {"codes": codes, "groups": groups, "lib": lib, "row_ptr": row_ptr, "col": col[:nnz], "val": val[:nnz]}


def fp4_unpack_v2a(codes, groups, lib, batch, rows, k, n_bits):
    """Dense V2a term as float32 [batch, rows, k] (exact fp16 values)."""
    out = torch.empty((batch, rows, k), dtype=torch.float32, device=codes.device)
    L.check("fp4_unpack_v2a", L.load().fp4_unpack_v2a(_ptr(codes), _ptr(groups), _ptr(lib), batch, rows, k, n_bits,
                                                      _ptr(out), _stream(codes.device)))
    return out


def fp4_unpack(codes, scales, tensor_scale=None, fmt="mxfp4", out_dtype=torch.float32):
    lib = L.load()
    f = fmt_code(fmt)
    _need(codes, "codes", torch.uint8)
    _need(scales, "scales", torch.uint8)
    *lead, n, k2 = codes.shape
    batch = 1
    for d in lead:
        batch *= d
    out = torch.empty((*lead, n, k2 * 2), dtype=out_dtype, device=codes.device)
    dt = L.FP4_F32 if out_dtype == torch.float32 else L.FP4_BF16
    L.check("fp4_unpack", lib.fp4_unpack(f, _ptr(codes), _ptr(scales), _ptr(tensor_scale), batch, n, k2 * 2,
                                         _ptr(out), dt, _stream(codes.device)))
    return out


def moe_route(x, router_w, router_bias, k, logits_in=None):
    """Router. x [T, H] bf16, router_w [E, H] f32. Returns a dict of device tensors."""
    lib = L.load()
    if logits_in is not None:
        _need(logits_in, "logits_in", torch.float32)
        T, E = logits_in.shape
        H = x.shape[1] if x is not None else 0
        dev = logits_in.device
    else:
        _need(x, "x", torch.bfloat16)
        _need(router_w, "router_w", torch.float32)
        T, H = x.shape
        E = router_w.shape[0]
        dev = x.device
    i32 = dict(dtype=torch.int32, device=dev)
    out = dict(
        logits=torch.empty((T, E), dtype=torch.float32, device=dev),
        topk_ids=torch.empty((T, k), **i32),
        topk_w=torch.empty((T, k), dtype=torch.float32, device=dev),
        counts=torch.empty((E,), **i32),
        offsets=torch.empty((E + 1,), **i32),
        perm=torch.empty((T * k,), **i32),
        inv=torch.empty((T * k,), **i32),
    )
    L.check("moe_route", lib.moe_route(_ptr(x), _ptr(router_w), _ptr(router_bias), T, H, E, k, _ptr(logits_in),
                                       _ptr(out["logits"]), _ptr(out["topk_ids"]), _ptr(out["topk_w"]),
                                       _ptr(out["counts"]), _ptr(out["offsets"]), _ptr(out["perm"]),
                                       _ptr(out["inv"]), _stream(dev)))
    return out


@dataclass
class MoEWeights:
    """Device tensors of one MoE layer (see fp4_moe_weights in include/fp4moe.h)."""
    fmt: str
    E: int
    H: int
    I: int
    gu_codes: torch.Tensor
    gu_scales: torch.Tensor
    dn_codes: torch.Tensor
    dn_scales: torch.Tensor
    gu_tscale: torch.Tensor | None = None
    dn_tscale: torch.Tensor | None = None
    swiglu_limit: float = 7.0
    gu_cb: torch.Tensor | None = None
    gu_rowptr: torch.Tensor | None = None
    gu_col: torch.Tensor | None = None
    gu_val: torch.Tensor | None = None
    dn_cb: torch.Tensor | None = None
    dn_rowptr: torch.Tensor | None = None
    dn_col: torch.Tensor | None = None
    dn_val: torch.Tensor | None = None
    # expert-GEMM kernels: 0 chosen per call, 1 CUDA-core GEMV, 2 tensor-core (MXFP4)
    kernel_variant: int = 0
    # tensor-core kernels: scales re-laid by fp4_mma_scales (else re-laid every call)
    gu_mma_scales: torch.Tensor | None = None
    dn_mma_scales: torch.Tensor | None = None
    # expert parallelism: these tensors hold experts [expert_begin, expert_begin + local_experts)
    # of the E routed experts (0, 0: all of them)
    expert_begin: int = 0
    local_experts: int = 0
    # mixed-format fused buffers (see mixed.py): per-expert format and byte offsets
    expert_format: torch.Tensor | None = None
    gu_offset: torch.Tensor | None = None
    gu_scale_offset: torch.Tensor | None = None
    dn_offset: torch.Tensor | None = None
    dn_scale_offset: torch.Tensor | None = None

    def c_struct(self):
        s = L.MoEWeightsC()
        s.fmt = fmt_code(self.fmt)
        s.num_experts, s.hidden, s.inter = self.E, self.H, self.I
        s.swiglu_limit = self.swiglu_limit
        s.kernel_variant = self.kernel_variant
        s.expert_begin, s.local_experts = self.expert_begin, self.local_experts
        if self.expert_format is not None:
            s.gu_bytes, s.dn_bytes = self.gu_codes.numel(), self.dn_codes.numel()
            s.gu_scale_bytes, s.dn_scale_bytes = self.gu_scales.numel(), self.dn_scales.numel()
        for name in ("gu_codes", "gu_scales", "gu_tscale", "dn_codes", "dn_scales", "dn_tscale", "gu_cb",
                     "gu_rowptr", "gu_col", "gu_val", "dn_cb", "dn_rowptr", "dn_col", "dn_val", "gu_mma_scales",
                     "dn_mma_scales", "expert_format", "gu_offset", "gu_scale_offset", "dn_offset",
                     "dn_scale_offset"):
            t = getattr(self, name)
            setattr(s, name, None if t is None else t.data_ptr())
        return s


def moe_fp4_workspace_size(weights: MoEWeights, T: int, k: int) -> int:
    s = weights.c_struct()
    return int(L.load().moe_fp4_workspace_size(ctypes.byref(s), T, k))


def moe_fp4_expert_kernels(weights: MoEWeights, T: int, k: int) -> int:
    """Expert kernels the library runs for this call shape: 1 CUDA-core GEMV, 2 tensor cores."""
    s = weights.c_struct()
    return int(L.load().moe_fp4_expert_kernels(ctypes.byref(s), T, k))


def alloc_workspace(nbytes: int, device) -> torch.Tensor:
    """A 256-byte aligned, zero-filled device buffer (torch allocations are 512-byte
    aligned; zero-filled so that the control block's timing fields start valid)."""
    return torch.zeros(max(int(nbytes), 256), dtype=torch.uint8, device=device)


def moe_fp4_forward(weights: MoEWeights, x, router_w, router_bias, k, workspace=None, route_out=None,
                    y=None, _struct=None):
    """y [T, H] bf16 = MoE layer(x). ``route_out``: optional dict of tensors receiving routing results."""
    lib = L.load()
    _need(x, "x", torch.bfloat16)
    _need(router_w, "router_w", torch.float32)
    T = x.shape[0]
    s = _struct if _struct is not None else weights.c_struct()
    need = int(lib.moe_fp4_workspace_size(ctypes.byref(s), T, k))
    if workspace is None:
        if need == 0:
            raise L.FP4Error("moe_fp4_workspace_size", 1, "invalid layer arguments")
        workspace = alloc_workspace(need, x.device)
    if y is None:
        y = torch.empty((T, weights.H), dtype=torch.bfloat16, device=x.device)
    ro = None
    if route_out is not None:
        ro = L.RouteOutC()
        for name in ("logits", "topk_ids", "topk_w", "counts", "offsets", "perm", "inv"):
            t = route_out.get(name)
            setattr(ro, name, None if t is None else t.data_ptr())
    L.check("moe_fp4_forward", lib.moe_fp4_forward(ctypes.byref(s), _ptr(x), _ptr(router_w), _ptr(router_bias),
                                                   T, k, _ptr(y), ctypes.byref(ro) if ro is not None else None,
                                                   _ptr(workspace), workspace.numel(), _stream(x.device)))
    return y


def moe_fp4_forward_partial(weights: MoEWeights, x, router_w, router_bias, k, workspace=None, route_out=None,
                            y_partial=None):
    """float32 [T, H] sum over the slots routed to this shard's experts (expert parallelism;
    see moe_fp4_forward_partial in include/fp4moe.h)."""
    lib = L.load()
    _need(x, "x", torch.bfloat16)
    _need(router_w, "router_w", torch.float32)
    T = x.shape[0]
    s = weights.c_struct()
    need = int(lib.moe_fp4_workspace_size(ctypes.byref(s), T, k))
    if workspace is None:
        if need == 0:
            raise L.FP4Error("moe_fp4_workspace_size", 1, "invalid layer arguments")
        workspace = alloc_workspace(need, x.device)
    if y_partial is None:
        y_partial = torch.empty((T, weights.H), dtype=torch.float32, device=x.device)
    ro = None
    if route_out is not None:
        ro = L.RouteOutC()
        for name in ("logits", "topk_ids", "topk_w", "counts", "offsets", "perm", "inv"):
            t = route_out.get(name)
            setattr(ro, name, None if t is None else t.data_ptr())
    L.check("moe_fp4_forward_partial", lib.moe_fp4_forward_partial(
        ctypes.byref(s), _ptr(x), _ptr(router_w), _ptr(router_bias), T, k, _ptr(y_partial),
        ctypes.byref(ro) if ro is not None else None, _ptr(workspace), workspace.numel(), _stream(x.device)))
    return y_partial


def fp4_f32_to_bf16(x: torch.Tensor, out=None) -> torch.Tensor:
    """bf16 copy of a float32 tensor, rounded by the library (nearest even)."""
    _need(x, "x", torch.float32)
    if out is None:
        out = torch.empty(x.shape, dtype=torch.bfloat16, device=x.device)
    L.check("fp4_f32_to_bf16", L.load().fp4_f32_to_bf16(_ptr(x), x.numel(), _ptr(out), _stream(x.device)))
    return out


def fp4_linear(x, codes, scales, tensor_scale=None, fmt="mxfp4", workspace=None, y=None):
    """y [T, N] bf16 = x [T, K] bf16 . W^T with W [N, K] in MXFP4 / NVFP4."""
    lib = L.load()
    _need(x, "x", torch.bfloat16)
    T, K = x.shape
    N = codes.shape[0]
    need = int(lib.fp4_linear_workspace_size(T, K))
    if workspace is None:
        workspace = alloc_workspace(need, x.device)
    if y is None:
        y = torch.empty((T, N), dtype=torch.bfloat16, device=x.device)
    L.check("fp4_linear", lib.fp4_linear(fmt_code(fmt), _ptr(x), T, K, _ptr(codes), _ptr(scales), _ptr(tensor_scale),
                                         N, _ptr(y), _ptr(workspace), workspace.numel(), _stream(x.device)))
    return y


def fp4_launch_count() -> int:
    """Kernel launches the library has issued in this process (see include/fp4moe.h)."""
    return int(L.load().fp4_launch_count())


def fp4_selftest_wait_timeout(workspace, limit_ns: int = 1_000_000):
    """Run the bounded-wait failure path once (see include/fp4moe.h)."""
    L.check("fp4_selftest_wait_timeout", L.load().fp4_selftest_wait_timeout(_ptr(workspace), int(limit_ns),
                                                                           _stream(workspace.device)))


def fp4_workspace_status(workspace) -> str:
    code = L.load().fp4_workspace_status(_ptr(workspace), _stream(workspace.device))
    return L.STATUS.get(code, str(code))


def fp4_workspace_kernel_stats(workspace, reset=False) -> dict:
    """Device time of the grouped expert kernels accumulated in ``workspace`` (see header)."""
    st = L.KernelStatsC()
    L.check("fp4_workspace_kernel_stats", L.load().fp4_workspace_kernel_stats(
        _ptr(workspace), 1 if reset else 0, ctypes.byref(st), _stream(workspace.device)))
    return {"gate_up_ns": st.gate_up_ns, "gate_up_launches": st.gate_up_launches,
            "down_ns": st.down_ns, "down_launches": st.down_launches}


def moe_fp4_forward_noalloc(weights: MoEWeights, x, router_w, router_bias, k, y=None):
    """The MoE layer without a caller workspace: scratch comes from the library's fixed
    device buffer (see moe_fp4_forward_noalloc in include/fp4moe.h)."""
    lib = L.load()
    _need(x, "x", torch.bfloat16)
    _need(router_w, "router_w", torch.float32)
    T = x.shape[0]
    s = weights.c_struct()
    if y is None:
        y = torch.empty((T, weights.H), dtype=torch.bfloat16, device=x.device)
    L.check("moe_fp4_forward_noalloc", lib.moe_fp4_forward_noalloc(
        ctypes.byref(s), _ptr(x), _ptr(router_w), _ptr(router_bias), T, k, _ptr(y), _stream(x.device)))
    return y


def moe_fp4_noalloc_status() -> str:
    """Status word of the no-alloc scratch on the current device (read and cleared)."""
    code = L.load().moe_fp4_noalloc_status(_stream())
    return L.STATUS.get(code, str(code))
