"""Mixed-format fused expert buffers.

"The gate that missed by 0.0202 pp", section "A fused tensor with two dtypes in it": a
fused MoE buffer holds every expert of a layer in one tensor; an expert excluded from
quantisation is stored in bf16 and keeps its full row width (2K bytes), while a 4-bit
expert packs two values per byte (K/2 bytes per row).  A loader that slices the buffer
with one dtype and one stride for all experts is off by exactly that factor of two, so
the format and the offset belong to each expert.  This module lays such a buffer out
(expert_layout), packs one on the device with the library's own packers (pack_mixed), and
hands it to the layer with its per-expert tables (see fp4_moe_weights in
include/fp4moe.h: expert_format, *_offset, *_scale_offset).
"""
from __future__ import annotations

import torch

from . import _lib as L
from .api import MoEWeights, fp4_f32_to_bf16, fp4_pack


def expert_layout(formats, rows: int, K: int):
    """Byte offsets of each expert in the fused code buffer and in the fused scale buffer
    for per-expert ``formats`` ("mxfp4" or "bf16"): returns (offsets, scale_offsets,
    code_bytes, scale_bytes).  MXFP4 experts take rows * K/2 code bytes and rows * K/32
    scale bytes; bf16 experts take rows * 2K bytes and no scales (their scale offset is
    the running position, unused)."""
    off, soff, pos, spos = [], [], 0, 0
    for f in formats:
        off.append(pos)
        soff.append(spos)
        if f == "bf16":
            pos += rows * 2 * K
        elif f == "mxfp4":
            pos += rows * K // 2
            spos += rows * K // 32
        else:
            raise ValueError(f"unknown expert format {f!r}")
    return off, soff, pos, spos


def pack_mixed(w_gu: torch.Tensor, w_dn: torch.Tensor, bf16_experts, swiglu_limit: float = 7.0) -> MoEWeights:
    """Fused mixed-format weights of one layer from float32 device weights w_gu [E, 2I, H]
    and w_dn [E, H, I]: experts in ``bf16_experts`` are rounded to bf16 (kept out of
    quantisation), the others packed to MXFP4."""
    E, two_i, H = w_gu.shape
    I = two_i // 2
    dev = w_gu.device
    formats = ["bf16" if e in set(bf16_experts) else "mxfp4" for e in range(E)]
    out = {}
    for name, w, rows, K in (("gu", w_gu, 2 * I, H), ("dn", w_dn, H, I)):
        off, soff, nbytes, sbytes = expert_layout(formats, rows, K)
        codes = torch.empty(nbytes, dtype=torch.uint8, device=dev)
        scales = torch.zeros(max(sbytes, K // 32), dtype=torch.uint8, device=dev)   # never empty
        for e, f in enumerate(formats):
            if f == "bf16":
                codes[off[e]:off[e] + rows * 2 * K].copy_(fp4_f32_to_bf16(w[e].contiguous()).view(torch.uint8).view(-1))
            else:
                c, s, _ = fp4_pack(w[e].contiguous(), "mxfp4")
                codes[off[e]:off[e] + rows * K // 2].copy_(c.view(-1))
                scales[soff[e]:soff[e] + rows * K // 32].copy_(s.view(-1))
        out[name] = (codes, scales, torch.tensor(off, dtype=torch.int64, device=dev),
                     torch.tensor(soff, dtype=torch.int64, device=dev))
    fmt_codes = torch.tensor([L.FP4_DENSE_BF16 if f == "bf16" else L.FP4_MXFP4 for f in formats], dtype=torch.uint8,
                             device=dev)
    gu, dn = out["gu"], out["dn"]
    return MoEWeights("mxfp4", E, H, I, gu[0], gu[1], dn[0], dn[1], None, None, swiglu_limit, kernel_variant=1,
                      expert_format=fmt_codes, gu_offset=gu[2], gu_scale_offset=gu[3], dn_offset=dn[2],
                      dn_scale_offset=dn[3])
