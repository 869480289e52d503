"""Packed expert weights of the synthetic workloads, built on the device.

The weights are drawn on the GPU by the seeded generator in ``synth`` (the same
Student-t / planted-outlier draws the host makes) and packed there by this
library's own packers (fp4_pack, fp4_pack_cb4): nothing here quantises on the host.
Used by the benchmark and by the GPU tests.
"""
from __future__ import annotations

import torch

from synth import configs as C, device as SD

from .api import MoEWeights, fp4_pack, fp4_pack_cb4, fp4_pack_v2a


def device_weights_cb4(cfg, device="cuda"):
    """CB4 weights drawn on the device and packed there with fp4_pack_cb4 over each fused
    expert matrix ([E * rows, K]; one CSR per matrix)."""
    out = {}
    for which, tid, rows, K in (("gu", C.TID_GATE_UP, 2 * cfg.I, cfg.H), ("dn", C.TID_DOWN, cfg.H, cfg.I)):
        w = torch.empty((cfg.E * rows, K), dtype=torch.float32, device=device)
        SD.expert_weights_into(w, cfg.seed, tid, start_row=0, sigma=cfg.sigma, outliers=cfg.outliers)
        out[which] = fp4_pack_cb4(w, cfg.cb4_threshold_sigma * cfg.sigma)
        del w
    gu, dn = out["gu"], out["dn"]
    return MoEWeights(cfg.fmt, cfg.E, cfg.H, cfg.I, gu["idx"].view(cfg.E, 2 * cfg.I, cfg.H // 2), None,
                      dn["idx"].view(cfg.E, cfg.H, cfg.I // 2), None, None, None, cfg.swiglu_limit,
                      gu_cb=gu["cb"], gu_rowptr=gu["row_ptr"], gu_col=gu["col"], gu_val=gu["val"],
                      dn_cb=dn["cb"], dn_rowptr=dn["row_ptr"], dn_col=dn["col"], dn_val=dn["val"])


def device_weights_v2a(cfg, device="cuda"):
    """V2a weights (4-bit codes, one shared library per expert matrix) drawn and packed
    on the device with fp4_pack_v2a (one CSR per fused matrix)."""
    out = {}
    for which, tid, rows, K in (("gu", C.TID_GATE_UP, 2 * cfg.I, cfg.H), ("dn", C.TID_DOWN, cfg.H, cfg.I)):
        w = torch.empty((cfg.E * rows, K), dtype=torch.float32, device=device)
        SD.expert_weights_into(w, cfg.seed, tid, start_row=0, sigma=cfg.sigma, outliers=cfg.outliers)
        out[which] = fp4_pack_v2a(w.view(cfg.E, rows, K), cfg.v2a_bits, cfg.cb4_threshold_sigma * cfg.sigma)
        del w
    gu, dn = out["gu"], out["dn"]
    return MoEWeights(cfg.fmt, cfg.E, cfg.H, cfg.I, gu["codes"].view(cfg.E, 2 * cfg.I, -1),
                      gu["groups"].view(torch.uint8).view(cfg.E, 2 * cfg.I, -1),
                      dn["codes"].view(cfg.E, cfg.H, -1), dn["groups"].view(torch.uint8).view(cfg.E, cfg.H, -1),
                      None, None, cfg.swiglu_limit,
                      gu_cb=gu["lib"], gu_rowptr=gu["row_ptr"], gu_col=gu["col"], gu_val=gu["val"],
                      dn_cb=dn["lib"], dn_rowptr=dn["row_ptr"], dn_col=dn["col"], dn_val=dn["val"])


def device_weights_mixed(cfg, device="cuda"):
    """A mixed-format fused buffer: the experts in cfg.bf16_experts kept in bf16, the rest
    MXFP4 (see mixed.py)."""
    from .mixed import pack_mixed
    ws = {}
    for which, tid, rows, K in (("gu", C.TID_GATE_UP, 2 * cfg.I, cfg.H), ("dn", C.TID_DOWN, cfg.H, cfg.I)):
        w = torch.empty((cfg.E, rows, K), dtype=torch.float32, device=device)
        SD.expert_weights_into(w.view(cfg.E * rows, K), cfg.seed, tid, start_row=0, sigma=cfg.sigma,
                               outliers=cfg.outliers)
        ws[which] = w
    return pack_mixed(ws["gu"], ws["dn"], cfg.bf16_experts, cfg.swiglu_limit)


def device_weights(cfg, device="cuda", chunk_elems=1 << 28):
    """Draw every expert's weights of ``cfg`` on the device and pack them there."""
    if cfg.fmt == "mixed":
        return device_weights_mixed(cfg, device)
    if cfg.fmt == "cb4":
        return device_weights_cb4(cfg, device)
    if cfg.fmt == "v2a":
        return device_weights_v2a(cfg, device)
    B = 32 if cfg.fmt == "mxfp4" else 16
    out = {}
    for which, tid, rows, K in (("gu", C.TID_GATE_UP, 2 * cfg.I, cfg.H), ("dn", C.TID_DOWN, cfg.H, cfg.I)):
        codes = torch.empty((cfg.E, rows, K // 2), dtype=torch.uint8, device=device)
        scales = torch.empty((cfg.E, rows, K // B), dtype=torch.uint8, device=device)
        ts = torch.empty((cfg.E,), dtype=torch.float32, device=device) if cfg.fmt == "nvfp4" else None
        per = max(1, chunk_elems // (rows * K))
        buf = torch.empty((min(per, cfg.E), rows, K), dtype=torch.float32, device=device)
        for e0 in range(0, cfg.E, per):
            n = min(per, cfg.E - e0)
            w = buf[:n]
            SD.expert_weights_into(w.view(n * rows, K), cfg.seed, tid, start_row=e0 * rows, sigma=cfg.sigma,
                                   outliers=cfg.outliers)
            c, s, t = fp4_pack(w, cfg.fmt)
            codes[e0:e0 + n].copy_(c)
            scales[e0:e0 + n].copy_(s)
            if ts is not None:
                ts[e0:e0 + n].copy_(t)
        del buf
        out[which] = (codes, scales, ts)
    return MoEWeights(cfg.fmt, cfg.E, cfg.H, cfg.I, out["gu"][0], out["gu"][1], out["dn"][0], out["dn"][1],
                      out["gu"][2], out["dn"][2], cfg.swiglu_limit)
