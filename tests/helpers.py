"""Shared builders for the parity tests: seeded layers on the host (for the oracle)
and on the device (for the CUDA library), from the same counter-based synth recipe."""
from __future__ import annotations

import numpy as np

from synth import configs as C, draws as D

REL_FRO = 5e-3       # relative Frobenius error bound of a layer output (fixed gate)
ELEM_A = 2e-2        # per-element bound: |err| <= ELEM_A * (|ref| + 1)


def check_tolerance(got, ref, mask_rows=None):
    """Assert the fixed output gates; returns (rel_fro, max_elem_ratio).  When the
    environment names a file in FP4_PARITY_LOG, each call appends one line: the test id,
    the relative Frobenius error and the largest per-element error ratio."""
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    if mask_rows is not None:
        got, ref = got[mask_rows], ref[mask_rows]
    err = got - ref
    rel = np.linalg.norm(err) / max(np.linalg.norm(ref), 1e-300)
    ratio = np.max(np.abs(err) / (ELEM_A * (np.abs(ref) + 1.0))) if err.size else 0.0
    log = __import__("os").environ.get("FP4_PARITY_LOG")
    if log:
        case = __import__("os").environ.get("PYTEST_CURRENT_TEST", "?").split(" ")[0]
        with open(log, "a") as f:
            f.write(f"{case}\trel_fro={rel:.3e}\tmax_elem_ratio={ratio:.4f}\n")
    assert np.all(np.isfinite(got)), "non-finite output"
    assert rel <= REL_FRO, f"relative Frobenius error {rel:.3e} > {REL_FRO}"
    assert ratio <= 1.0, f"per-element error exceeds {ELEM_A}(|ref|+1) by factor {ratio:.3f}"
    return rel, ratio


def host_small_inputs(cfg):
    """x (bf16 bits), router weights and bias, drawn on the host."""
    x_bits = D.activations_bf16(cfg.seed, cfg.T, cfg.H)
    wr = D.router_weights(cfg.seed, cfg.E, cfg.H)
    bias = D.zipf_bias(cfg.seed, cfg.E) if cfg.zipf_bias else None
    return x_bits, wr, bias


def expert_host(cfg, which, e):
    """float32 weights of expert e: which = 'gu' -> [2I, H], 'dn' -> [H, I]."""
    if which == "gu":
        return D.expert_weights(cfg.seed, C.TID_GATE_UP, (cfg.E, 2 * cfg.I, cfg.H), start_row=e * 2 * cfg.I,
                                rows=2 * cfg.I, sigma=cfg.sigma, outliers=cfg.outliers)
    return D.expert_weights(cfg.seed, C.TID_DOWN, (cfg.E, cfg.H, cfg.I), start_row=e * cfg.H, rows=cfg.H,
                            sigma=cfg.sigma, outliers=cfg.outliers)


class LazyOracleBank:
    """Oracle expert bank that draws and quantises an expert only when it is used."""

    def __init__(self, cfg):
        from oracle import moe as M
        self.cfg = cfg
        self.E, self.H, self.I = cfg.E, cfg.H, cfg.I
        self._cache = {}
        self._M = M

    def packed(self, which, e):
        from oracle import codebook as CB, formats as F
        key = (which, e)
        if key not in self._cache:
            w = expert_host(self.cfg, which, e)
            if self.cfg.fmt == "cb4":
                self._cache[key] = CB.cb4_fit(w, self.cfg.cb4_threshold_sigma * self.cfg.sigma)
            elif self.cfg.fmt == "mxfp4":
                self._cache[key] = F.mxfp4_quantize(w) + (None,)
            else:
                c, s, t = F.nvfp4_quantize(w[None])
                self._cache[key] = (c[0], s[0], t[0])
        return self._cache[key]

    def dequant(self, which, e):
        from oracle import codebook as CB, formats as F
        if self.cfg.fmt == "cb4":
            fit = self.packed(which, e)
            n, k2 = fit["idx"].shape
            return CB.cb4_dense(fit["idx"], fit["cb_val"]) + CB.cb4_sparse(fit["row_ptr"], fit["col"], fit["val"],
                                                                           n, 2 * k2)
        c, s, t = self.packed(which, e)
        if self.cfg.fmt == "mxfp4":
            return F.mxfp4_dequantize(c, s)
        return F.nvfp4_dequantize(c, s, t)

    def apply_gate_up(self, e, x):
        return x @ self.dequant("gu", e).T

    def apply_down(self, e, h):
        return h @ self.dequant("dn", e).T


def device_weights_cb4(cfg, device="cuda"):
    """CB4 weights drawn on the device and packed there with fp4_pack_cb4 over each fused
    expert matrix ([E * rows, K]; one CSR per matrix)."""
    import torch
    from fp4_block_scaled_moe_b200 import MoEWeights, fp4_pack_cb4
    from synth import device as SD
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


def device_weights(cfg, device="cuda", chunk_elems=1 << 28):
    """Draw every expert's weights on the device and pack them there with fp4_pack."""
    import torch
    from fp4_block_scaled_moe_b200 import MoEWeights, fp4_pack
    from synth import device as SD
    if cfg.fmt == "cb4":
        return device_weights_cb4(cfg, device)
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
