"""Shared builders for the parity tests: seeded layers on the host (for the oracle)
and on the device (for the CUDA library), from the same counter-based synth recipe."""
from __future__ import annotations

import functools
import os

import numpy as np

from synth import configs as C, draws as D

REL_FRO = 5e-3       # relative Frobenius error bound of a layer output (fixed gate)
ELEM_A = 2e-2        # per-element bound: |err| <= ELEM_A * (|ref| + 1)


def tolerance_stats(got, ref):
    """(relative Frobenius error, largest |err| / (ELEM_A (|ref| + 1)), all finite)."""
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    err = got - ref
    rel = np.linalg.norm(err) / max(np.linalg.norm(ref), 1e-300)
    with np.errstate(invalid="ignore"):
        ratio = np.max(np.abs(err) / (ELEM_A * (np.abs(ref) + 1.0))) if err.size else 0.0
    return rel, ratio, bool(np.all(np.isfinite(got)))


def within_gates(got, ref):
    """True when ``got`` passes the fixed output gates against ``ref``."""
    rel, ratio, fin = tolerance_stats(got, ref)
    return fin and rel <= REL_FRO and ratio <= 1.0


def parity_log(line):
    """Append one line to the file named by FP4_PARITY_LOG (if set), prefixed by the test id."""
    log = os.environ.get("FP4_PARITY_LOG")
    if log:
        case = os.environ.get("PYTEST_CURRENT_TEST", "?").split(" ")[0]
        with open(log, "a") as f:
            f.write(f"{case}\t{line}\n")


def check_tolerance(got, ref, mask_rows=None):
    """Assert the fixed output gates; returns (rel_fro, max_elem_ratio).  When the
    environment names a file in FP4_PARITY_LOG, each call appends one line: the test id,
    the relative Frobenius error and the largest per-element error ratio."""
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    if mask_rows is not None:
        got, ref = got[mask_rows], ref[mask_rows]
    rel, ratio, fin = tolerance_stats(got, ref)
    parity_log(f"rel_fro={rel:.3e}\tmax_elem_ratio={ratio:.4f}")
    assert fin, "non-finite output"
    assert rel <= REL_FRO, f"relative Frobenius error {rel:.3e} > {REL_FRO}"
    assert ratio <= 1.0, f"per-element error exceeds {ELEM_A}(|ref|+1) by factor {ratio:.3f}"
    return rel, ratio


def host_small_inputs(cfg, x_scale=1.0):
    """x (bf16 bits), router weights and bias, drawn on the host.  ``x_scale`` (a power
    of two, so the bf16 values scale exactly) widens the activations."""
    x_bits = D.activations_bf16(cfg.seed, cfg.T, cfg.H)
    if x_scale != 1.0:
        assert np.log2(x_scale) == int(np.log2(x_scale))
        x_bits = D.f32_to_bf16_bits(D.bf16_bits_to_f32(x_bits) * np.float32(x_scale))
    wr = D.router_weights(cfg.seed, cfg.E, cfg.H)
    bias = D.zipf_bias(cfg.seed, cfg.E) if cfg.zipf_bias else None
    return x_bits, wr, bias


def expert_host(cfg, which, e):
    """float32 weights of expert e: which = 'gu' -> [2I, H], 'dn' -> [H, I]."""
    return C.expert_rows(cfg, which, e)


def oracle_bank(cfg):
    """The oracle's lazily quantised expert bank for a workload (host draws)."""
    from oracle import moe as M
    return M.LazyExpertBank(cfg.fmt, cfg.E, cfg.H, cfg.I, draw=functools.partial(C.expert_rows, cfg),
                            cb4_threshold=cfg.cb4_threshold_sigma * cfg.sigma, v2a_bits=cfg.v2a_bits,
                            bf16_experts=cfg.bf16_experts)


LazyOracleBank = oracle_bank


def device_weights(cfg, device="cuda"):
    """Every expert drawn and packed on the device by the library (see workloads.py)."""
    from fp4_block_scaled_moe_b200.workloads import device_weights as dw
    return dw(cfg, device=device)
