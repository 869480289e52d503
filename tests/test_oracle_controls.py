"""Planted controls on the CPU: each plausible mistake (tests/controls.py), planted into
the oracle, turns the fixed output gates red against the unmodified oracle on the same
inputs the GPU parity tests use.  This pins the gates' power to catch those mistakes
without relying on the GPU path."""
import numpy as np
import pytest

from oracle import routing as R
from synth import configs as C, draws as D

from controls import corrupt_oracle
from helpers import host_small_inputs, within_gates
from oracle_pool import moe_reference

CLAMP_X_SCALE = 16.0


def _ref(cfg, x_scale=1.0, limit=None, corrupt=None):
    x_bits, wr, bias = host_small_inputs(cfg, x_scale)
    xf = D.bf16_bits_to_f32(x_bits)
    lg = R.router_logits(xf, wr, bias)
    ids = R.topk(lg, cfg.k)
    y, st = moe_reference(cfg, xf, ids, R.softmax_selected(lg, ids), limit=limit, parallel=False, corrupt=corrupt)
    return y, st


_PLANTS = [("scale_byte", "mxfp4"), ("scale_byte", "nvfp4"), ("nibble_swap", "mxfp4"), ("nibble_swap", "nvfp4"),
           ("skip_tensor_scale", "nvfp4")]


@pytest.mark.parametrize("control,fmt", _PLANTS, ids=[f"{c}_{f}" for c, f in _PLANTS])
def test_planted_weight_mistake_turns_gate_red(control, fmt):
    cfg = C.small({"mxfp4": C.MOE_C2, "nvfp4": C.MOE_C3}[fmt])
    clean, _ = _ref(cfg)
    bad, _ = _ref(cfg, corrupt=corrupt_oracle(control, fmt))
    assert within_gates(clean, clean)
    assert not within_gates(bad, clean), f"{control} planted in {fmt} stays within the gates"


@pytest.mark.parametrize("fmt", ["mxfp4", "nvfp4", "cb4"])
def test_dropped_clamp_turns_gate_red(fmt):
    cfg = C.small({"mxfp4": C.MOE_C2, "nvfp4": C.MOE_C3, "cb4": C.MOE_C5}[fmt])
    clean, st = _ref(cfg, CLAMP_X_SCALE)
    assert st["g_clamped"] >= 0.1 * st["pairs"] and st["u_clamped"] >= 0.1 * st["pairs"]
    bad, _ = _ref(cfg, CLAMP_X_SCALE, limit=128.0)
    assert not within_gates(bad, clean)


def test_clamp_never_fires_on_the_plain_workload_inputs():
    """Why the clamp tests scale x: on the N(0, 1) workload activations no pair reaches
    the clamp, so those cases cannot tell a missing clamp apart."""
    for base in (C.MOE_C2, C.MOE_C3):
        _, st = _ref(C.small(base))
        assert st["g_clamped"] == 0 and st["u_clamped"] == 0
