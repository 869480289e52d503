"""Planted controls through the C ABI: the same mistakes as tests/controls.py, planted
into the packed weights on the device (data only; the kernels are untouched) or into
the layer's clamp limit, must make the GPU output fail the fixed gates against the
unmodified oracle, while the clean run on the same inputs passes."""
import numpy as np
import pytest
import torch

from oracle import routing as R
from synth import configs as C, draws as D

from controls import bump_scale_byte, swap_nibbles
from helpers import device_weights, host_small_inputs, within_gates
from oracle_pool import moe_reference

pytestmark = pytest.mark.gpu


def _run(cfg, plant=None, x_scale=1.0, variant=0):
    from fp4_block_scaled_moe_b200 import moe_fp4_forward
    x_bits, wr, bias = host_small_inputs(cfg, x_scale)
    w = device_weights(cfg)
    w.kernel_variant = variant
    if plant == "scale_byte":
        s = w.gu_scales.cpu().numpy()
        for e in range(cfg.E):
            s[e, 0, 0] = bump_scale_byte(s[e, 0, 0], cfg.fmt)
        w.gu_scales.copy_(torch.from_numpy(s))
    elif plant == "nibble_swap":
        w.gu_codes.copy_(torch.from_numpy(swap_nibbles(w.gu_codes.cpu().numpy())))
        w.dn_codes.copy_(torch.from_numpy(swap_nibbles(w.dn_codes.cpu().numpy())))
    elif plant == "skip_tensor_scale":
        w.gu_tscale.fill_(1.0)
        w.dn_tscale.fill_(1.0)
    elif plant == "drop_clamp":
        w.swiglu_limit = 128.0
    x = torch.from_numpy(x_bits.view(np.int16)).cuda().view(torch.bfloat16)
    y = moe_fp4_forward(w, x, torch.from_numpy(wr).cuda(), None if bias is None else torch.from_numpy(bias).cuda(),
                        cfg.k)
    torch.cuda.synchronize()
    got = D.bf16_bits_to_f32(y.view(torch.int16).cpu().numpy().view(np.uint16)).reshape(cfg.T, cfg.H)
    xf = D.bf16_bits_to_f32(x_bits)
    lg = R.router_logits(xf, wr, bias)
    ids = R.topk(lg, cfg.k)
    ref, _ = moe_reference(cfg, xf, ids, R.softmax_selected(lg, ids), parallel=False)
    return got, ref


_CASES = [("scale_byte", "mxfp4", 1), ("scale_byte", "mxfp4", 2), ("scale_byte", "nvfp4", 1),
          ("nibble_swap", "mxfp4", 1), ("nibble_swap", "mxfp4", 2), ("nibble_swap", "nvfp4", 1),
          ("skip_tensor_scale", "nvfp4", 1), ("drop_clamp", "mxfp4", 1), ("drop_clamp", "mxfp4", 2),
          ("drop_clamp", "nvfp4", 1), ("scale_byte", "nvfp4", 2), ("nibble_swap", "nvfp4", 2),
          ("skip_tensor_scale", "nvfp4", 2), ("drop_clamp", "nvfp4", 2)]


@pytest.mark.parametrize("plant,fmt,variant", _CASES, ids=[f"{p}_{f}_v{v}" for p, f, v in _CASES])
def test_planted_control_is_red(plant, fmt, variant):
    cfg = C.small({"mxfp4": C.MOE_C2, "nvfp4": C.MOE_C3}[fmt])
    xs = 16.0 if plant == "drop_clamp" else 1.0
    got, ref = _run(cfg, None, xs, variant)
    assert within_gates(got, ref), "the clean run must pass"
    got, ref = _run(cfg, plant, xs, variant)
    assert not within_gates(got, ref), f"{plant} planted on the device stays within the gates"
