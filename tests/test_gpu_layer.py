"""Layer outputs on the GPU against the float64 oracle, within the fixed gates:
relative Frobenius error <= 5e-3 and |err| <= 2e-2 (|ref| + 1) per element."""
import numpy as np
import pytest
import torch

from oracle import formats as F, moe as M, routing as R
from synth import configs as C, draws as D

from helpers import LazyOracleBank, check_tolerance, device_weights, host_small_inputs

pytestmark = pytest.mark.gpu


def _bf16_dev(bits):
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).cuda().view(torch.bfloat16)


def _y_host(y):
    return D.bf16_bits_to_f32(y.view(torch.int16).cpu().numpy().view(np.uint16)).reshape(y.shape)


@pytest.mark.parametrize("cfg", [C.small(C.LINEAR_C1), C.LINEAR_C1,
                                 C.small(C.LinearConfig("linear_nvfp4", "nvfp4", 16, 2048, 2048))],
                         ids=["c1_small", "c1_full", "nvfp4_small"])
def test_linear(cfg):
    from fp4_block_scaled_moe_b200 import fp4_linear, fp4_pack
    w = D.expert_weights(cfg.seed, C.TID_LINEAR, (cfg.N, cfg.K), sigma=cfg.sigma)
    x_bits = D.activations_bf16(cfg.seed, cfg.T, cfg.K)
    c, s, t = fp4_pack(torch.from_numpy(w).cuda(), cfg.fmt)
    y = fp4_linear(_bf16_dev(x_bits), c, s, t, cfg.fmt)
    torch.cuda.synchronize()
    if cfg.fmt == "mxfp4":
        deq = F.mxfp4_dequantize(*F.mxfp4_quantize(w))
    else:
        deq = F.nvfp4_dequantize(*F.nvfp4_quantize(w))
    ref = M.linear(D.bf16_bits_to_f32(x_bits), deq)
    check_tolerance(_y_host(y), ref)


def _moe_case(cfg, tokens=None, variant=0, prepared=False):
    from fp4_block_scaled_moe_b200 import moe_fp4_forward, prepare_mma_scales
    x_bits, wr, bias = host_small_inputs(cfg)
    wdev = device_weights(cfg)
    wdev.kernel_variant = variant
    if prepared:
        prepare_mma_scales(wdev)
    x = _bf16_dev(x_bits)
    route = {n: torch.empty(s, dtype=d, device="cuda") for n, s, d in (
        ("logits", (cfg.T, cfg.E), torch.float32), ("topk_ids", (cfg.T, cfg.k), torch.int32))}
    y = moe_fp4_forward(wdev, x, torch.from_numpy(wr).cuda(), None if bias is None else torch.from_numpy(bias).cuda(),
                        cfg.k, route_out=route)
    torch.cuda.synchronize()
    bank = LazyOracleBank(cfg)
    xf = D.bf16_bits_to_f32(x_bits)
    lg = R.router_logits(xf, wr, bias)
    ids = R.topk(lg, cfg.k)
    w = R.softmax_selected(lg, ids)
    tok = np.arange(cfg.T) if tokens is None else np.asarray(tokens)
    ref = M.moe_forward(xf, ids, w, bank, cfg.swiglu_limit, tokens=tok)
    got = _y_host(y)[tok]
    ok = ~R.near_ties(lg, cfg.k)[tok]
    assert np.array_equal(route["topk_ids"].cpu().numpy()[tok][ok], ids[tok][ok])
    return check_tolerance(got, ref, mask_rows=ok)


@pytest.mark.parametrize("cfg", [C.small(C.MOE_C2), C.small(C.MOE_C3), C.small(C.MOE_C4), C.small(C.MOE_C5)],
                         ids=["c2_small", "c3_small", "c4_small_prefill_shape", "c5_small_cb4"])
def test_moe_small(cfg):
    _moe_case(cfg)


def test_moe_c5_cb4_full_sampled_tokens():
    """The CB4 decode layer at full size (64 experts, hidden 2048, intermediate 768,
    top-8, 16 tokens; codebooks per 128 weights plus the CSR outlier term)."""
    _moe_case(C.MOE_C5, tokens=[9])


def test_moe_c2_full_sampled_tokens():
    _moe_case(C.MOE_C2, tokens=[0, 5, 11, 15])


# Both expert-GEMM kernels on every MXFP4 shape: 1 = CUDA-core GEMV, 2 = block-scaled
# tensor cores with two-term MXFP8 activations.
@pytest.mark.parametrize("variant,prepared", [(1, False), (2, False), (2, True)],
                         ids=["gemv", "tensor", "tensor_prepared_scales"])
@pytest.mark.parametrize("cfg", [C.small(C.MOE_C2), C.small(C.MOE_C4)], ids=["c2_small", "c4_small_prefill_shape"])
def test_moe_variants(cfg, variant, prepared):
    _moe_case(cfg, variant=variant, prepared=prepared)


def test_moe_c2_full_tensor_variant_sampled_tokens():
    _moe_case(C.MOE_C2, tokens=[0, 7, 15], variant=2)


def test_moe_c4_full_prefill_sampled_tokens():
    """The full prefill layer (8192 tokens, 256 experts, hidden 6144, inter 2048, top-8)
    through the auto-selected tensor-core kernels; the oracle checks three tokens."""
    _moe_case(C.MOE_C4, tokens=[0, 8191], prepared=True)


# Degenerate routings: one token on one expert, every expert selected (k = E), and a
# single expert (E = 1, k = 1: the layer is a plain SwiGLU FFN), on both expert kernels
# and all three formats.
_EDGE = [
    ("mxfp4", 1, 8, 1, 1), ("mxfp4", 1, 8, 1, 2), ("mxfp4", 5, 4, 4, 1), ("mxfp4", 5, 4, 4, 2),
    ("mxfp4", 3, 1, 1, 2), ("nvfp4", 3, 1, 1, 1), ("nvfp4", 6, 4, 4, 1), ("cb4", 2, 1, 1, 1), ("cb4", 4, 4, 4, 1),
]


@pytest.mark.parametrize("fmt,T,E,k,variant", _EDGE, ids=[f"{f}_t{t}_e{e}_k{k}_v{v}" for f, t, e, k, v in _EDGE])
def test_moe_edge_routings(fmt, T, E, k, variant):
    from dataclasses import replace
    base = {"mxfp4": C.MOE_C2, "nvfp4": C.MOE_C3, "cb4": C.MOE_C5}[fmt]
    cfg = replace(base, name=f"edge_{fmt}_t{T}_e{E}_k{k}", T=T, E=E, H=512, I=256, k=k, zipf_bias=False)
    _moe_case(cfg, variant=variant)
