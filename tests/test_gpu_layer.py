"""Layer outputs on the GPU against the float64 oracle, within the fixed gates:
relative Frobenius error <= 5e-3 and |err| <= 2e-2 (|ref| + 1) per element.

Every case compares every sampled token with no token left out: where the fp64 logits
of a token leave its k-th and (k+1)-th expert within the tie band, the GPU's own
selection is checked for validity and fed to the oracle.  Full-size layers run the
oracle expert by expert in a spawn process pool (tests/oracle_pool.py)."""
import numpy as np
import pytest
import torch

from oracle import formats as F, moe as M, routing as R
from synth import configs as C, draws as D

from helpers import check_tolerance, device_weights, host_small_inputs, parity_log
from oracle_pool import moe_reference

pytestmark = pytest.mark.gpu

CLAMP_X_SCALE = 16.0   # activations N(0, 16^2): the SwiGLU clamp fires on a large share of pairs
MIN_CLAMP_SHARE = 0.10


def _bf16_dev(bits):
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).cuda().view(torch.bfloat16)


def _y_host(y):
    return D.bf16_bits_to_f32(y.view(torch.int16).cpu().numpy().view(np.uint16)).reshape(y.shape)


# up to 64 tokens the dense layer is one kernel that converts x itself; above, x is
# converted by a separate launch first (the many-token cases)
@pytest.mark.parametrize("cfg", [C.small(C.LINEAR_C1), C.LINEAR_C1,
                                 C.small(C.LinearConfig("linear_nvfp4", "nvfp4", 16, 2048, 2048)),
                                 C.LinearConfig("linear_mxfp4_many_tokens", "mxfp4", 1100, 128, 512),
                                 C.LinearConfig("linear_nvfp4_many_tokens", "nvfp4", 1030, 192, 768)],
                         ids=["c1_small", "c1_full", "nvfp4_small", "mxfp4_many_tokens", "nvfp4_many_tokens"])
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


@pytest.mark.parametrize("fmt", ["mxfp4", "nvfp4"])
def test_linear_fused_conversion_bits(fmt):
    """The one-launch dense layer (64 tokens) converts x to f16 inside the GEMV; the
    two-launch one (65 tokens) converts it in a separate kernel first.  A token's output
    does not depend on the other tokens, so the first 64 rows of both calls agree bit for
    bit -- over rows whose power-of-two scale spans the whole bf16 range: a zero row, rows
    of subnormal size (scale factor above 2^127), rows near the bf16 maximum."""
    from fp4_block_scaled_moe_b200 import fp4_linear, fp4_pack
    K, N = 1024, 192
    w = D.expert_weights(11, C.TID_LINEAR, (N, K), sigma=0.02)
    x = D.bf16_bits_to_f32(D.activations_bf16(11, 65, K)).astype(np.float32)
    exps = np.arange(65) % 41 - 20
    exps[3], exps[5], exps[9], exps[17] = -128, -131, 100, 110
    x = np.ldexp(x, exps[:, None]).astype(np.float32)
    x[7] = 0.0
    x_bits = D.f32_to_bf16_bits(x)
    c, s, t = fp4_pack(torch.from_numpy(w).cuda(), fmt)
    xd = _bf16_dev(x_bits)
    y65 = fp4_linear(xd, c, s, t, fmt)
    y64 = fp4_linear(xd[:64].contiguous(), c, s, t, fmt)
    torch.cuda.synchronize()
    assert torch.equal(y64.view(torch.int16), y65[:64].view(torch.int16))
    if fmt == "mxfp4":
        deq = F.mxfp4_dequantize(*F.mxfp4_quantize(w))
    else:
        deq = F.nvfp4_dequantize(*F.nvfp4_quantize(w))
    ref = M.linear(D.bf16_bits_to_f32(x_bits), deq)
    got = _y_host(y65)
    for r in range(65):          # each row against its own magnitude (normal bf16 outputs)
        scale = float(np.max(np.abs(ref[r])))
        if scale > 2.0 ** -100:
            check_tolerance(got[r] / scale, ref[r] / scale)
        else:
            assert np.all(np.abs(got[r]) <= 2.0 ** -100)


def check_selection(lg, gids, k):
    """Routing of the GPU against the fp64 logits: identical ids (order included) for
    every token outside the tie band; inside it, a valid top-k (k distinct experts, no
    unselected logit above a selected one by more than the band, descending within the
    band).  Returns the number of tokens whose selection differs from the fp64 one."""
    ref = R.topk(lg, k)
    ties = R.near_ties(lg, k)
    differ = np.any(ref != gids, axis=1)
    assert not np.any(differ & ~ties), f"tokens {np.nonzero(differ & ~ties)[0][:8]} routed differently"
    for t in np.nonzero(differ)[0]:
        sel = gids[t]
        assert len(set(sel.tolist())) == k
        band = 1e-4 * max(1.0, float(np.max(np.abs(lg[t]))))
        unsel = np.setdiff1d(np.arange(lg.shape[1]), sel)
        assert lg[t, sel].min() >= lg[t, unsel].max() - band
        assert np.all(np.diff(lg[t, sel]) <= band)
    return int(differ.sum())


def _moe_case(cfg, tokens=None, variant=0, prepared=False, x_scale=1.0, parallel=None, min_clamp=None):
    from fp4_block_scaled_moe_b200 import moe_fp4_forward, prepare_mma_scales
    x_bits, wr, bias = host_small_inputs(cfg, x_scale)
    wdev = device_weights(cfg)
    wdev.kernel_variant = variant
    if prepared:
        prepare_mma_scales(wdev)
    x = _bf16_dev(x_bits)
    route = {"topk_ids": torch.empty((cfg.T, cfg.k), dtype=torch.int32, device="cuda")}
    y = moe_fp4_forward(wdev, x, torch.from_numpy(wr).cuda(), None if bias is None else torch.from_numpy(bias).cuda(),
                        cfg.k, route_out=route)
    torch.cuda.synchronize()
    gids = route["topk_ids"].cpu().numpy()
    del wdev
    xf = D.bf16_bits_to_f32(x_bits)
    lg = R.router_logits(xf, wr, bias)
    n_alt = check_selection(lg, gids, cfg.k)
    w = R.softmax_selected(lg, gids)
    tok = np.arange(cfg.T) if tokens is None else np.asarray(tokens)
    if parallel is None:
        parallel = cfg.H * cfg.I >= 2048 * 768
    ref, st = moe_reference(cfg, xf, gids, w, tok, parallel=parallel)
    share_g, share_u = st["g_clamped"] / st["pairs"], st["u_clamped"] / st["pairs"]
    parity_log(f"tokens={tok.size}\tselection_differs={n_alt}\tclamped_g={st['g_clamped']}\t"
               f"clamped_u={st['u_clamped']}\tpairs={st['pairs']}")
    if min_clamp is not None:
        assert share_g >= min_clamp and share_u >= min_clamp, (share_g, share_u)
    return check_tolerance(_y_host(y)[tok], ref)


@pytest.mark.parametrize("cfg", [C.small(C.MOE_C2), C.small(C.MOE_C3), C.small(C.MOE_C4), C.small(C.MOE_C5),
                                 C.small(C.MOE_C5_V2A)],
                         ids=["c2_small", "c3_small", "c4_small_prefill_shape", "c5_small_cb4", "v2a_small"])
def test_moe_small(cfg):
    _moe_case(cfg)


# NVFP4 GEMV units of up to 16 tokens (T >= 32 and T k >= 2E): the Zipf-skewed router puts
# 17-48 tokens on four experts (two or three 16-token units each), 9-16 on one and 1-8 on
# five, so full, partial and single-tile units all run
@pytest.mark.parametrize("variant", [0, 1], ids=["auto", "gemv"])
def test_moe_nvfp4_sixteen_token_units(variant):
    from dataclasses import replace
    cfg = replace(C.MOE_C3, name="nvfp4_t48_e64_k4_zipf", T=48, E=64, H=512, I=256, k=4)
    _moe_case(cfg, variant=variant)


@pytest.mark.parametrize("cfg", [C.small(C.MOE_C2_MIXED), C.MOE_C2_MIXED], ids=["small", "full"])
def test_moe_mixed_format_buffer(cfg):
    """A fused buffer holding MXFP4 experts and bf16 experts (kept out of quantisation),
    each at its own offset: every token, and both kinds of expert are routed."""
    routed = set(np.unique(R.topk(R.router_logits(D.bf16_bits_to_f32(host_small_inputs(cfg)[0]),
                                                  host_small_inputs(cfg)[1]), cfg.k)).tolist())
    assert routed & set(cfg.bf16_experts) and routed - set(cfg.bf16_experts)
    _moe_case(cfg)


def test_moe_v2a_full_sampled_tokens():
    """The V2a layer at full size (the CB4 layer's dimensions and outliers, 4-bit codes
    into one shared 32-codebook library per expert matrix), on six tokens spread over the
    batch (the oracle fits each expert in about a minute)."""
    _moe_case(C.MOE_C5_V2A, tokens=[0, 3, 6, 9, 12, 15])


def test_moe_c2_full_all_tokens():
    """The MXFP4 decode layer at full size (64 experts, hidden 2048, intermediate 768,
    top-8, 16 tokens), every token, on the kernels the library picks for unprepared
    weights."""
    _moe_case(C.MOE_C2)


def test_moe_c2_full_tensor_all_tokens():
    _moe_case(C.MOE_C2, prepared=True, variant=2)


def test_moe_c3_full_all_tokens():
    """The NVFP4 decode layer at full size (256 experts, hidden 6144, intermediate 2048,
    top-8, 64 tokens, Zipf(1.1) router bias, 0.3% outliers at 10-49 sigma), every token:
    hot experts run several units of tokens each."""
    _moe_case(C.MOE_C3)


def test_moe_c3_full_tensor_all_tokens():
    """The NVFP4 decode layer at full size on the tensor-core kernels (weights widened to
    f16 on chip, prepared scale atoms), every token."""
    _moe_case(C.MOE_C3, variant=2, prepared=True)


def test_moe_c5_cb4_full_all_tokens():
    """The CB4 decode layer at full size (codebooks per 128 weights plus the CSR outlier
    term), every token."""
    _moe_case(C.MOE_C5)


UNIT_MX = 112   # slots per work unit of the MXFP4 tensor-core kernels at prefill sizes
UNIT_NV = 256   # and of the NVFP4 ones


def c4_sample_tokens(n=64, unit=UNIT_MX):
    """Tokens of the prefill layer whose (expert, slot) pairs, taken modulo the work-unit
    width, cover every position of a unit; the first, a middle and the last token and
    some near-tie tokens included; the rest chosen to reuse experts already sampled
    (bounds the oracle's work)."""
    cfg = C.MOE_C4
    x_bits, wr, bias = host_small_inputs(cfg)
    lg = R.router_logits(D.bf16_bits_to_f32(x_bits), wr, bias)
    ids = R.topk(lg, cfg.k)
    _, off, _, inv = R.permutation(ids, cfg.E)
    pos = (inv.reshape(cfg.T, cfg.k) - off[ids]) % unit
    chosen = [0, 4099, 8191] + [int(t) for t in np.nonzero(R.near_ties(lg, cfg.k))[0][:4]]
    cover = set(pos[chosen].ravel().tolist())
    while len(cover) < unit:
        t = max(range(cfg.T), key=lambda t: len(set(pos[t].tolist()) - cover))
        chosen.append(t)
        cover |= set(pos[t].tolist())
    experts = set(ids[chosen].ravel().tolist())
    while len(chosen) < n:
        score = np.array([len(set(ids[t].tolist()) - experts) for t in range(cfg.T)])
        score[chosen] = 1 << 30
        t = int(np.argmin(score))
        chosen.append(t)
        experts |= set(ids[t].tolist())
    return sorted(set(chosen))


def test_moe_c4_nvfp4_full_prefill_sampled_tokens():
    """NVFP4 on the prefill layer (8192 tokens, 256 experts, hidden 6144, inter 2048,
    top-8) through the auto-selected tensor-core kernels, on the same token sample."""
    _moe_case(C.MOE_C4_NV, tokens=c4_sample_tokens(unit=UNIT_NV), prepared=True)


def test_moe_c4_full_prefill_sampled_tokens():
    """The full prefill layer (8192 tokens, 256 experts, hidden 6144, inter 2048, top-8)
    through the auto-selected tensor-core kernels, on 64 tokens that cover every slot
    position of a work unit, include near-tie tokens, the first, a middle and the last."""
    _moe_case(C.MOE_C4, tokens=c4_sample_tokens(), prepared=True)


# The clamp h = silu(min(g, 7)) clamp(u, -7, 7) must act: activations scaled by 16 put
# at least 10% of the gate values above 7 and 10% of the up values outside [-7, 7].
_CLAMP = [("mxfp4", 1), ("mxfp4", 2), ("nvfp4", 1), ("nvfp4", 2), ("cb4", 1), ("v2a", 1)]


@pytest.mark.parametrize("fmt,variant", _CLAMP, ids=[f"{f}_v{v}" for f, v in _CLAMP])
def test_moe_clamp_active_small(fmt, variant):
    base = {"mxfp4": C.MOE_C2, "nvfp4": C.MOE_C3, "cb4": C.MOE_C5, "v2a": C.MOE_C5_V2A}[fmt]
    _moe_case(C.small(base), variant=variant, x_scale=CLAMP_X_SCALE, min_clamp=MIN_CLAMP_SHARE)


@pytest.mark.parametrize("base", [C.MOE_C4, C.MOE_C4_NV], ids=["mxfp4", "nvfp4"])
def test_moe_clamp_active_prefill_shape(base):
    _moe_case(C.small(base), variant=2, x_scale=CLAMP_X_SCALE, min_clamp=MIN_CLAMP_SHARE)


@pytest.mark.parametrize("variant", [1, 2], ids=["gemv", "tensor"])
def test_moe_clamp_active_c2_full(variant):
    _moe_case(C.MOE_C2, variant=variant, prepared=variant == 2, x_scale=CLAMP_X_SCALE, min_clamp=MIN_CLAMP_SHARE)


# Both expert-GEMM kernels on every MXFP4 and NVFP4 shape: 1 = CUDA-core GEMV, 2 = tensor
# cores (MXFP4: block-scaled with two-term MXFP8 activations; NVFP4: weights widened to
# f16 on chip, kind::f16), with and without the prepared scale atoms.
@pytest.mark.parametrize("variant,prepared", [(1, False), (2, False), (2, True)],
                         ids=["gemv", "tensor", "tensor_prepared_scales"])
@pytest.mark.parametrize("cfg", [C.small(C.MOE_C2), C.small(C.MOE_C4), C.small(C.MOE_C3), C.small(C.MOE_C4_NV)],
                         ids=["c2_small", "c4_small_prefill_shape", "c3_small_nvfp4", "c4nv_small_prefill_shape"])
def test_moe_variants(cfg, variant, prepared):
    _moe_case(cfg, variant=variant, prepared=prepared)


# Degenerate routings: one token on one expert, every expert selected (k = E), and a
# single expert (E = 1, k = 1: the layer is a plain SwiGLU FFN), on both expert kernels
# and all three formats.
_EDGE = [
    ("mxfp4", 1, 8, 1, 1), ("mxfp4", 1, 8, 1, 2), ("mxfp4", 5, 4, 4, 1), ("mxfp4", 5, 4, 4, 2),
    ("mxfp4", 3, 1, 1, 2), ("nvfp4", 3, 1, 1, 1), ("nvfp4", 6, 4, 4, 1), ("nvfp4", 1, 8, 1, 2),
    ("nvfp4", 6, 4, 4, 2), ("nvfp4", 3, 1, 1, 2), ("cb4", 2, 1, 1, 1), ("cb4", 4, 4, 4, 1),
    ("v2a", 2, 1, 1, 1), ("v2a", 4, 4, 4, 1),
]


@pytest.mark.parametrize("fmt,T,E,k,variant", _EDGE, ids=[f"{f}_t{t}_e{e}_k{k}_v{v}" for f, t, e, k, v in _EDGE])
def test_moe_edge_routings(fmt, T, E, k, variant):
    from dataclasses import replace
    base = {"mxfp4": C.MOE_C2, "nvfp4": C.MOE_C3, "cb4": C.MOE_C5, "v2a": C.MOE_C5_V2A}[fmt]
    cfg = replace(base, name=f"edge_{fmt}_t{T}_e{E}_k{k}", T=T, E=E, H=512, I=256, k=k, zipf_bias=False)
    _moe_case(cfg, variant=variant)
