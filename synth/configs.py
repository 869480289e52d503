"""The workloads: a dense MXFP4 linear layer and four routed-expert MoE layers.

Dimensions, formats and input distributions follow the five benchmark
workloads of the FP4 block-scaled MoE study; ``small`` variants keep each
layer's structure (format, skew, outliers) at sizes a plain CPU reference
finishes in seconds while still spanning several kernel tiles and a ragged
tail of expert loads.
"""
from __future__ import annotations

from dataclasses import dataclass, replace

SEED = 0
SIGMA = 0.02

# tensor ids: the second Philox key word of each weight tensor
TID_LINEAR = 1
TID_GATE_UP = 2
TID_DOWN = 3


@dataclass(frozen=True)
class LinearConfig:
    name: str
    fmt: str          # "mxfp4" | "nvfp4"
    T: int
    N: int
    K: int
    seed: int = SEED
    sigma: float = SIGMA

    kind = "linear"


@dataclass(frozen=True)
class MoEConfig:
    name: str
    fmt: str          # "mxfp4" | "nvfp4" | "cb4"
    T: int
    E: int
    H: int
    I: int
    k: int
    zipf_bias: bool = False
    # planted outliers: (fraction, lo_sigma, hi_sigma) or None
    outliers: tuple | None = None
    # CB4 / V2a: absolute outlier threshold for the sparse term (in sigma)
    cb4_threshold_sigma: float = 6.0
    # V2a: bits per code (N)
    v2a_bits: int = 4
    # mixed-format buffers: experts kept in bf16 (the rest MXFP4)
    bf16_experts: tuple = ()
    swiglu_limit: float = 7.0
    seed: int = SEED
    sigma: float = SIGMA

    kind = "moe"


LINEAR_C1 = LinearConfig("linear_mxfp4_t16_n2048_k2048", "mxfp4", T=16, N=2048, K=2048)
MOE_C2 = MoEConfig("moe_mxfp4_decode_e64_h2048_i768_k8_t16", "mxfp4", T=16, E=64, H=2048, I=768, k=8)
MOE_C3 = MoEConfig("moe_nvfp4_decode_e256_h6144_i2048_k8_t64_zipf", "nvfp4", T=64, E=256, H=6144,
                   I=2048, k=8, zipf_bias=True, outliers=(0.003, 10.0, 49.0))
MOE_C4 = MoEConfig("moe_mxfp4_prefill_e256_h6144_i2048_k8_t8192", "mxfp4", T=8192, E=256, H=6144,
                   I=2048, k=8)
# ~0.106% of t4 draws exceed 6 sigma on their own; 0.394% more are planted in [6, 49] sigma
MOE_C5 = MoEConfig("moe_cb4_decode_e64_h2048_i768_k8_t16", "cb4", T=16, E=64, H=2048, I=768, k=8,
                   outliers=(0.00394, 6.0, 49.0))

# NVFP4 on the prefill shape: the prefill layer's dimensions, router and weight
# distribution with the NVFP4 format (E4M3 scale per 16 and a float32 scale per expert
# matrix) -- the format x phase pairing the benchmark configurations leave open.
MOE_C4_NV = MoEConfig("moe_nvfp4_prefill_e256_h6144_i2048_k8_t8192", "nvfp4", T=8192, E=256, H=6144,
                      I=2048, k=8)

# The V2a shared-library variant of the codebook layer: the CB4 layer's dimensions,
# weights and outliers, with 4-bit codes into one 32-codebook library per expert matrix.
MOE_C5_V2A = MoEConfig("moe_v2a4_decode_e64_h2048_i768_k8_t16", "v2a", T=16, E=64, H=2048, I=768, k=8,
                       outliers=(0.00394, 6.0, 49.0))

# A mixed-format fused buffer: the MXFP4 decode layer with five experts excluded from
# quantisation and kept in bf16 (full-width rows) inside the same fused tensor.
MOE_C2_MIXED = MoEConfig("moe_mixed_mxfp4_bf16_decode_e64_h2048_i768_k8_t16", "mixed", T=16, E=64, H=2048, I=768,
                         k=8, bf16_experts=(3, 6, 11, 42, 60))

FULL = {c.name: c for c in (LINEAR_C1, MOE_C2, MOE_C3, MOE_C4, MOE_C5, MOE_C4_NV, MOE_C5_V2A, MOE_C2_MIXED)}
# The prefill layer at a quarter of the experts and tokens (same per-expert load, same
# tile shapes; 1.3 GB of weights): the size used for full hardware-counter captures.
MOE_C4_PROFILE = MoEConfig("moe_mxfp4_prefill_e64_h6144_i2048_k8_t2048", "mxfp4", T=2048, E=64, H=6144,
                           I=2048, k=8)
# The NVFP4 decode layer and the NVFP4 prefill layer at a quarter of the experts (and of
# the tokens for prefill): 1.36 GB of weights, the sizes used for hardware-counter captures.
MOE_C3_PROFILE = MoEConfig("moe_nvfp4_decode_e64_h6144_i2048_k8_t16_zipf", "nvfp4", T=16, E=64, H=6144, I=2048,
                           k=8, zipf_bias=True, outliers=(0.003, 10.0, 49.0))
MOE_C4NV_PROFILE = MoEConfig("moe_nvfp4_prefill_e64_h6144_i2048_k8_t2048", "nvfp4", T=2048, E=64, H=6144,
                             I=2048, k=8)
# The NVFP4 decode layer at a quarter of the experts with all 64 tokens (units of up to
# 16 tokens, as in the full layer): 1.36 GB of weights.
MOE_C3_PROFILE_T64 = MoEConfig("moe_nvfp4_decode_e64_h6144_i2048_k8_t64_zipf", "nvfp4", T=64, E=64, H=6144,
                               I=2048, k=8, zipf_bias=True, outliers=(0.003, 10.0, 49.0))
PROFILE = {c.name: c for c in (MOE_C4_PROFILE, MOE_C3_PROFILE, MOE_C4NV_PROFILE, MOE_C3_PROFILE_T64)}


def small(cfg):
    """A reduced copy of ``cfg`` with the same structure, for exhaustive CPU comparison."""
    if cfg.kind == "linear":
        return replace(cfg, name=cfg.name + "_small", T=5, N=320, K=768)
    if cfg.fmt in ("cb4", "v2a"):
        return replace(cfg, name=cfg.name + "_small", T=7, E=8, H=512, I=256, k=3)
    if cfg.fmt == "mixed":
        return replace(cfg, name=cfg.name + "_small", T=9, E=16, H=768, I=512, k=4,
                       bf16_experts=tuple(e for e in cfg.bf16_experts if e < 16))
    if cfg.T > 1000:  # prefill-shaped: many tokens per expert
        return replace(cfg, name=cfg.name + "_small", T=300, E=8, H=512, I=256, k=2)
    return replace(cfg, name=cfg.name + "_small", T=9, E=16, H=768, I=512, k=4)


def expert_rows(cfg, which, e):
    """float32 weights of expert e drawn on the host: which = 'gu' -> [2I, H] (gate rows
    then up rows), 'dn' -> [H, I].  The same draws the device generator makes for the
    fused [E, rows, K] tensors."""
    from . import draws
    if which == "gu":
        return draws.expert_weights(cfg.seed, TID_GATE_UP, (cfg.E, 2 * cfg.I, cfg.H), start_row=e * 2 * cfg.I,
                                    rows=2 * cfg.I, sigma=cfg.sigma, outliers=cfg.outliers)
    return draws.expert_weights(cfg.seed, TID_DOWN, (cfg.E, cfg.H, cfg.I), start_row=e * cfg.H, rows=cfg.H,
                                sigma=cfg.sigma, outliers=cfg.outliers)
