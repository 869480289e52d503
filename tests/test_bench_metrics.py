"""The benchmark's work accounting, pinned to closed forms of the layer shapes: the
active-bytes rule for decode (codes + scales of each routed expert, once) and
6 T k H I dense-equivalent flops for prefill."""
import numpy as np

import bench
from synth import configs as C


def test_per_expert_bytes_closed_forms():
    # MXFP4, H=2048, I=768: codes (2I*H + H*I)/2 + UE8M0 scales (2I*H + H*I)/32
    assert bench.per_expert_bytes(C.MOE_C2) == (2_506_752, 2 * 768 * 2048 // 2 + 2 * 768 * 2048 // 32)
    # NVFP4, H=6144, I=2048: codes/2 + E4M3 scales/16 + two fp32 tensor scales
    assert bench.per_expert_bytes(C.MOE_C3)[0] == 21_233_672
    # CB4 dense part: 4-bit indices + 16 fp16 entries per 128 weights (CSR counted separately)
    assert bench.per_expert_bytes(C.MOE_C5)[0] == 3_538_944


def test_algorithmic_bytes_counts_routed_experts_once():
    cfg = C.MOE_C2
    counts = np.zeros(cfg.E, dtype=np.int64)
    counts[[1, 5, 9]] = [3, 1, 12]
    router = cfg.E * cfg.H * 4
    xy = 2 * cfg.T * cfg.H * 2
    assert bench.algorithmic_bytes(cfg, counts) == 3 * 2_506_752 + router + xy
    extra = np.arange(cfg.E, dtype=np.int64) * 10
    assert bench.algorithmic_bytes(cfg, counts, extra=extra) == 3 * 2_506_752 + (1 + 5 + 9) * 10 + router + xy


def test_prefill_flops_and_units():
    assert bench.layer_flops(C.MOE_C4) == 6 * 8192 * 8 * 6144 * 2048
    work, unit = bench.work_per_step(C.MOE_C4, np.ones(C.MOE_C4.E))
    assert unit == "TFLOP/s" and abs(work - 4.948e12 / 1e12) < 1e-3
    work, unit = bench.work_per_step(C.MOE_C2, np.ones(C.MOE_C2.E))
    assert unit == "GB/s"


def test_mixed_gemv_roofline_counts_only_the_mxfp4_experts():
    """In a mixed buffer the GEMV reads the routed MXFP4 experts; the bf16 experts run in
    their own kernel, so the GEMV's roofline bytes leave them out (the layer's bytes keep
    them)."""
    cfg = C.MOE_C2_MIXED
    counts = np.zeros(cfg.E, dtype=np.int64)
    bf = list(cfg.bf16_experts)
    counts[[0, 1, 2] + bf[:2]] = 1                     # three MXFP4 experts and two bf16 ones
    r = bench.moe_roofline(cfg, counts, None, {"gate_up": 1.0, "down": 1.0}, False, {})
    gu = bench.per_expert_bytes(cfg)[1]
    P = cfg.T * cfg.k
    assert r["bytes_per_launch"] == 3 * gu + cfg.T * cfg.H * 2 + P * cfg.I * 2
    # the same routing in a pure MXFP4 buffer counts all five
    r2 = bench.moe_roofline(C.MOE_C2, counts, None, {"gate_up": 1.0, "down": 1.0}, False, {})
    assert r2["bytes_per_launch"] == 5 * gu + cfg.T * cfg.H * 2 + P * cfg.I * 2
