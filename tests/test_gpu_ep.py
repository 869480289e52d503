"""Expert parallelism through the C ABI on one GPU: the layer's experts are cut into
ranges (ep.shard), each range runs moe_fp4_forward_partial in turn (no kernel waits on
another), the fp32 partial sums are added in rank order -- what the all-reduce over the
ranks computes -- and fp4_f32_to_bf16 rounds the result.  It must pass the fixed gates
against the float64 oracle, agree with the single-call layer, and each partial must hold
only its own experts' pairs."""
import numpy as np
import pytest
import torch

from oracle import routing as R
from synth import configs as C, draws as D

from helpers import check_tolerance, device_weights, host_small_inputs, tolerance_stats
from oracle_pool import moe_reference

pytestmark = pytest.mark.gpu

_CASES = [("mxfp4", 1, 2, False), ("mxfp4", 2, 3, True), ("mxfp4", 2, 2, False), ("nvfp4", 1, 2, False),
          ("nvfp4", 2, 3, True), ("nvfp4", 2, 2, False), ("cb4", 1, 2, False)]


@pytest.mark.parametrize("fmt,variant,world,prepared", _CASES,
                         ids=[f"{f}_v{v}_w{w}{'_prepared' if p else ''}" for f, v, w, p in _CASES])
def test_expert_parallel_ranks_reassemble_the_layer(fmt, variant, world, prepared):
    from fp4_block_scaled_moe_b200 import ep, fp4_f32_to_bf16, moe_fp4_forward, moe_fp4_forward_partial
    from fp4_block_scaled_moe_b200 import prepare_mma_scales
    cfg = C.small({"mxfp4": C.MOE_C2, "nvfp4": C.MOE_C3, "cb4": C.MOE_C5}[fmt])
    x_bits, wr, bias = host_small_inputs(cfg)
    full = device_weights(cfg)
    full.kernel_variant = variant
    if prepared:
        prepare_mma_scales(full)
    x = torch.from_numpy(x_bits.view(np.int16)).cuda().view(torch.bfloat16)
    wr_t = torch.from_numpy(wr).cuda()
    bias_t = None if bias is None else torch.from_numpy(bias).cuda()
    ids_t = torch.empty((cfg.T, cfg.k), dtype=torch.int32, device="cuda")
    y_one = moe_fp4_forward(full, x, wr_t, bias_t, cfg.k, route_out={"topk_ids": ids_t})
    total = torch.zeros((cfg.T, cfg.H), dtype=torch.float32, device="cuda")
    for r in range(world):
        part = moe_fp4_forward_partial(ep.shard(full, r, world), x, wr_t, bias_t, cfg.k)
        torch.cuda.synchronize()
        b, n = ep.expert_range(r, world, cfg.E)
        ids = ids_t.cpu().numpy()
        none_local = ~np.any((ids >= b) & (ids < b + n), axis=1)
        assert bool((part[torch.from_numpy(none_local).cuda()] == 0).all()), "a partial holds foreign pairs"
        total += part
    y = fp4_f32_to_bf16(total)
    torch.cuda.synchronize()
    to_host = lambda t: D.bf16_bits_to_f32(t.view(torch.int16).cpu().numpy().view(np.uint16)).reshape(t.shape)
    xf = D.bf16_bits_to_f32(x_bits)
    lg = R.router_logits(xf, wr, bias)
    gids = ids_t.cpu().numpy()
    ref, _ = moe_reference(cfg, xf, gids, R.softmax_selected(lg, gids), parallel=False)
    check_tolerance(to_host(y), ref)
    rel, _, _ = tolerance_stats(to_host(y), to_host(y_one))
    assert rel < 2e-3                         # the same pairs summed in another order, then rounded


def test_f32_to_bf16_rounds_to_nearest_even():
    from fp4_block_scaled_moe_b200 import fp4_f32_to_bf16
    v = np.array([1.0, 1.0 + 2.0 ** -8, 1.0 + 3 * 2.0 ** -8, -2.5, 3.0e38, 1e-40, 0.0, -0.0], np.float32)
    got = fp4_f32_to_bf16(torch.from_numpy(v).cuda()).view(torch.int16).cpu().numpy().view(np.uint16)
    assert np.array_equal(got, D.f32_to_bf16_bits(v))
