"""Expert parallelism for the routed-expert MoE layer.

The experts of a layer are split over the ranks of a process group, each rank holding a
contiguous range of them (the TP4/EP4 placement the "GLM-5.3-Flash-MXFP4" card serves
with). Every rank sees the same tokens (in a tensor/expert-parallel deployment x is
already replicated after the attention block's all-reduce), routes them over all E
experts, runs only the (token, expert) pairs whose expert it holds, and contributes an
fp32 partial sum of the layer output; one all-reduce of the partial sums (NCCL over
NVLink / NVSwitch on GPUs) and one rounding to bf16 finish the layer.

The computation is the library's (moe_fp4_forward_partial, fp4_f32_to_bf16); this module
only slices the weights and runs the exchange.
"""
from __future__ import annotations

import dataclasses

import torch

from .api import MoEWeights, fp4_f32_to_bf16, moe_fp4_forward_partial


def expert_range(rank: int, world: int, E: int):
    """(first expert, count) of ``rank``: E split into ``world`` contiguous ranges, the
    first E % world ranks holding one expert more."""
    if not (0 <= rank < world) or E < world:
        raise ValueError("need 0 <= rank < world <= E")
    base, extra = divmod(E, world)
    begin = rank * base + min(rank, extra)
    return begin, base + (1 if rank < extra else 0)


def shard(weights: MoEWeights, rank: int, world: int) -> MoEWeights:
    """The experts of ``rank`` cut from a full layer's weights (copies, contiguous). The
    CB4 / V2a outlier CSR, one per fused matrix over E * rows rows, is cut to the local rows
    and its row pointers re-based; CB4 codebooks are cut by rows, V2a libraries (one per
    expert matrix) by expert.  Mixed-format buffers are refused (their byte offsets would
    need re-basing, which is not implemented)."""
    if weights.local_experts not in (0, weights.E) or weights.expert_begin != 0:
        raise ValueError("shard() takes a full layer")
    if weights.expert_format is not None:
        raise ValueError("shard() does not cut mixed-format buffers")
    b, n = expert_range(rank, world, weights.E)
    cut = {}
    per_expert = ("gu_codes", "gu_scales", "dn_codes", "dn_scales", "gu_tscale", "dn_tscale")
    for name in per_expert:
        t = getattr(weights, name)
        cut[name] = None if t is None else t[b:b + n].contiguous()
    if weights.fmt in ("cb4", "v2a"):
        for pre, rows in (("gu", 2 * weights.I), ("dn", weights.H)):
            cb = getattr(weights, pre + "_cb")
            if weights.fmt == "cb4":
                cut[pre + "_cb"] = cb.view(weights.E, rows, *cb.shape[1:])[b:b + n].reshape(n * rows, *cb.shape[1:]).contiguous()
            else:
                cut[pre + "_cb"] = cb[b:b + n].contiguous()
            rp = getattr(weights, pre + "_rowptr")
            r0, r1 = b * rows, (b + n) * rows
            lo = rp[r0:r0 + 1]
            hi = rp[r1:r1 + 1]
            cut[pre + "_rowptr"] = (rp[r0:r1 + 1] - lo).contiguous()
            start, stop = int(lo.item()), int(hi.item())
            col, val = getattr(weights, pre + "_col"), getattr(weights, pre + "_val")
            cut[pre + "_col"] = col[start:stop].contiguous() if stop > start else col[:1].clone()
            cut[pre + "_val"] = val[start:stop].contiguous() if stop > start else val[:1].clone()
    # re-laid scale atoms are per tile, and tiles do not cross experts: cut them the same way
    for name, rows_per in (("gu_mma_scales", 2 * weights.I * weights.H), ("dn_mma_scales", weights.H * weights.I)):
        t = getattr(weights, name)
        if t is not None:
            per = t.numel() // weights.E
            cut[name] = t[b * per:(b + n) * per].contiguous()
    return dataclasses.replace(weights, **cut, expert_begin=b, local_experts=n)


def exchange(y_partial: torch.Tensor, group=None) -> torch.Tensor:
    """Sum the ranks' fp32 partial outputs in place (all-reduce over ``group``)."""
    import torch.distributed as dist
    if dist.is_available() and dist.is_initialized() and dist.get_world_size(group) > 1:
        dist.all_reduce(y_partial, op=dist.ReduceOp.SUM, group=group)
    return y_partial


class ExpertParallelMoE:
    """One rank of an expert-parallel MoE layer: ``local`` holds this rank's experts
    (see shard), ``group`` the ranks that share the layer."""

    def __init__(self, local: MoEWeights, group=None):
        self.local = local
        self.group = group

    def forward(self, x, router_w, router_bias, k, workspace=None, y_partial=None):
        y_part = moe_fp4_forward_partial(self.local, x, router_w, router_bias, k, workspace=workspace,
                                         y_partial=y_partial)
        exchange(y_part, self.group)
        return fp4_f32_to_bf16(y_part)
