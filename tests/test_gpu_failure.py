"""Failure detection on the GPU without a fault: a bounded device wait is made to run
out (a barrier phase nothing completes), the status word reports FP4_ERR_TIMEOUT, and
the context and the workspace stay usable for a correct layer call afterwards."""
import numpy as np
import pytest
import torch

from synth import configs as C, draws as D

from helpers import LazyOracleBank, check_tolerance, device_weights, host_small_inputs

pytestmark = pytest.mark.gpu


def test_bounded_wait_timeout_reports_and_recovers():
    from fp4_block_scaled_moe_b200 import api
    from oracle import moe as M, routing as R
    cfg = C.small(C.MOE_C2)
    w = device_weights(cfg)
    ws = api.alloc_workspace(api.moe_fp4_workspace_size(w, cfg.T, cfg.k), torch.device("cuda"))
    assert api.fp4_workspace_status(ws) in ("FP4_OK", "FP4_ERR_TIMEOUT")      # clears any old word
    api.fp4_selftest_wait_timeout(ws, 2_000_000)                              # 2 ms
    assert api.fp4_workspace_status(ws) == "FP4_ERR_TIMEOUT"
    assert api.fp4_workspace_status(ws) == "FP4_OK"                           # read clears it
    x_bits, wr, bias = host_small_inputs(cfg)
    x = torch.from_numpy(x_bits.view(np.int16)).cuda().view(torch.bfloat16)
    y = api.moe_fp4_forward(w, x, torch.from_numpy(wr).cuda(), None, cfg.k, workspace=ws)
    assert api.fp4_workspace_status(ws) == "FP4_OK"
    xf = D.bf16_bits_to_f32(x_bits)
    lg = R.router_logits(xf, wr, bias)
    ids = R.topk(lg, cfg.k)
    ref = M.moe_forward(xf, ids, R.softmax_selected(lg, ids), LazyOracleBank(cfg), cfg.swiglu_limit)
    got = D.bf16_bits_to_f32(y.view(torch.int16).cpu().numpy().view(np.uint16)).reshape(cfg.T, cfg.H)
    check_tolerance(got, ref, mask_rows=~R.near_ties(lg, cfg.k))
