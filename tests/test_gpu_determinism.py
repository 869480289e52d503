"""The layer is deterministic: the same call twice, a call on another workspace, and
every replay of a captured CUDA graph give identical y bits.  Work units are handed to
CTAs from an atomic counter, so which CTA runs a unit varies from call to call; each
unit owns its output rows and sums its K in a fixed order, and the combine adds the k
slots of a token in j order, so the bits do not depend on that schedule."""
from dataclasses import replace

import numpy as np
import pytest
import torch

from synth import configs as C

from helpers import device_weights, host_small_inputs

pytestmark = pytest.mark.gpu

_CASES = [
    ("c2_full_gemv", C.MOE_C2, 1, False),
    ("c2_full_tensor", C.MOE_C2, 2, True),
    ("c3_small_nvfp4", C.small(C.MOE_C3), 0, False),
    ("c5_small_cb4", C.small(C.MOE_C5), 0, False),
    ("c4_small_tensor", C.small(C.MOE_C4), 2, False),
    ("c4_full_tensor", C.MOE_C4, 0, True),
    ("c3_small_nvfp4_tensor", C.small(C.MOE_C3), 2, False),
    ("c3_full_nvfp4_tensor", C.MOE_C3, 2, True),
    ("c4nv_full_tensor", C.MOE_C4_NV, 0, True),
    ("nvfp4_t48_gemv_16_token_units", replace(C.MOE_C3, name="nvfp4_t48_e64_k4_zipf", T=48, E=64, H=512, I=256, k=4),
     1, False),
]


@pytest.mark.parametrize("name,cfg,variant,prepared", _CASES, ids=[c[0] for c in _CASES])
def test_repeat_and_graph_replay_bit_identical(name, cfg, variant, prepared):
    from fp4_block_scaled_moe_b200 import api, prepare_mma_scales
    x_bits, wr, bias = host_small_inputs(cfg)
    w = device_weights(cfg)
    w.kernel_variant = variant
    if prepared:
        prepare_mma_scales(w)
    x = torch.from_numpy(x_bits.view(np.int16)).cuda().view(torch.bfloat16)
    wr_t = torch.from_numpy(wr).cuda()
    bias_t = None if bias is None else torch.from_numpy(bias).cuda()
    nbytes = api.moe_fp4_workspace_size(w, cfg.T, cfg.k)
    ws1 = api.alloc_workspace(nbytes, x.device)
    ws2 = api.alloc_workspace(nbytes + 4096, x.device)
    y1 = api.moe_fp4_forward(w, x, wr_t, bias_t, cfg.k, workspace=ws1)
    y2 = api.moe_fp4_forward(w, x, wr_t, bias_t, cfg.k, workspace=ws1)
    y3 = api.moe_fp4_forward(w, x, wr_t, bias_t, cfg.k, workspace=ws2)
    torch.cuda.synchronize()
    b1 = y1.view(torch.int16)
    assert torch.equal(b1, y2.view(torch.int16)), "second call differs"
    assert torch.equal(b1, y3.view(torch.int16)), "call on another workspace differs"
    assert bool(torch.isfinite(y1.float()).all())

    yg = torch.empty_like(y1)
    s = torch.cuda.Stream()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.stream(s):
        api.moe_fp4_forward(w, x, wr_t, bias_t, cfg.k, workspace=ws1, y=yg)
        torch.cuda.synchronize()
        with torch.cuda.graph(g, stream=s):
            api.moe_fp4_forward(w, x, wr_t, bias_t, cfg.k, workspace=ws1, y=yg)
    for _ in range(3):
        yg.fill_(float("nan"))
        with torch.cuda.stream(s):
            g.replay()
        torch.cuda.synchronize()
        assert torch.equal(b1, yg.view(torch.int16)), "graph replay differs"
    assert api.fp4_workspace_status(ws1) == "FP4_OK"
    del g


_LINEAR = [
    ("c1_full_split", C.LINEAR_C1),                                               # one launch + K shares
    ("nvfp4_t48_split2", C.LinearConfig("linear_nvfp4_t48", "nvfp4", 48, 1024, 2048)),
    ("mxfp4_t200", C.LinearConfig("linear_mxfp4_t200", "mxfp4", 200, 512, 1024)),   # separate x conversion
]


@pytest.mark.parametrize("name,cfg", _LINEAR, ids=[c[0] for c in _LINEAR])
def test_linear_repeat_and_graph_replay_bit_identical(name, cfg):
    """The dense layer likewise: its K shares are added in a fixed order by the reduce."""
    from fp4_block_scaled_moe_b200 import api, fp4_linear, fp4_pack
    from synth import draws as D
    w = D.expert_weights(cfg.seed, C.TID_LINEAR, (cfg.N, cfg.K), sigma=cfg.sigma)
    x_bits = D.activations_bf16(cfg.seed, cfg.T, cfg.K)
    c, s_, t = fp4_pack(torch.from_numpy(w).cuda(), cfg.fmt)
    x = torch.from_numpy(x_bits.view(np.int16)).cuda().view(torch.bfloat16)
    nbytes = int(api.L.load().fp4_linear_workspace_size(cfg.T, cfg.K))
    ws1 = api.alloc_workspace(nbytes, x.device)
    ws2 = api.alloc_workspace(nbytes + 4096, x.device)
    y1 = fp4_linear(x, c, s_, t, cfg.fmt, workspace=ws1)
    y2 = fp4_linear(x, c, s_, t, cfg.fmt, workspace=ws1)
    y3 = fp4_linear(x, c, s_, t, cfg.fmt, workspace=ws2)
    torch.cuda.synchronize()
    b1 = y1.view(torch.int16)
    assert torch.equal(b1, y2.view(torch.int16))
    assert torch.equal(b1, y3.view(torch.int16))
    yg = torch.empty_like(y1)
    st = torch.cuda.Stream()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.stream(st):
        fp4_linear(x, c, s_, t, cfg.fmt, workspace=ws1, y=yg)
        torch.cuda.synchronize()
        with torch.cuda.graph(g, stream=st):
            fp4_linear(x, c, s_, t, cfg.fmt, workspace=ws1, y=yg)
    for _ in range(3):
        yg.fill_(float("nan"))
        with torch.cuda.stream(st):
            g.replay()
        torch.cuda.synchronize()
        assert torch.equal(b1, yg.view(torch.int16))
    assert api.fp4_workspace_status(ws1) == "FP4_OK"
    del g
