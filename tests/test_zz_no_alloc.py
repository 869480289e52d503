"""The allocation-free forward entry point, for callers that cannot allocate device
memory (a graph captured once, a plugin whose host owns every allocation, a real-time
loop).  It must give the same layer output as moe_fp4_forward, call after call, while
taking its scratch from the library's fixed device buffer.

This file is collected last on purpose: the entry point's buffer is shared per device,
so it also runs after everything else the suite did on the GPU."""
import ctypes

import numpy as np
import pytest
import torch

from synth import configs as C, draws as D

from helpers import check_tolerance, device_weights, host_small_inputs

pytestmark = pytest.mark.gpu


def _noalloc(lib, wstruct, x, wr, bias, T, k, y):
    return lib.moe_fp4_forward_noalloc(ctypes.byref(wstruct), ctypes.c_void_p(x.data_ptr()),
                                       ctypes.c_void_p(wr.data_ptr()),
                                       None if bias is None else ctypes.c_void_p(bias.data_ptr()), T, k,
                                       ctypes.c_void_p(y.data_ptr()),
                                       ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))


def _y_host(y):
    return D.bf16_bits_to_f32(y.view(torch.int16).cpu().numpy().view(np.uint16)).reshape(y.shape)


# nvfp4_small and c2_full run the CUDA-core GEMV kernels; c2_full_tensor the tensor-core
# kernels with the weights' re-laid scale atoms (3.3 MiB of scratch).
@pytest.mark.parametrize("cfg,tensor", [(C.small(C.MOE_C3), False), (C.MOE_C2, False), (C.MOE_C2, True)],
                         ids=["nvfp4_small", "c2_full", "c2_full_tensor"])
def test_noalloc_matches_forward_two_calls(cfg, tensor):
    from fp4_block_scaled_moe_b200 import _lib as L, moe_fp4_expert_kernels, moe_fp4_forward, prepare_mma_scales
    lib = L.load()
    x_bits, wr, bias = host_small_inputs(cfg)
    w = device_weights(cfg)
    if tensor:
        prepare_mma_scales(w)
        w.kernel_variant = 2
    assert moe_fp4_expert_kernels(w, cfg.T, cfg.k) == (2 if tensor else 1)
    ws = w.c_struct()
    wr_t = torch.from_numpy(wr).cuda()
    bias_t = None if bias is None else torch.from_numpy(bias).cuda()
    x1 = torch.from_numpy(x_bits.view(np.int16)).cuda().view(torch.bfloat16)
    x2 = (x1.float() * -0.5).to(torch.bfloat16)                  # a different batch for the second call
    for x in (x1, x2):
        ref = moe_fp4_forward(w, x, wr_t, bias_t, cfg.k)
        y = torch.full((cfg.T, cfg.H), float("nan"), dtype=torch.bfloat16, device="cuda")
        assert _noalloc(lib, ws, x, wr_t, bias_t, cfg.T, cfg.k, y) == 0
        torch.cuda.synchronize()
        # the same kernels on the same inputs: identical bits, and within the gates
        assert torch.equal(y.view(torch.int16), ref.view(torch.int16))
        check_tolerance(_y_host(y), _y_host(ref))
        assert lib.moe_fp4_noalloc_status(ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)) == 0


def test_noalloc_refuses_a_batch_larger_than_its_buffer():
    from fp4_block_scaled_moe_b200 import _lib as L
    lib = L.load()
    cfg = C.small(C.MOE_C2)
    w = device_weights(cfg)
    ws = w.c_struct()
    T = 4096                                                       # workspace far above the 16 MiB buffer
    assert lib.moe_fp4_workspace_size(ctypes.byref(ws), T, cfg.k) > lib.moe_fp4_noalloc_capacity()
    x = torch.zeros((T, cfg.H), dtype=torch.bfloat16, device="cuda")
    wr = torch.zeros((cfg.E, cfg.H), dtype=torch.float32, device="cuda")
    y = torch.full((T, cfg.H), 3.0, dtype=torch.bfloat16, device="cuda")
    assert _noalloc(lib, ws, x, wr, None, T, cfg.k, y) == 6      # FP4_ERR_WORKSPACE
    torch.cuda.synchronize()
    assert bool((y == 3.0).all())                                  # nothing launched


def test_noalloc_status_reports_a_timed_out_wait():
    """A bounded device wait that gives up in the fixed buffer's control block is
    reported by moe_fp4_noalloc_status (and cleared), and the next call is correct."""
    from fp4_block_scaled_moe_b200 import _lib as L, moe_fp4_forward
    lib = L.load()
    st = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    cfg = C.small(C.MOE_C2)
    x_bits, wr, bias = host_small_inputs(cfg)
    w = device_weights(cfg)
    x = torch.from_numpy(x_bits.view(np.int16)).cuda().view(torch.bfloat16)
    wr_t = torch.from_numpy(wr).cuda()
    y = torch.empty((cfg.T, cfg.H), dtype=torch.bfloat16, device="cuda")
    assert _noalloc(lib, w.c_struct(), x, wr_t, None, cfg.T, cfg.k, y) == 0
    assert lib.moe_fp4_noalloc_status(st) == 0
    assert lib.fp4_selftest_wait_timeout(None, 2_000_000, st) == 0        # NULL: the fixed buffer
    assert lib.moe_fp4_noalloc_status(st) == 8                            # FP4_ERR_TIMEOUT
    assert lib.moe_fp4_noalloc_status(st) == 0                            # read clears it
    assert _noalloc(lib, w.c_struct(), x, wr_t, None, cfg.T, cfg.k, y) == 0
    ref = moe_fp4_forward(w, x, wr_t, None, cfg.k)
    torch.cuda.synchronize()
    assert torch.equal(y.view(torch.int16), ref.view(torch.int16))
