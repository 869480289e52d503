"""CB4 packing on the GPU against the oracle's fit, bit for bit: indices, fp16
codebooks, CSR row pointers, columns and fp16 residual values."""
import numpy as np
import pytest
import torch

from oracle import codebook as CB
from synth import configs as C, draws as D

pytestmark = pytest.mark.gpu


def _check(w32, thr, mu=0.0, dtype=torch.float32):
    from fp4_block_scaled_moe_b200 import fp4_pack_cb4
    wt = torch.from_numpy(w32).cuda()
    if dtype == torch.bfloat16:
        wt = wt.to(torch.bfloat16)
        w32 = wt.float().cpu().numpy()           # the values the packer sees
    got = fp4_pack_cb4(wt, thr, mu)
    torch.cuda.synchronize()
    ref = CB.cb4_fit(w32, thr, mu)
    assert np.array_equal(got["row_ptr"].cpu().numpy(), ref["row_ptr"])
    assert np.array_equal(got["col"].cpu().numpy(), ref["col"])
    assert np.array_equal(got["val"].cpu().numpy().view(np.uint16),
                          ref["val"].astype(np.float16).view(np.uint16))
    assert np.array_equal(got["cb"].cpu().numpy().view(np.uint16), ref["cb"])
    assert np.array_equal(got["idx"].cpu().numpy(), ref["idx"])
    return ref


@pytest.mark.parametrize("rows,k", [(64, 512), (7, 128), (33, 1024)])
def test_cb4_pack_bit_exact_t4_with_outliers(rows, k):
    cfg = C.MOE_C5
    w = D.expert_weights(cfg.seed, C.TID_GATE_UP, (rows, k), sigma=cfg.sigma, outliers=cfg.outliers)
    ref = _check(w, cfg.cb4_threshold_sigma * cfg.sigma)
    assert ref["row_ptr"][-1] > 0                  # the sparse term is exercised


def test_cb4_pack_bit_exact_bf16_input_and_mu():
    cfg = C.MOE_C5
    w = D.expert_weights(cfg.seed, C.TID_DOWN, (40, 256), sigma=cfg.sigma, outliers=cfg.outliers)
    _check(w, 0.1, mu=0.003, dtype=torch.bfloat16)


def test_cb4_pack_degenerate_groups():
    """Constant groups, a group with fewer than 16 distinct values, exact ties and no
    outliers at all."""
    w = np.zeros((4, 256), dtype=np.float32)
    w[1] = 0.01
    w[2, :128] = np.repeat(np.arange(8, dtype=np.float32) * 0.001, 16)
    w[3] = np.tile(np.array([-0.02, 0.02], dtype=np.float32), 128)
    ref = _check(w, 0.5)
    assert ref["row_ptr"][-1] == 0
