"""The V2a packer on the GPU is bit-exact with the oracle (codes, group records, library,
outlier CSR) for 2- and 4-bit codes, float32 and bf16 weights; the GPU's dense term is
bit-exact with the oracle's reconstruction."""
import numpy as np
import pytest
import torch

from oracle import formats as F, v2a as V
from synth import draws as D

pytestmark = pytest.mark.gpu


def _weights(batch, rows, k, seed, dtype):
    w = D.expert_weights(seed, 77, (batch * rows, k), sigma=0.02, outliers=(0.004, 6.0, 49.0)).reshape(batch, rows, k)
    if dtype == "bf16":
        w = D.bf16_bits_to_f32(D.f32_to_bf16_bits(w)).reshape(w.shape)
    return w


@pytest.mark.parametrize("n_bits", [4, 2])
@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("batch,rows,k", [(2, 64, 256), (1, 96, 768)])
def test_pack_v2a_bit_exact(n_bits, dtype, batch, rows, k):
    from fp4_block_scaled_moe_b200 import fp4_pack_v2a, fp4_unpack_v2a
    w = _weights(batch, rows, k, 5 + n_bits, dtype)
    t = torch.from_numpy(w).cuda()
    if dtype == "bf16":
        t = t.to(torch.bfloat16)
    thr = 6 * 0.02
    got = fp4_pack_v2a(t, n_bits, thr)
    dense = fp4_unpack_v2a(got["codes"], got["groups"], got["lib"], batch, rows, k, n_bits).cpu().numpy()
    torch.cuda.synchronize()
    rec = got["groups"].cpu().numpy().view(np.uint64)
    nnz_seen = 0
    for b in range(batch):
        fit = V.v2a_fit(w[b], n_bits, thr)
        sl = slice(b * rows, (b + 1) * rows)
        assert np.array_equal(got["lib"][b].cpu().numpy().view(np.uint16), fit["lib"]), "library"
        assert np.array_equal(got["codes"][sl].cpu().numpy(), fit["codes"]), "codes"
        r = rec[sl]
        assert np.array_equal((r & 0xFFFF).astype(np.uint16), F.f16_bits(fit["mid"])), "mid"
        assert np.array_equal(((r >> 16) & 0xFFFF).astype(np.uint16), F.f16_bits(fit["scale"])), "scale"
        assert np.array_equal((r >> 32).astype(np.uint8), fit["lib_idx"]), "library index"
        assert np.array_equal(dense[b].astype(np.float64), V.v2a_dense(fit, k)), "dense term"
        rp = got["row_ptr"].cpu().numpy()[b * rows:(b + 1) * rows + 1]
        assert np.array_equal(rp - rp[0], fit["row_ptr"])
        lo, hi = int(rp[0]), int(rp[-1])
        assert np.array_equal(got["col"].cpu().numpy()[lo:hi], fit["col"])
        assert np.array_equal(got["val"].cpu().numpy()[lo:hi].view(np.uint16), F.f16_bits(fit["val"]))
        nnz_seen += hi - lo
    assert nnz_seen > 0
