"""moe_route on the GPU: bit-exact ids / counts / offsets / perm / inv on given logits,
and logits from x within float32 accumulation error of the float64 oracle."""
import numpy as np
import pytest
import torch

from oracle import routing as R
from synth import configs as C, draws as D

pytestmark = pytest.mark.gpu


def _run(x=None, wr=None, bias=None, k=8, logits_in=None):
    from fp4_block_scaled_moe_b200 import moe_route
    out = moe_route(x, wr, bias, k, logits_in=logits_in)
    torch.cuda.synchronize()
    return {n: t.cpu().numpy() for n, t in out.items()}


@pytest.mark.parametrize("T,E,k", [(16, 64, 8), (64, 256, 8), (300, 8, 2), (7, 5, 5), (1, 1024, 32), (1000, 33, 3)])
def test_route_given_logits_bit_exact(T, E, k):
    rng = np.random.default_rng(T * 1000 + E)
    lg = rng.integers(-4, 5, size=(T, E)).astype(np.float32)          # many exact ties
    lg[:, ::7] += rng.normal(size=lg[:, ::7].shape).astype(np.float32)
    if T > 1:
        lg[0, :] = -0.0
        lg[0, 1::2] = 0.0
    got = _run(logits_in=torch.from_numpy(lg).cuda(), k=k)
    ids = R.topk(lg, k)
    counts, offsets, perm, inv = R.permutation(ids, E)
    assert np.array_equal(got["topk_ids"], ids)
    assert np.array_equal(got["counts"], counts)
    assert np.array_equal(got["offsets"], offsets)
    assert np.array_equal(got["perm"], perm)
    assert np.array_equal(got["inv"], inv)
    w = R.softmax_selected(lg, ids)
    assert np.allclose(got["topk_w"], w, rtol=2e-6, atol=1e-7)


# C4 (8192 tokens) and a ragged shape take the tensor-core logits kernel (T >= 256)
_RAGGED = C.MoEConfig("route_ragged_t300_e40", "mxfp4", T=300, E=40, H=544, I=256, k=3, zipf_bias=True)


@pytest.mark.parametrize("cfg", [C.MOE_C2, C.MOE_C3, C.MOE_C4, _RAGGED], ids=["c2", "c3", "c4", "ragged_t300_e40"])
def test_route_from_x(cfg):
    x_bits = D.activations_bf16(cfg.seed, cfg.T, cfg.H)
    wr = D.router_weights(cfg.seed, cfg.E, cfg.H)
    bias = D.zipf_bias(cfg.seed, cfg.E) if cfg.zipf_bias else None
    x = torch.from_numpy(x_bits.view(np.int16)).cuda().view(torch.bfloat16)
    got = _run(x, torch.from_numpy(wr).cuda(), None if bias is None else torch.from_numpy(bias).cuda(), cfg.k)
    lg = R.router_logits(D.bf16_bits_to_f32(x_bits), wr, bias)
    assert np.allclose(got["logits"], lg, rtol=1e-5, atol=2e-5)
    ids = R.topk(lg, cfg.k)
    ok = ~R.near_ties(lg, cfg.k)
    assert np.array_equal(got["topk_ids"][ok], ids[ok])
    # every token: the GPU's selection is a valid top-k of the float64 logits
    for t in np.nonzero(~ok)[0]:
        kth = np.sort(lg[t])[::-1][cfg.k - 1]
        assert np.all(lg[t][got["topk_ids"][t]] >= kth - 1e-4 * max(1, abs(kth)))
    counts, offsets, perm, inv = R.permutation(got["topk_ids"], cfg.E)
    assert np.array_equal(got["perm"], perm) and np.array_equal(got["inv"], inv)
