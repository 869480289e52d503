"""fp4_pack / fp4_unpack on the GPU against the oracle: bit-exact."""
import numpy as np
import pytest
import torch

from oracle import formats as F
from synth import draws as D

pytestmark = pytest.mark.gpu


def _to_dev(a):
    return torch.from_numpy(np.ascontiguousarray(a)).cuda()


def _quant_oracle(w, fmt):
    if fmt == "mxfp4":
        c, s = F.mxfp4_quantize(w)
        return c, s, None
    return F.nvfp4_quantize(w)


def _pack_gpu(w_dev, fmt):
    from fp4_block_scaled_moe_b200 import fp4_pack
    c, s, t = fp4_pack(w_dev, fmt)
    torch.cuda.synchronize()
    return c.cpu().numpy(), s.cpu().numpy(), (None if t is None else t.cpu().numpy())


def _assert_same(got, want, fmt):
    assert np.array_equal(got[0], want[0]), "codes differ"
    assert np.array_equal(got[1], want[1]), "scales differ"
    if fmt == "nvfp4":
        assert np.array_equal(got[2].view(np.uint32), np.asarray(want[2], np.float32).view(np.uint32))


@pytest.mark.parametrize("fmt", ["mxfp4", "nvfp4"])
@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_pack_t4_weights(fmt, dtype):
    w = D.expert_weights(0, 50, (3, 40, 512), outliers=(0.003, 10.0, 49.0)).reshape(3, 40, 512)
    if dtype == "bf16":
        bits = D.f32_to_bf16_bits(w)
        w = D.bf16_bits_to_f32(bits).reshape(w.shape)
        dev = _to_dev(bits.view(np.int16).reshape(w.shape)).view(torch.bfloat16)
    else:
        dev = _to_dev(w)
    _assert_same(_pack_gpu(dev, fmt), _quant_oracle(w, fmt), fmt)


def _adversarial_rows(block):
    rng = np.random.default_rng(20)
    mags = np.array([0, .5, 1, 1.5, 2, 3, 4, 6])
    mids = np.array([.25, .75, 1.25, 1.75, 2.5, 3.5, 5.0])
    rows = []
    for e in (-130, -127, -126, -100, -20, -3, 0, 7, 60, 120, 125):
        sc = 2.0 ** e
        r = rng.choice(np.concatenate([mags, mids, -mags, -mids]), size=4 * block) * sc
        r[0] = 6 * sc
        rows.append(r)
    rows.append(np.zeros(4 * block))
    rows.append(-np.zeros(4 * block))
    r = rng.normal(size=4 * block); r[3] = np.inf; rows.append(r)
    r = rng.normal(size=4 * block); r[block + 1] = np.nan; rows.append(r)
    r = rng.normal(size=4 * block) * 1e-40; rows.append(r)           # subnormal amax
    r = rng.normal(size=4 * block) * 1e37; rows.append(r)            # near the float32 top
    r = rng.normal(size=4 * block); r[5] = 7.0; r[6] = 7.9; rows.append(r)   # saturation
    r = rng.normal(size=4 * block) * 1e-3; r[:block] *= 1e-7; rows.append(r)  # tiny blocks beside big
    with np.errstate(over="ignore"):
        return np.stack(rows).astype(np.float32)


@pytest.mark.parametrize("fmt", ["mxfp4", "nvfp4"])
def test_pack_adversarial(fmt):
    block = 32 if fmt == "mxfp4" else 16
    w = _adversarial_rows(block)
    if fmt == "nvfp4":      # per-row tensors, so each row gets its own global scale
        w = w[:, None, :]
    _assert_same(_pack_gpu(_to_dev(w), fmt), _quant_oracle(w, fmt), fmt)


@pytest.mark.parametrize("fmt", ["mxfp4", "nvfp4"])
@pytest.mark.parametrize("out", ["f32", "bf16"])
def test_unpack_bit_exact(fmt, out):
    from fp4_block_scaled_moe_b200 import fp4_unpack
    rng = np.random.default_rng(21)
    B = 32 if fmt == "mxfp4" else 16
    n, k = 37, 256
    codes = rng.integers(0, 256, size=(2, n, k // 2), dtype=np.uint8)
    scales = rng.integers(0, 256, size=(2, n, k // B), dtype=np.uint8)
    ts = np.array([3.0e-3, 7.5], dtype=np.float32) if fmt == "nvfp4" else None
    if fmt == "mxfp4":
        ref = F.mxfp4_dequantize(codes, scales)
    else:
        ref = F.nvfp4_dequantize(codes, scales, ts)
    got = fp4_unpack(_to_dev(codes), _to_dev(scales), None if ts is None else _to_dev(ts), fmt,
                     torch.float32 if out == "f32" else torch.bfloat16)
    torch.cuda.synchronize()
    nan = np.isnan(ref)
    if out == "f32":
        g = got.cpu().numpy()
        assert np.all(np.isnan(g[nan]))
        with np.errstate(over="ignore"):
            want = ref[~nan].astype(np.float32)
        assert np.array_equal(g[~nan].view(np.uint32), want.view(np.uint32))
    else:
        g = got.view(torch.int16).cpu().numpy().view(np.uint16)
        assert np.all(np.isnan(D.bf16_bits_to_f32(g[nan])))
        with np.errstate(over="ignore"):
            want = F.bf16_bits(F.round_to_bf16(ref[~nan]))
        assert np.array_equal(g[~nan], want)
