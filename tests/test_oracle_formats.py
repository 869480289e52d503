"""Pins of the oracle's element and block formats (CPU only).

Each check ties oracle.formats to something other than itself: the value
sets and code points fixed by the format definitions (golden fixtures with
citations), exhaustive round trips of representable values, an independent
library implementation (torch's float8_e4m3fn / bfloat16, numpy's float16),
and the 49-sigma worked example of the XFP page.
"""
import math

import numpy as np
import pytest
import torch

from oracle import formats as F


def test_e2m1_value_set(golden):
    rows = golden("e2m1_values.txt")
    assert len(rows) == 16
    for code, val in rows:
        v = F.e2m1_value(int(code))
        assert float(v) == float(val)
        assert math.copysign(1.0, float(v)) == math.copysign(1.0, float(val))
    mags = sorted({abs(float(F.e2m1_value(c))) for c in range(16)})
    assert mags == [0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0]


def test_e2m1_encode_decode_exhaustive():
    codes = np.arange(16, dtype=np.uint8)
    assert np.array_equal(F.e2m1_round(F.e2m1_value(codes)), codes)


def test_e2m1_rounding_points(golden):
    for x, code in golden("e2m1_rounding.txt"):
        assert int(F.e2m1_round(np.float64(x))) == int(code), x


def test_e2m1_nearest_property():
    rng = np.random.default_rng(1)
    x = np.concatenate([rng.uniform(-7, 7, 20000), rng.normal(0, 2, 20000)])
    c = F.e2m1_round(x)
    got = np.abs(F.e2m1_value(c) - x)
    all_d = np.abs(F.e2m1_value(np.arange(16))[None, :] - x[:, None])
    assert np.all(got <= all_d.min(axis=1) + 0.0)
    assert np.all(np.signbit(F.e2m1_value(c)) == np.signbit(x))


def test_e4m3_points(golden):
    for code, val in golden("e4m3_points.txt"):
        v = float(F.e4m3_value(int(code, 16)))
        if val == "nan":
            assert math.isnan(v)
        else:
            assert v == float(val) and math.copysign(1, v) == math.copysign(1, float(val))


def test_e4m3_decode_matches_torch():
    b = torch.arange(256, dtype=torch.uint8).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    ours = F.e4m3_value(np.arange(256))
    both_nan = np.isnan(b) & np.isnan(ours)
    assert np.all(both_nan | (b == ours))


def test_e4m3_encode_exhaustive_and_vs_torch():
    codes = np.arange(127, dtype=np.uint8)
    assert np.array_equal(F.e4m3_round(F.e4m3_value(codes)), codes)
    rng = np.random.default_rng(2)
    x = np.concatenate([rng.uniform(0, 448, 50000), np.exp(rng.uniform(-12, 6, 50000))]).astype(np.float32)
    x = x[x <= 448]
    t = torch.from_numpy(x).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(F.e4m3_round(x.astype(np.float64)), t)
    assert int(F.e4m3_round(np.float64(1e9))) == 0x7E     # satfinite
    assert int(F.e4m3_round(np.float64(2.0 ** -10))) == 0  # tie between 0 and 2^-9 -> even


def test_ue8m0():
    assert float(F.ue8m0_value(127)) == 1.0
    assert float(F.ue8m0_value(0)) == 2.0 ** -127
    assert float(F.ue8m0_value(254)) == 2.0 ** 127
    assert math.isnan(float(F.ue8m0_value(255)))


def test_bf16_f16_rounding_vs_libraries():
    rng = np.random.default_rng(3)
    x = np.concatenate([rng.normal(0, 1, 20000), rng.normal(0, 1e-38, 2000),
                        np.exp(rng.uniform(-100, 88, 20000))]).astype(np.float32)
    tb = torch.from_numpy(x).to(torch.bfloat16).to(torch.float64).numpy()
    assert np.array_equal(F.round_to_bf16(x.astype(np.float64)), tb)
    y = np.concatenate([rng.normal(0, 100, 20000), rng.normal(0, 1e-6, 2000)])
    assert np.array_equal(F.round_to_f16(y), y.astype(np.float16).astype(np.float64))
    assert np.all(np.isinf(F.round_to_f16(np.array([65520.0, -1e6]))))


def test_nibble_order():
    codes = np.array([[1, 2, 3, 4, 15, 0, 7, 8]], dtype=np.uint8)
    p = F.pack_nibbles(codes)
    assert p.tolist() == [[0x21, 0x43, 0x0F, 0x87]]
    assert np.array_equal(F.unpack_nibbles(p), codes)


def _mx_block(byte):
    """All 16 E2M1 codes twice at scale 2^(byte-127), as float32 (exactly representable)."""
    vals = np.ldexp(F.e2m1_value(np.tile(np.arange(16), 2)), byte - 127)
    return vals.astype(np.float32)


def test_mxfp4_roundtrip_exhaustive_bytes():
    # bytes 0..252: 6 * 2^(b-127) is finite in float32 up to b = 252
    rows = np.stack([_mx_block(b) for b in range(0, 253)])
    codes, scales = F.mxfp4_quantize(rows)
    assert np.array_equal(scales[:, 0], np.arange(0, 253, dtype=np.uint8))
    want = F.pack_nibbles(np.tile(np.arange(16, dtype=np.uint8), (253, 2)))
    assert np.array_equal(codes, want)
    assert np.array_equal(F.mxfp4_dequantize(codes, scales), rows.astype(np.float64))


def test_mxfp4_roundtrip_values_any_block():
    rng = np.random.default_rng(4)
    byte = rng.integers(1, 250, size=(500, 1))
    c = rng.integers(0, 16, size=(500, 32))
    w = np.ldexp(F.e2m1_value(c), byte - 127).astype(np.float32)
    codes, scales = F.mxfp4_quantize(w)
    assert np.array_equal(F.mxfp4_dequantize(codes, scales), w.astype(np.float64))


def test_mxfp4_scale_rule_and_saturation():
    e = -5
    blk = np.zeros(32, np.float32)
    blk[3] = 6 * 2.0 ** e
    _, s = F.mxfp4_quantize(blk[None])
    assert int(s[0, 0]) == e + 127
    blk[3] = 7 * 2.0 ** e                        # in (6, 8) * 2^e: saturates to 6
    codes, s = F.mxfp4_quantize(blk[None])
    assert int(s[0, 0]) == e + 127
    assert int(F.unpack_nibbles(codes)[0, 3]) == 7
    blk[3] = 8 * 2.0 ** e                        # next binade: scale goes up
    _, s = F.mxfp4_quantize(blk[None])
    assert int(s[0, 0]) == e + 128
    codes, s = F.mxfp4_quantize(np.zeros((1, 32), np.float32))
    assert int(s[0, 0]) == 0 and not codes.any()
    blk[5] = np.nan
    codes, s = F.mxfp4_quantize(blk[None])
    assert int(s[0, 0]) == 255 and not codes.any()


def test_mxfp4_49_sigma_example():
    """XFP, 路线一: one 49-sigma outlier forces a scale under which the bulk of the
    block (within +-1 sigma) has only zero as its nearest grid point."""
    sigma = 0.02
    rng = np.random.default_rng(5)
    blk = rng.uniform(-sigma, sigma, 32).astype(np.float32)
    blk[17] = 49 * sigma
    codes, _ = F.mxfp4_quantize(blk[None])
    c = F.unpack_nibbles(codes)[0]
    assert np.all((c[np.arange(32) != 17] & 7) == 0)
    assert int(c[17] & 7) != 0
    # the page's linear 4-bit arithmetic: 15 non-zero levels across +-50 sigma
    assert abs(100 / 15 - 6.7) < 0.05


def test_nvfp4_roundtrip_exhaustive_scales():
    """Every positive finite E4M3 scale (subnormals included), each block holding all 16
    codes: with a power-of-two tensor scale the packed form comes back bit for bit."""
    ts = 2.0 ** -10
    sb = np.arange(1, 127)
    w = (F.e2m1_value(np.arange(16))[None, :] * F.e4m3_value(sb)[:, None] * ts).astype(np.float32)
    codes, scales, t = F.nvfp4_quantize(w)
    assert float(t) == ts                                        # amax = 6 * 448 * ts
    assert np.array_equal(scales[:, 0], sb.astype(np.uint8))
    assert np.array_equal(F.unpack_nibbles(codes), np.tile(np.arange(16, dtype=np.uint8), (len(sb), 1)))
    assert np.array_equal(F.nvfp4_dequantize(codes, scales, t), w.astype(np.float64))


def test_nvfp4_two_level_product_exact_in_bf16():
    prod = F.e2m1_value(np.arange(8))[:, None] * F.e4m3_value(np.arange(127))[None, :]
    assert np.array_equal(F.round_to_bf16(prod), prod)
    assert np.array_equal(F.round_to_f16(prod[:, 1:]), prod[:, 1:])    # also in fp16 above 2^-24


def test_nvfp4_scale_formula_small_case():
    """Hand-evaluated: amax_t = 2688 -> ts = 1; a block with amax 6 -> s_b = 1 (0x38)."""
    w = np.zeros((2, 16), np.float32)
    w[0, 0] = 2688.0
    w[1, 0] = 6.0
    w[1, 1] = 1.0
    w[1, 2] = -0.74
    codes, scales, ts = F.nvfp4_quantize(w)
    assert float(ts) == 1.0
    assert scales.tolist() == [[0x7E], [0x38]]
    c = F.unpack_nibbles(codes)
    assert c[1, :3].tolist() == [7, 2, 9]                    # 6, 1, -0.5
    codes, scales, ts = F.nvfp4_quantize(np.zeros((1, 16), np.float32))
    assert float(ts) == 1.0 and not codes.any() and not scales.any()


def test_nvfp4_error_smaller_than_mxfp4_on_t4():
    """XFP 路线二: the fractional FP8 scale gives lower error than the power-of-two one."""
    from synth import draws
    w = draws.expert_weights(0, 99, (64, 256))
    e_mx = F.mxfp4_dequantize(*F.mxfp4_quantize(w)) - w
    e_nv = F.nvfp4_dequantize(*F.nvfp4_quantize(w)) - w
    assert np.linalg.norm(e_nv) < np.linalg.norm(e_mx)


def test_nvfp4_op_order_non_power_of_two_tensor_scale(golden):
    """A hand-worked NVFP4 case (tests/golden/nvfp4_op_order.txt) with a tensor scale that
    is not a power of two: the oracle's codes follow the stated float32 order, and the
    two plausible slips (ts = amax/6/448; dividing by the block scale and the tensor
    scale separately) give a different code on the same value."""
    g = {k: v for k, v in golden("nvfp4_op_order.txt")}
    f = lambda h: np.frombuffer(bytes.fromhex(h)[::-1], dtype=np.float32)[0]
    amax_t, amax_b, v = f(g["amax_t_bits"]), f(g["amax_b_bits"]), f(g["v_bits"])
    w = np.zeros((2, 16), np.float32)
    w[0, 0], w[1, 0], w[1, 1] = amax_t, amax_b, v
    codes, scales, ts = F.nvfp4_quantize(w)
    assert np.float32(ts).tobytes()[::-1].hex() == g["ts_bits"]
    assert scales[:, 0].tolist() == [int(g["scale_row0"], 16), int(g["scale_row1"], 16)]
    c = F.unpack_nibbles(codes)
    assert int(c[0, 0]) == int(g["code_row0_col0"])
    assert int(c[1, 0]) == int(g["code_row1_col0"])
    assert int(c[1, 1]) == int(g["code_row1_col1"])
    assert not c[:, 2:].any() and not c[0, 1:].any()
    # the slips, evaluated in float32 with the same element rounding, give the tie code
    sbv = np.float32(F.e4m3_value(scales[1, 0]))
    ts_slip = np.float32(np.float32(amax_t / np.float32(6)) / np.float32(448))
    assert ts_slip != ts
    six = np.float32(6) * ts_slip
    sb_slip = F.e4m3_round(np.float64(np.float32(amax_b / six)))
    q1 = np.float32(v / np.float32(np.float32(F.e4m3_value(sb_slip)) * ts_slip))
    q2 = np.float32(np.float32(v / sbv) / np.float32(ts))
    assert int(F.e2m1_round(np.float64(q1))) == int(g["slip_code_row1_col1"])
    assert int(F.e2m1_round(np.float64(q2))) == int(g["slip_code_row1_col1"])
