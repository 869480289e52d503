"""Oracle: the 4-bit element, the block scales, and MXFP4 / NVFP4 block quantisation.

TEST INFRASTRUCTURE ONLY (see ``oracle/__init__``).

Definitions followed:
* E2M1 element: 1 sign, 2 exponent, 1 mantissa bit; NVFP4 and MXFP4 both use
  it ([XFP] 路线二). Value = (-1)^s 2^(e-1) (1 + m/2) for e >= 1 and
  (-1)^s m/2 for e = 0, giving the set {0, +-0.5, +-1, +-1.5, +-2, +-3, +-4, +-6}.
* MXFP4: 32 elements share one 8-bit power-of-two scale, per the OCP
  Microscaling format ([XFP] 路线二). The shared exponent is
  floor(log2(amax)) - 2 (2 = the largest E2M1 exponent), stored biased by 127
  (UE8M0); byte 255 is NaN.
* NVFP4: 16 elements share one FP8 E4M3 scale, and a float32 per-tensor
  ("global") scale multiplies it ([XFP] 路线二; [TF] W4A16_NVFP4 packing with
  the global scale). E4M3: bias 7, no infinities, S.1111.111 is NaN, largest
  finite 448.
* Two 4-bit values per byte ([GATE] "A fused tensor with two dtypes in it");
  the element with the even index takes the low nibble.

Readings where the pages are silent:
* Rounding to E2M1 and to E4M3 is round-to-nearest, ties to the even
  mantissa; values above the largest finite magnitude saturate; the sign of a
  value that rounds to zero is kept (code 8 is -0).
* NVFP4 scale order, in float32 with correctly rounded operations:
  ts = amax_tensor / 2688 (= 6 * 448), or 1 when amax_tensor = 0;
  s_b = E4M3(amax_block / (6 * ts)); q = E2M1(v / (E4M3value(s_b) * ts)).
  A block whose s_b is zero stores all-zero codes.
* Non-finite inputs: an MXFP4 block holding one stores scale 0xFF (NaN) and
  zero codes; an NVFP4 block holding one stores scale 0x7F (NaN) and zero
  codes, and the tensor amax ignores non-finite elements.
"""
from __future__ import annotations

import numpy as np

MX_BLOCK = 32
NV_BLOCK = 16
E2M1_EMAX = 2           # largest E2M1 exponent: 6 = 2^2 * 1.5
E4M3_MAX = 448.0
E2M1_MAX = 6.0


# --- generic float64 -> narrow float rounding ------------------------------------------

def round_to_narrow(a, mant_bits: int, emin: int, emax: int, max_finite: float):
    """Round float64 values to a binary format with ``mant_bits`` fraction bits,
    normal exponent range [emin, emax], subnormals below 2^emin, round to nearest
    with ties to even. Overflow goes to +-inf. Returns float64 holding the
    rounded values exactly.
    """
    a = np.asarray(a, dtype=np.float64)
    out = np.array(a, dtype=np.float64, copy=True)
    fin = np.isfinite(a) & (a != 0)
    x = a[fin]
    mag = np.abs(x)
    _, ex = np.frexp(mag)                 # mag = f * 2^ex, f in [0.5, 1)
    e = np.maximum(ex - 1, emin)          # exponent of the binade (subnormals share emin)
    ulp_exp = e - mant_bits
    q = np.ldexp(np.rint(np.ldexp(mag, -ulp_exp)), ulp_exp)   # rint: ties to even
    q = np.where(q > max_finite, np.inf, q)
    out[fin] = np.copysign(q, x)
    return out


def round_to_bf16(a):
    """float64 -> nearest bfloat16 value (ties to even), as float64."""
    return round_to_narrow(a, 7, -126, 127, float.fromhex("0x1.fep127"))


def round_to_f16(a):
    """float64 -> nearest IEEE binary16 value (ties to even), as float64."""
    return round_to_narrow(a, 10, -14, 15, 65504.0)


def f16_bits(a):
    """float64 values already representable in binary16 -> uint16 bit patterns."""
    return np.asarray(a, dtype=np.float64).astype(np.float16).view(np.uint16)


def bf16_bits(a):
    """float64 values already representable in bfloat16 -> uint16 bit patterns."""
    f = np.asarray(a, dtype=np.float64).astype(np.float32).view(np.uint32)
    return (f >> np.uint32(16)).astype(np.uint16)


# --- E2M1 ------------------------------------------------------------------------------

def e2m1_value(code):
    """Decode 4-bit E2M1 codes (uint8 0..15) from their bit fields; float64."""
    code = np.asarray(code).astype(np.int64)
    s = (code >> 3) & 1
    e = (code >> 1) & 3
    m = code & 1
    mag = np.where(e == 0, 0.5 * m, np.ldexp(1.0 + 0.5 * m, e - 1))
    return np.where(s == 1, -mag, mag)


_E2M1_MAGS = [float(e2m1_value(c)) for c in range(8)]


def e2m1_round(a):
    """Nearest E2M1 code of each float64 value (ties to the even mantissa, saturating
    at 6, sign kept). NaN maps to code 0."""
    a = np.asarray(a, dtype=np.float64)
    mag = np.minimum(np.abs(a), E2M1_MAX)      # saturation: anything above 6 is nearest to 6
    best = np.zeros(a.shape, dtype=np.uint8)
    best_d = np.abs(mag - _E2M1_MAGS[0])
    for c in range(1, 8):
        d = np.abs(mag - _E2M1_MAGS[c])
        take = (d < best_d) | ((d == best_d) & (c % 2 == 0))
        best = np.where(take, np.uint8(c), best)
        best_d = np.where(take, d, best_d)
    best = np.where(np.isnan(a), np.uint8(0), best)
    sign = np.signbit(a) & ~np.isnan(a)
    return (best | (sign.astype(np.uint8) << 3)).astype(np.uint8)


# --- UE8M0 and E4M3 scales -------------------------------------------------------------

def ue8m0_value(byte):
    """UE8M0 scale byte -> 2^(byte - 127); 255 is NaN."""
    b = np.asarray(byte).astype(np.int64)
    return np.where(b == 255, np.nan, np.ldexp(1.0, b - 127))


def e4m3_value(code):
    """Decode FP8 E4M3 bytes from their bit fields; float64 (NaN for S.1111.111)."""
    c = np.asarray(code).astype(np.int64)
    s = (c >> 7) & 1
    e = (c >> 3) & 15
    m = c & 7
    mag = np.where(e == 0, np.ldexp(m / 8.0, -6), np.ldexp(1.0 + m / 8.0, e - 7))
    mag = np.where((e == 15) & (m == 7), np.nan, mag)
    return np.where(s == 1, -mag, mag)


_E4M3_MAGS = e4m3_value(np.arange(127))   # codes 0..126: all finite non-negative values, ascending


def e4m3_round(a):
    """Nearest non-negative E4M3 code of float64 values >= 0 (ties to even,
    saturating at 448). NaN maps to 0x7F."""
    a = np.asarray(a, dtype=np.float64)
    x = np.minimum(np.where(np.isnan(a), 0.0, a), E4M3_MAX)
    hi = np.clip(np.searchsorted(_E4M3_MAGS, x, side="left"), 0, 126)
    lo = np.clip(hi - 1, 0, 126)
    d_hi = _E4M3_MAGS[hi] - x
    d_lo = x - _E4M3_MAGS[lo]
    pick_lo = (d_lo < d_hi) | ((d_lo == d_hi) & (lo % 2 == 0))
    code = np.where(pick_lo, lo, hi).astype(np.uint8)
    return np.where(np.isnan(a), np.uint8(0x7F), code).astype(np.uint8)


# --- nibble packing --------------------------------------------------------------------

def pack_nibbles(codes):
    """[..., K] codes 0..15 -> [..., K/2] bytes, even index in the low nibble."""
    c = np.asarray(codes, dtype=np.uint8)
    return (c[..., 0::2] | (c[..., 1::2] << 4)).astype(np.uint8)


def unpack_nibbles(packed):
    p = np.asarray(packed, dtype=np.uint8)
    out = np.empty(p.shape[:-1] + (p.shape[-1] * 2,), dtype=np.uint8)
    out[..., 0::2] = p & 0xF
    out[..., 1::2] = p >> 4
    return out


# --- MXFP4 -----------------------------------------------------------------------------

def mxfp4_quantize(w):
    """w: float32 [..., K], K % 32 == 0 -> (codes uint8 [..., K/2], scales uint8 [..., K/32])."""
    w = np.asarray(w, dtype=np.float32)
    K = w.shape[-1]
    assert K % MX_BLOCK == 0
    blocks = w.reshape(w.shape[:-1] + (K // MX_BLOCK, MX_BLOCK)).astype(np.float64)
    finite = np.isfinite(blocks).all(axis=-1)
    amax = np.where(finite, np.abs(np.where(np.isfinite(blocks), blocks, 0.0)).max(axis=-1), 0.0)
    _, ex = np.frexp(amax)                                  # amax = f 2^ex, f in [0.5, 1)
    e_s = np.where(amax > 0, ex - 1 - E2M1_EMAX, -127)      # floor(log2 amax) - 2
    e_s = np.clip(e_s, -127, 127)
    scales = np.where(finite, e_s + 127, 255).astype(np.uint8)
    scaled = np.ldexp(np.where(np.isfinite(blocks), blocks, 0.0), -e_s[..., None])  # exact
    codes = e2m1_round(scaled)
    codes = np.where(finite[..., None], codes, np.uint8(0))
    codes = codes.reshape(w.shape)
    return pack_nibbles(codes), scales


def mxfp4_dequantize(codes_packed, scales):
    """-> float64 [..., K]: E2M1(code) * 2^(byte - 127)."""
    codes = unpack_nibbles(codes_packed)
    K = codes.shape[-1]
    v = e2m1_value(codes).reshape(codes.shape[:-1] + (K // MX_BLOCK, MX_BLOCK))
    return (v * ue8m0_value(scales)[..., None]).reshape(codes.shape)


# --- NVFP4 -----------------------------------------------------------------------------

def nvfp4_quantize(w):
    """w: float32 [..., N, K] (each trailing [N, K] matrix is one tensor), K % 16 == 0
    -> (codes uint8 [..., N, K/2], scales uint8 E4M3 [..., N, K/16], tensor_scale f32 [...])."""
    w = np.asarray(w, dtype=np.float32)
    lead = w.shape[:-2]
    N, K = w.shape[-2:]
    assert K % NV_BLOCK == 0
    flat = w.reshape((-1, N * K))
    fin = np.isfinite(flat)
    amax_t = np.where(fin, np.abs(flat), np.float32(0)).max(axis=-1).astype(np.float32)
    ts = np.where(amax_t > 0, amax_t / np.float32(6.0 * E4M3_MAX), np.float32(1.0)).astype(np.float32)
    six_ts = (np.float32(6.0) * ts).astype(np.float32)
    blocks = flat.reshape((flat.shape[0], N * K // NV_BLOCK, NV_BLOCK))
    bfin = np.isfinite(blocks).all(axis=-1)
    amax_b = np.where(bfin, np.abs(np.where(np.isfinite(blocks), blocks, np.float32(0))).max(axis=-1),
                      np.float32(0)).astype(np.float32)
    s = (amax_b / six_ts[:, None]).astype(np.float32)
    sb = e4m3_round(s.astype(np.float64))
    sbv = e4m3_value(sb).astype(np.float32)
    denom = (sbv * ts[:, None]).astype(np.float32)
    safe = (denom > 0)[..., None] & np.ones(blocks.shape, dtype=bool)
    with np.errstate(divide="ignore", invalid="ignore"):
        q = (np.where(np.isfinite(blocks), blocks, np.float32(0)) / denom[..., None]).astype(np.float32)
    codes = e2m1_round(q.astype(np.float64))
    codes = np.where(safe & bfin[..., None], codes, np.uint8(0))
    sb = np.where(bfin, sb, np.uint8(0x7F)).astype(np.uint8)
    codes = codes.reshape(lead + (N, K))
    return (pack_nibbles(codes), sb.reshape(lead + (N, K // NV_BLOCK)), ts.reshape(lead))


def nvfp4_dequantize(codes_packed, scales, tensor_scale):
    """-> float64 [..., N, K]: E2M1(code) * E4M3(scale) * ts, exact in float64."""
    codes = unpack_nibbles(codes_packed)
    K = codes.shape[-1]
    v = e2m1_value(codes).reshape(codes.shape[:-1] + (K // NV_BLOCK, NV_BLOCK))
    ts = np.asarray(tensor_scale, dtype=np.float64)
    s = e4m3_value(scales) * ts.reshape(ts.shape + (1, 1))
    return (v * s[..., None]).reshape(codes.shape)
