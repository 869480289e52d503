"""Seeded synthetic inputs for the routed-expert MoE layer.

Two kinds of tensor are drawn here:

* Expert weights (large): a counter-based recipe, so that the device can draw
  any slice of them on its own (``synth/csrc/synth_gen.cu``) and the host can
  draw the same slice again, bit for bit, for a spot check. Each element is a
  Student-t draw with nu = 4 scaled to standard deviation sigma (Bailey's polar
  method, "Polar generation of random variates with the t-distribution",
  Math. Comp. 62 (1994)), optionally replaced by a planted outlier. Only
  correctly rounded float32 operations (+, -, *, /, sqrt) are used, in a fixed
  order, so that host and device agree exactly.
* Activations, router weights and the router bias (small): numpy's PCG64 on
  the host, copied to the device by whoever needs them.

Nothing here quantises, routes or multiplies: the method's arithmetic lives in
``oracle/`` and in the CUDA library, which share none of it.
"""
from __future__ import annotations

import numpy as np

from .philox import philox4x32_10

# Reserved third counter word for the outlier draw of an element.
OUTLIER_ATTEMPT = 0xFFFFFFFF
MAX_ATTEMPTS = 8
_TWO_M23 = np.float32(2.0 ** -23)
_TWO_M24 = np.float32(2.0 ** -24)


def t4_scale(sigma: float) -> np.float32:
    """Factor that maps a unit Student-t(4) draw (variance 2) to std ``sigma``."""
    return np.float32(sigma / np.sqrt(2.0))


def _signed_uniform(r: np.ndarray) -> np.ndarray:
    """uint32 word -> float32 in [-1, 1), a multiple of 2^-23 (exact)."""
    return ((r >> np.uint32(8)).astype(np.int64) - (1 << 23)).astype(np.float32) * _TWO_M23


def _unit_uniform(r: np.ndarray) -> np.ndarray:
    """uint32 word -> float32 in [0, 1), a multiple of 2^-24 (exact)."""
    return (r >> np.uint32(8)).astype(np.float32) * _TWO_M24


def _polar_t4(u: np.ndarray, v: np.ndarray, w: np.ndarray) -> np.ndarray:
    """Bailey's polar step for nu = 4 in float32: u * sqrt(4 (w^-1/2 - 1) / w)."""
    s = np.sqrt(w)
    s = np.float32(1.0) / s
    s = s - np.float32(1.0)
    s = s * np.float32(4.0)
    s = s / w
    s = np.sqrt(s)
    return u * s


def t4_draws(seed: int, tensor_id: int, start: int, count: int) -> np.ndarray:
    """Unit Student-t(4) draws for element indices [start, start + count) (float32)."""
    idx = np.arange(start, start + count, dtype=np.uint64)
    lo = (idx & np.uint64(0xFFFFFFFF)).astype(np.uint32)
    hi = (idx >> np.uint64(32)).astype(np.uint32)
    out = np.zeros(count, dtype=np.float32)
    todo = np.arange(count)
    for attempt in range(MAX_ATTEMPTS):
        if todo.size == 0:
            break
        r0, r1, r2, r3 = philox4x32_10(lo[todo], hi[todo], np.uint32(attempt), np.uint32(0),
                                       np.uint32(seed), np.uint32(tensor_id))
        done = np.zeros(todo.size, dtype=bool)
        for ra, rb in ((r0, r1), (r2, r3)):
            u = _signed_uniform(ra)
            v = _signed_uniform(rb)
            w = u * u + v * v
            ok = (w > 0) & (w <= 1) & ~done
            if ok.any():
                with np.errstate(divide="ignore", invalid="ignore"):
                    t = _polar_t4(u, v, w)
                out[todo[ok]] = t[ok]
                done |= ok
        todo = todo[~done]
    return out


def planted_outliers(seed: int, tensor_id: int, start: int, count: int, frac: float,
                     lo_sigma: float, hi_sigma: float, sigma: float):
    """Positions and values of planted outliers: |w| = (lo + (hi - lo) u) sigma, random sign.

    Returns (mask, values) for element indices [start, start + count).
    """
    idx = np.arange(start, start + count, dtype=np.uint64)
    lo = (idx & np.uint64(0xFFFFFFFF)).astype(np.uint32)
    hi = (idx >> np.uint64(32)).astype(np.uint32)
    r0, r1, r2, _ = philox4x32_10(lo, hi, np.uint32(OUTLIER_ATTEMPT), np.uint32(0),
                                  np.uint32(seed), np.uint32(tensor_id))
    mask = _unit_uniform(r0) < np.float32(frac)
    m = np.float32(hi_sigma - lo_sigma) * _unit_uniform(r1)
    m = np.float32(lo_sigma) + m
    m = m * np.float32(sigma)
    neg = (r2 & np.uint32(1)).astype(bool)
    vals = np.where(neg, -m, m).astype(np.float32)
    return mask, vals


_HOST_LIB = None


def _host_lib():
    """The C twin of this recipe (synth/csrc/synth_host.c), or None if it is not built."""
    global _HOST_LIB
    if _HOST_LIB is None:
        import ctypes
        import os
        path = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libfp4synth_host.so")
        if not os.path.exists(path):
            return None
        lib = ctypes.CDLL(path)
        lib.synth_t4_host.restype = None
        lib.synth_t4_host.argtypes = [ctypes.c_void_p, ctypes.c_int64, ctypes.c_int64, ctypes.c_uint32,
                                      ctypes.c_uint32, ctypes.c_float, ctypes.c_int, ctypes.c_float,
                                      ctypes.c_float, ctypes.c_float, ctypes.c_float]
        _HOST_LIB = lib
    return _HOST_LIB


def expert_weights_c(seed, tensor_id, start, count, sigma=0.02, outliers=None):
    """Same draws as the numpy path below, computed by the C twin (multi-threaded)."""
    import ctypes
    lib = _host_lib()
    out = np.empty(count, dtype=np.float32)
    if outliers is None:
        wo, frac, lo, span = 0, 0.0, 0.0, 0.0
    else:
        frac, lo_s, hi_s = outliers
        wo, frac, lo, span = 1, float(np.float32(frac)), float(np.float32(lo_s)), float(np.float32(hi_s - lo_s))
    lib.synth_t4_host(out.ctypes.data_as(ctypes.c_void_p), start, count, seed, tensor_id, float(t4_scale(sigma)),
                      wo, frac, lo, span, float(np.float32(sigma)))
    return out


def expert_weights(seed: int, tensor_id: int, shape, start_row: int = 0, rows: int | None = None,
                   sigma: float = 0.02, outliers=None, use_c: bool = True) -> np.ndarray:
    """Rows [start_row, start_row + rows) of a weight tensor of ``shape`` (last dim = K).

    The tensor is flattened row-major; element i of the flattened tensor is
    drawn from counter i. ``outliers`` is None or (frac, lo_sigma, hi_sigma).
    ``use_c`` takes the C twin when it is built (identical bits, much faster).
    """
    k = int(shape[-1])
    total_rows = int(np.prod(shape[:-1]))
    if rows is None:
        rows = total_rows - start_row
    assert 0 <= start_row and start_row + rows <= total_rows
    start = start_row * k
    count = rows * k
    if use_c and _host_lib() is not None:
        return expert_weights_c(seed, tensor_id, start, count, sigma, outliers).reshape(rows, k)
    w = t4_draws(seed, tensor_id, start, count) * t4_scale(sigma)
    if outliers is not None:
        frac, lo_s, hi_s = outliers
        mask, vals = planted_outliers(seed, tensor_id, start, count, frac, lo_s, hi_s, sigma)
        w = np.where(mask, vals, w).astype(np.float32)
    return w.reshape(rows, k)


# --- host-side small tensors -------------------------------------------------

def _rng(seed: int, stream: int) -> np.random.Generator:
    return np.random.Generator(np.random.PCG64(np.random.SeedSequence([seed, stream])))


def f32_to_bf16_bits(a: np.ndarray) -> np.ndarray:
    """Round float32 to bfloat16 (nearest, ties to even); returns uint16 bit patterns."""
    b = np.ascontiguousarray(a, dtype=np.float32).view(np.uint32).astype(np.uint64)
    rounded = (b + np.uint64(0x7FFF) + ((b >> np.uint64(16)) & np.uint64(1))) >> np.uint64(16)
    out = rounded.astype(np.uint16)
    nan = np.isnan(a)
    if nan.any():
        out[nan] = 0x7FC0
    return out


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    return (np.asarray(b, dtype=np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32)


def activations_bf16(seed: int, t: int, h: int) -> np.ndarray:
    """x ~ N(0, 1), rounded to float32 then to bf16; returned as uint16 bits [t, h]."""
    x = _rng(seed, 11).standard_normal((t, h)).astype(np.float32)
    return f32_to_bf16_bits(x)


def router_weights(seed: int, e: int, h: int, std: float = 0.02) -> np.ndarray:
    """Router weight ~ N(0, std^2) in float32, [e, h]."""
    return (_rng(seed, 12).standard_normal((e, h)) * std).astype(np.float32)


def zipf_bias(seed: int, e: int, s: float = 1.1) -> np.ndarray:
    """Per-expert logit bias -s ln(rank), rank a seeded permutation of 1..e, centred."""
    rank = _rng(seed, 13).permutation(e).astype(np.float64) + 1.0
    b = -s * np.log(rank)
    return (b - b.mean()).astype(np.float32)
