"""Planted mistakes for the control tests.  Each one is a plausible slip of an FP4 MoE
implementation; planted into the oracle's quantised weights (CPU) or into the packed
weights the GPU reads (device data only, never a kernel), it must turn the parity gate
red on the same inputs the parity tests use.

* ``scale_byte``: the first block scale of every expert's first gate row raised (UE8M0
  byte + 8, i.e. x 2^8; or the E4M3 exponent field + 4, i.e. x 16) -- a flipped or
  misindexed scale byte.
* ``nibble_swap``: the two codes of every byte exchanged -- the wrong nibble order.
* ``skip_tensor_scale``: NVFP4's per-tensor float32 scale left out (taken as 1).
* ``drop_clamp``: the SwiGLU clamp limit raised from 7 to 128 -- the clamp omitted.
"""
from __future__ import annotations

import numpy as np

CONTROLS = ("scale_byte", "nibble_swap", "skip_tensor_scale", "drop_clamp")


def bump_scale_byte(b, fmt):
    """The scale byte of a block made 2^8 (UE8M0) or 2^4 (E4M3) times larger."""
    b = int(b)
    if fmt == "mxfp4":
        return min(b + 8, 254)
    e = (b >> 3) & 0xF                      # E4M3: raise the exponent field by 4 (x16)
    return (b & 0x87) | (min(e + 4, 14) << 3)


def swap_nibbles(codes):
    c = np.asarray(codes, dtype=np.uint8)
    return ((c >> 4) | (c << 4)).astype(np.uint8)


def corrupt_oracle(name, fmt):
    """A function (bank, e) -> None planting ``name`` into expert e of an oracle bank
    (module-level, so spawn workers can receive it)."""
    return {"scale_byte": _plant_scale, "nibble_swap": _plant_swap,
            "skip_tensor_scale": _plant_skip_ts}.get(name)


def _plant_scale(bank, e):
    for which in ("gu",):
        c, s, t = bank.packed(which, e)
        s = s.copy()
        s[0, 0] = bump_scale_byte(s[0, 0], bank.fmt)
        bank._cache[(which, e)] = (c, s, t)


def _plant_swap(bank, e):
    for which in ("gu", "dn"):
        c, s, t = bank.packed(which, e)
        bank._cache[(which, e)] = (swap_nibbles(c), s, t)


def _plant_skip_ts(bank, e):
    for which in ("gu", "dn"):
        c, s, t = bank.packed(which, e)
        bank._cache[(which, e)] = (c, s, np.float32(1.0))
