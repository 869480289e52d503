"""Oracle: the dense 4-bit linear layer and the routed-expert MoE layer, in float64.

TEST INFRASTRUCTURE ONLY (see ``oracle/__init__``).

* Linear layer (W4A16, [TF] "What this changes": 4-bit weights read with bf16
  activations): y = x . W^T with W the dequantised weights.
* MoE layer: for each token t and selected slot j with expert e = ids[t, j]:
  [g; u] = W_gu(e) x_t (rows 0..I-1 gate, I..2I-1 up), h = silu(min(g, L))
  * clamp(u, -L, L) with L = 7 ([CARD] "Verification compute and EAGLE":
  experts keep the SwiGLU gate and its clamp), o = W_d(e) h, and
  y_t = sum_j w[t, j] o_{t, j} over j = 0..k-1 in that order.
  silu(z) = z / (1 + exp(-z)).
"""
from __future__ import annotations

import numpy as np

from . import formats, codebook, routing


def silu(z):
    with np.errstate(over="ignore"):
        return z / (1.0 + np.exp(-z))


def swiglu_clamp(g, u, limit: float = 7.0):
    return silu(np.minimum(g, limit)) * np.clip(u, -limit, limit)


def linear(x, w_deq):
    """x [T, K], w_deq [N, K] -> float64 [T, N]."""
    return np.asarray(x, dtype=np.float64) @ np.asarray(w_deq, dtype=np.float64).T


class ExpertBank:
    """Quantised expert weights of one MoE layer with per-expert dequantisation.

    fmt "mxfp4": gu_codes [E,2I,H/2], gu_scales [E,2I,H/32], dn_* likewise [E,H,...].
    fmt "nvfp4": as above with E4M3 scales per 16 and gu_ts / dn_ts [E].
    fmt "cb4":   per expert a dict from codebook.cb4_fit for gate_up and for down.
    """

    def __init__(self, fmt, E, H, I, **t):
        self.fmt, self.E, self.H, self.I = fmt, E, H, I
        self.t = t

    def gate_up(self, e):
        t = self.t
        if self.fmt == "mxfp4":
            return formats.mxfp4_dequantize(t["gu_codes"][e], t["gu_scales"][e])
        if self.fmt == "nvfp4":
            return formats.nvfp4_dequantize(t["gu_codes"][e], t["gu_scales"][e], t["gu_ts"][e])
        return None

    def down(self, e):
        t = self.t
        if self.fmt == "mxfp4":
            return formats.mxfp4_dequantize(t["dn_codes"][e], t["dn_scales"][e])
        if self.fmt == "nvfp4":
            return formats.nvfp4_dequantize(t["dn_codes"][e], t["dn_scales"][e], t["dn_ts"][e])
        return None

    def apply_gate_up(self, e, x):
        if self.fmt == "cb4":
            c = self.t["gu"][e]
            return codebook.cb4_matvec(x, c["idx"], c["cb_val"], c["row_ptr"], c["col"], c["val"])
        return x @ self.gate_up(e).T

    def apply_down(self, e, h):
        if self.fmt == "cb4":
            c = self.t["dn"][e]
            return codebook.cb4_matvec(h, c["idx"], c["cb_val"], c["row_ptr"], c["col"], c["val"])
        return h @ self.down(e).T


def moe_forward(x, ids, w, bank: ExpertBank, limit: float = 7.0, tokens=None):
    """Routed-expert MoE layer in float64.

    x [T, H]; ids int [T, k]; w float [T, k]. ``tokens`` optionally restricts the
    computation to a subset of token indices (rows of the result follow it).
    Returns y float64 [len(tokens), H].
    """
    x = np.asarray(x, dtype=np.float64)
    T, k = ids.shape
    tok = np.arange(T) if tokens is None else np.asarray(tokens)
    I = bank.I
    o = np.zeros((tok.size, k, bank.H), dtype=np.float64)
    sub_ids = ids[tok]
    for e in np.unique(sub_ids):
        ti, jj = np.nonzero(sub_ids == e)
        xe = x[tok[ti]]
        gu = bank.apply_gate_up(int(e), xe)
        h = swiglu_clamp(gu[:, :I], gu[:, I:], limit)
        o[ti, jj] = bank.apply_down(int(e), h)
    wsub = np.asarray(w, dtype=np.float64)[tok]
    y = np.zeros((tok.size, bank.H), dtype=np.float64)
    for j in range(k):
        y += wsub[:, j:j + 1] * o[:, j]
    return y


def moe_layer(x, wr, bias, k, bank: ExpertBank, limit: float = 7.0, tokens=None):
    """Router + experts: returns (y, ids, w, logits) in float64."""
    lg = routing.router_logits(x, wr, bias)
    ids = routing.topk(lg, k)
    w = routing.softmax_selected(lg, ids)
    return moe_forward(x, ids, w, bank, limit, tokens), ids, w, lg
