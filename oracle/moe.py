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

from . import formats, codebook, routing, v2a


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


class LazyExpertBank:
    """Expert bank that quantises an expert the first time it is used.

    ``draw(which, e)`` returns the float32 weights of expert e (which = "gu" -> [2I, H],
    "dn" -> [H, I]); they are quantised here with this package's own formats (MXFP4,
    NVFP4 with one tensor scale per expert matrix, CB4 or V2a (``v2a_bits`` per code,
    one library per expert matrix) with ``cb4_threshold`` as the absolute outlier
    threshold around mu = 0, or "mixed": MXFP4 except the ``bf16_experts``, which are
    rounded to bf16) and dequantised exactly in float64.
    """

    def __init__(self, fmt, E, H, I, draw, cb4_threshold=None, v2a_bits=4, bf16_experts=()):
        self.fmt, self.E, self.H, self.I = fmt, E, H, I
        self.draw = draw
        self.cb4_threshold = cb4_threshold
        self.v2a_bits = v2a_bits
        self.bf16_experts = set(bf16_experts)
        self._cache = {}

    def packed(self, which, e):
        key = (which, e)
        if key not in self._cache:
            w = self.draw(which, e)
            if self.fmt == "mixed" and e in self.bf16_experts:
                self._cache[key] = ("bf16", formats.round_to_bf16(w.astype(np.float64)))
            elif self.fmt == "cb4":
                self._cache[key] = codebook.cb4_fit(w, self.cb4_threshold)
            elif self.fmt == "v2a":
                self._cache[key] = v2a.v2a_fit(w, self.v2a_bits, self.cb4_threshold)
            elif self.fmt in ("mxfp4", "mixed"):
                self._cache[key] = formats.mxfp4_quantize(w) + (None,)
            else:
                c, s, t = formats.nvfp4_quantize(w[None])
                self._cache[key] = (c[0], s[0], t[0])
        return self._cache[key]

    def dequant(self, which, e):
        if self.fmt == "mixed" and e in self.bf16_experts:
            return self.packed(which, e)[1]
        if self.fmt == "v2a":
            return v2a.v2a_matrix(self.packed(which, e), self.H if which == "gu" else self.I)
        if self.fmt == "cb4":
            fit = self.packed(which, e)
            n, k2 = fit["idx"].shape
            return (codebook.cb4_dense(fit["idx"], fit["cb_val"])
                    + codebook.cb4_sparse(fit["row_ptr"], fit["col"], fit["val"], n, 2 * k2))
        c, s, t = self.packed(which, e)
        if self.fmt in ("mxfp4", "mixed"):
            return formats.mxfp4_dequantize(c, s)
        return formats.nvfp4_dequantize(c, s, t)

    def apply_gate_up(self, e, x):
        return np.asarray(x, dtype=np.float64) @ self.dequant("gu", e).T

    def apply_down(self, e, h):
        return np.asarray(h, dtype=np.float64) @ self.dequant("dn", e).T

    def preload(self, which, e, packed):
        """Install an expert's quantised form made earlier by ``packed`` (e.g. in another
        process) so that later calls skip quantising it."""
        self._cache[(which, e)] = packed

    def drop(self, e):
        """Forget the quantised copies of expert e (bounds memory on full-size layers)."""
        self._cache.pop(("gu", e), None)
        self._cache.pop(("dn", e), None)


def expert_outputs(bank, e, x_rows, limit: float = 7.0):
    """One expert on the rows routed to it: o = W_d(e) (silu(min(g, L)) clamp(u, -L, L))
    with [g; u] = W_gu(e) x, float64 [n, H].  The per-expert body of ``moe_forward``."""
    gu = bank.apply_gate_up(int(e), np.asarray(x_rows, dtype=np.float64))
    h = swiglu_clamp(gu[:, :bank.I], gu[:, bank.I:], limit)
    return bank.apply_down(int(e), h)


def moe_forward(x, ids, w, bank: ExpertBank, limit: float = 7.0, tokens=None):
    """Routed-expert MoE layer in float64.

    x [T, H]; ids int [T, k]; w float [T, k]. ``tokens`` optionally restricts the
    computation to a subset of token indices (rows of the result follow it).
    Returns y float64 [len(tokens), H].
    """
    x = np.asarray(x, dtype=np.float64)
    T, k = ids.shape
    tok = np.arange(T) if tokens is None else np.asarray(tokens)
    o = np.zeros((tok.size, k, bank.H), dtype=np.float64)
    sub_ids = ids[tok]
    for e in np.unique(sub_ids):
        ti, jj = np.nonzero(sub_ids == e)
        o[ti, jj] = expert_outputs(bank, e, x[tok[ti]], limit)
    return combine_slots(np.asarray(w, dtype=np.float64)[tok], o)


def combine_slots(w, o):
    """y_t = sum_{j = 0..k-1} w[t, j] o[t, j] accumulated in j order: w [n, k], o [n, k, H]."""
    w = np.asarray(w, dtype=np.float64)
    y = np.zeros((o.shape[0], o.shape[2]), dtype=np.float64)
    for j in range(o.shape[1]):
        y += w[:, j:j + 1] * o[:, j]
    return y


def moe_layer(x, wr, bias, k, bank: ExpertBank, limit: float = 7.0, tokens=None):
    """Router + experts: returns (y, ids, w, logits) in float64."""
    lg = routing.router_logits(x, wr, bias)
    ids = routing.topk(lg, k)
    w = routing.softmax_selected(lg, ids)
    return moe_forward(x, ids, w, bank, limit, tokens), ids, w, lg
