"""Pins of the oracle's linear layer and MoE layer: brute force on tiny shapes,
closed forms of the clamped SwiGLU, and reductions to a textbook FFN."""
import math

import numpy as np

from oracle import formats as F, moe as M, routing as R


def test_linear_brute_force_enumerated_codes():
    """All 16 codes x a few scales against hand-style sums (K = 32, N <= 4, T <= 3)."""
    rng = np.random.default_rng(11)
    N, K, T = 4, 32, 3
    codes = np.tile(np.arange(16, dtype=np.uint8), (N, 2))
    codes = rng.permuted(codes, axis=1)
    scales = np.array([[120], [127], [130], [1]], dtype=np.uint8)
    packed = F.pack_nibbles(codes)
    w = F.mxfp4_dequantize(packed, scales)
    x = rng.normal(size=(T, K))
    y = M.linear(x, w)
    e2m1 = {0: 0.0, 1: 0.5, 2: 1.0, 3: 1.5, 4: 2.0, 5: 3.0, 6: 4.0, 7: 6.0}
    for t in range(T):
        for n in range(N):
            s = 0.0
            for kk in range(K):
                c = int(codes[n, kk])
                v = e2m1[c & 7] * (-1 if c & 8 else 1) * 2.0 ** (int(scales[n, 0]) - 127)
                s += v * x[t, kk]
            assert abs(y[t, n] - s) <= 1e-12 * max(1.0, abs(s))


def test_nvfp4_linear_brute_force():
    rng = np.random.default_rng(12)
    w = rng.standard_t(4, size=(3, 32)).astype(np.float32) * 0.02
    codes, scales, ts = F.nvfp4_quantize(w)
    deq = F.nvfp4_dequantize(codes, scales, ts)
    c = F.unpack_nibbles(codes)
    for n in range(3):
        for kk in range(32):
            want = float(F.e2m1_value(c[n, kk])) * float(F.e4m3_value(scales[n, kk // 16])) * float(ts)
            assert deq[n, kk] == want


def test_swiglu_clamp_closed_forms():
    L = 7.0
    silu7 = 7.0 / (1.0 + math.exp(-7.0))
    g = np.array([7.0, 50.0, 1e6, 0.0, -3.0])
    u = np.array([1.0, 1.0, 100.0, 5.0, -100.0])
    h = M.swiglu_clamp(g, u, L)
    assert h[0] == silu7 and h[1] == silu7 and h[2] == silu7 * 7.0
    assert h[3] == 0.0
    assert abs(h[4] - (-3.0 / (1 + math.exp(3.0))) * -7.0) < 1e-15
    assert np.all(np.abs(M.swiglu_clamp(np.linspace(-50, 50, 1001), np.linspace(-50, 50, 1001), L))
                  <= silu7 * 7.0 + 1e-12)


class _DenseBank(M.ExpertBank):
    def __init__(self, gu, dn):
        super().__init__("dense", gu.shape[0], dn.shape[1], dn.shape[2])
        self.gu, self.dn = gu, dn

    def apply_gate_up(self, e, x):
        return x @ self.gu[e].T

    def apply_down(self, e, h):
        return h @ self.dn[e].T


def _ffn(x, gu, dn, I, L=7.0):
    g = x @ gu[:I].T
    u = x @ gu[I:].T
    return (M.silu(np.minimum(g, L)) * np.clip(u, -L, L)) @ dn.T


def test_moe_single_expert_is_dense_ffn():
    rng = np.random.default_rng(13)
    H, I, T = 24, 10, 5
    gu = rng.normal(0, 0.5, (1, 2 * I, H))
    dn = rng.normal(0, 0.5, (1, H, I))
    x = rng.normal(size=(T, H))
    ids = np.zeros((T, 1), np.int32)
    w = np.ones((T, 1))
    y = M.moe_forward(x, ids, w, _DenseBank(gu, dn))
    assert np.allclose(y, _ffn(x, gu[0], dn[0], I), rtol=1e-13, atol=1e-13)


def test_moe_identical_experts_invariant_to_routing():
    rng = np.random.default_rng(14)
    E, H, I, T, k = 6, 16, 8, 7, 3
    gu1 = rng.normal(0, 0.5, (2 * I, H))
    dn1 = rng.normal(0, 0.5, (H, I))
    bank = _DenseBank(np.repeat(gu1[None], E, 0), np.repeat(dn1[None], E, 0))
    x = rng.normal(size=(T, H))
    wr = rng.normal(size=(E, H))
    y, ids, w, _ = M.moe_layer(x, wr, None, k, bank)
    assert np.allclose(y, _ffn(x, gu1, dn1, I), rtol=1e-12, atol=1e-12)


def test_moe_brute_force_loops():
    rng = np.random.default_rng(15)
    E, H, I, T, k = 5, 6, 4, 4, 2
    gu = rng.normal(0, 1, (E, 2 * I, H))
    dn = rng.normal(0, 1, (E, H, I))
    x = rng.normal(size=(T, H))
    wr = rng.normal(size=(E, H))
    y, ids, w, lg = M.moe_layer(x, wr, None, k, _DenseBank(gu, dn))
    for t in range(T):
        order = sorted(range(E), key=lambda e: (-sum(x[t, h] * wr[e, h] for h in range(H)), e))[:k]
        sel = [sum(x[t, h] * wr[e, h] for h in range(H)) for e in order]
        z = [math.exp(s - max(sel)) for s in sel]
        ws = [v / sum(z) for v in z]
        acc = [0.0] * H
        for j, e in enumerate(order):
            hh = []
            for i in range(I):
                g = sum(gu[e, i, c] * x[t, c] for c in range(H))
                u = sum(gu[e, I + i, c] * x[t, c] for c in range(H))
                gg = min(g, 7.0)
                hh.append(gg / (1 + math.exp(-gg)) * max(-7.0, min(7.0, u)))
            for n in range(H):
                acc[n] += ws[j] * sum(dn[e, n, i] * hh[i] for i in range(I))
        assert np.allclose(y[t], acc, rtol=1e-12, atol=1e-12)


def test_moe_token_subset_matches_full():
    rng = np.random.default_rng(16)
    E, H, I, T, k = 8, 12, 6, 9, 3
    bank = _DenseBank(rng.normal(size=(E, 2 * I, H)), rng.normal(size=(E, H, I)))
    x = rng.normal(size=(T, H))
    lg = rng.normal(size=(T, E))
    ids = R.topk(lg, k)
    w = R.softmax_selected(lg, ids)
    full = M.moe_forward(x, ids, w, bank)
    sub = M.moe_forward(x, ids, w, bank, tokens=[7, 2, 5])
    assert np.allclose(sub, full[[7, 2, 5]], rtol=1e-13, atol=1e-13)


def test_mixed_bank_reduces_to_its_parts():
    """A mixed-format bank ("The gate that missed by 0.0202 pp", "A fused tensor with two
    dtypes in it") is, expert by expert, the MXFP4 bank for the quantised experts and the
    bf16-rounded weights for the excluded ones: a single excluded expert gives the textbook
    FFN on bf16 weights, and no excluded expert gives the MXFP4 bank."""
    rng = np.random.default_rng(17)
    E, H, I, T = 3, 64, 32, 4
    gu = rng.normal(0, 0.05, (E, 2 * I, H)).astype(np.float32)
    dn = rng.normal(0, 0.05, (E, H, I)).astype(np.float32)
    draw = lambda which, e: gu[e] if which == "gu" else dn[e]   # noqa: E731
    x = rng.normal(size=(T, H))
    mixed = M.LazyExpertBank("mixed", E, H, I, draw, bf16_experts=(1,))
    mx = M.LazyExpertBank("mxfp4", E, H, I, draw)
    ids = np.full((T, 1), 1, np.int32)
    w = np.ones((T, 1))
    y_bf16 = M.moe_forward(x, ids, w, mixed)
    ref = _ffn(x, F.round_to_bf16(gu[1].astype(np.float64)), F.round_to_bf16(dn[1].astype(np.float64)), I)
    assert np.allclose(y_bf16, ref, rtol=1e-13, atol=1e-13)
    for e in (0, 2):
        ids = np.full((T, 1), e, np.int32)
        assert np.array_equal(M.moe_forward(x, ids, w, mixed), M.moe_forward(x, ids, w, mx))
    # the bf16 expert differs from its MXFP4 quantisation (the formats really differ)
    ids = np.full((T, 1), 1, np.int32)
    assert not np.allclose(M.moe_forward(x, ids, w, mixed), M.moe_forward(x, ids, w, mx), rtol=1e-3)
