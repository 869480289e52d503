"""Pins of the oracle's CB4 (codebook + sparse outlier) format."""
import numpy as np

from oracle import codebook as C, formats as F


def _accounting(golden):
    return {r[0]: (float(r[1]), float(r[2])) for r in golden("xfp_accounting.txt")}


def test_page_storage_arithmetic(golden):
    acc = _accounting(golden)
    for n, key in ((2, "v2a_effective_bits_n2"), (4, "v2a_effective_bits_n4")):
        v, tol = acc[key]
        assert abs(C.bits_per_weight_v2a(n) - v) <= tol
    v, tol = acc["v2a_constant_overhead_bits"]
    assert abs(C.bits_per_weight_v2a(0) - v) <= tol
    v, _ = acc["v2a_library_bytes_l32_n4"]
    assert 32 * 2 ** 4 * 2 == v
    v, tol = acc["v2_outlier_bytes_per_weight_cap2"]
    assert abs(0.02 * (8 + 8 + 2) - v) <= tol
    for n, key in ((4, "lanes_per_group_n4"), (2, "lanes_per_group_n2")):
        assert 128 // (32 // n) == acc[key][0]
    assert C.bits_per_weight_cb4() == 6.0          # this workload: 4 + 16 * 16 / 128


def test_quantile_initialisation_hand_worked():
    g = np.arange(128, dtype=np.float64)[None]
    c0 = C.lloyd_codebooks(g, rounds=0)
    assert c0[0].tolist() == [8.0 * i + 4 for i in range(16)]


def test_lloyd_recovers_16_clusters():
    vals = np.linspace(-1, 1, 16)
    rng = np.random.default_rng(17)
    g = rng.permutation(np.repeat(vals, 8))[None]
    c = C.lloyd_codebooks(g, rounds=20)
    assert np.allclose(np.sort(c[0]), vals, rtol=0, atol=1e-15)


def _objective(g, c):
    return ((g[:, :, None] - c[:, None, :]) ** 2).min(axis=2).sum()


def test_lloyd_invariants():
    rng = np.random.default_rng(18)
    g = rng.standard_t(4, size=(40, 128)) * 0.014
    prev = None
    for r in range(0, 21):
        c = C.lloyd_codebooks(g, rounds=r)
        obj = _objective(g, c)
        if prev is not None:
            assert obj <= prev * (1 + 1e-12)
        prev = obj
    # round r's entries are the conditional means of round r-1's nearest-entry cells
    c19 = C.lloyd_codebooks(g, rounds=19)
    c20 = C.lloyd_codebooks(g, rounds=20)
    for i in range(g.shape[0]):
        a = np.argmin(np.abs(g[i][:, None] - c19[i][None, :]), axis=1)
        for j in range(16):
            if (a == j).any():
                assert abs(c20[i, j] - g[i][a == j].mean()) <= 1e-15
            else:
                assert c20[i, j] == c19[i, j]


def test_cb4_fit_structure_and_dense_plus_sparse():
    rng = np.random.default_rng(19)
    N, K = 6, 384
    w = (rng.standard_t(4, size=(N, K)) * 0.014).astype(np.float32)
    w[2, 7] = 0.9
    w[4, 300] = -0.5
    thr = 0.12
    fit = C.cb4_fit(w, thr)
    out = np.abs(w.astype(np.float64)) > thr
    assert fit["row_ptr"][-1] == out.sum()
    rows = np.repeat(np.arange(N), np.diff(fit["row_ptr"]))
    assert np.array_equal(np.stack([rows, fit["col"]], 1), np.argwhere(out))
    # final assignment is the nearest fp16 entry (brute force)
    a = F.unpack_nibbles(fit["idx"]).astype(int)
    bulk = np.where(out, 0.0, w.astype(np.float64))
    for r in range(N):
        for c in range(0, K, 37):
            ent = fit["cb_val"][r, c // 128]
            d = np.abs(bulk[r, c] - ent)
            assert a[r, c] == int(np.argmin(d))
    assert np.array_equal(F.round_to_f16(fit["cb_val"]), fit["cb_val"])
    dense = C.cb4_dense(fit["idx"], fit["cb_val"])
    sparse = C.cb4_sparse(fit["row_ptr"], fit["col"], fit["val"], N, K)
    x = rng.normal(size=(3, K))
    assert np.allclose(C.cb4_matvec(x, fit["idx"], fit["cb_val"], fit["row_ptr"], fit["col"], fit["val"]),
                       x @ (dense + sparse).T, rtol=1e-13, atol=1e-13)
    # at an outlier, dense + sparse reproduces w to fp16 rounding of the residual
    recon = dense + sparse
    assert np.all(np.abs(recon[out] - w[out]) <= np.abs(w[out]) * 2.0 ** -11 + 1e-7)
    # reconstruction error well below the weights' scale elsewhere
    err = np.linalg.norm((recon - w)[~out]) / np.linalg.norm(w[~out])
    assert err < 0.2


def test_cb4_nibble_lanes():
    """子字节打包 at N = 4: 8 indices per 32-bit word, 16 words per 128-group."""
    a = np.arange(128, dtype=np.uint8) % 16
    p = F.pack_nibbles(a[None])[0]
    words = p.view(np.uint32)
    assert words.size == 16
    assert int(words[0]) == 0x76543210
