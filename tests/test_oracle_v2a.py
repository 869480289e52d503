"""Pins of the V2a oracle (shared codebook library) to facts the page and the mathematics
fix: the bit accounting and library size the page states, exact reconstruction of values
the library represents, a library that reduces to per-channel codebooks when there are
as many rows as library entries, Lloyd invariants of LibFit, brute-force group choice on
a tiny case, single rounding of the reconstruction, and the packing of 2- and 4-bit codes."""
import itertools

import numpy as np
import pytest

from oracle import formats as F, v2a as V


def test_bit_accounting_and_library_size():
    # N + 37/128: the page prints about 2.31 and 4.31 (0.29 bits above N; partial pin, the
    # page's own formula is lost) and a 1 KB library for L = 32, N = 4
    assert V.bits_per_weight(2) == 2 + 37 / 128 and V.bits_per_weight(4) == 4 + 37 / 128
    assert abs(V.bits_per_weight(4) - 4.31) < 0.025 and abs(V.bits_per_weight(2) - 2.31) < 0.025
    assert V.library_bytes(4) == 1024
    # packing constraint: values per 32-bit word divide the 128-weight group only for N in {2, 4}
    assert [n for n in range(2, 7) if 128 % (32 // n) == 0 and 32 % n == 0] == [2, 4]


@pytest.mark.parametrize("n_bits", [2, 4])
def test_pack_round_trip(n_bits):
    rng = np.random.default_rng(3)
    c = rng.integers(0, 1 << n_bits, size=(5, 256)).astype(np.uint8)
    p = V.pack_codes(c, n_bits)
    assert p.shape == (5, 256 * n_bits // 8)
    assert np.array_equal(V.unpack_codes(p, n_bits, 256), c)
    if n_bits == 4:
        assert np.array_equal(p, F.pack_nibbles(c))          # the same nibble order as E2M1 codes
    else:
        assert p[0, 0] == c[0, 0] | (c[0, 1] << 2) | (c[0, 2] << 4) | (c[0, 3] << 6)


def test_reconstruction_is_one_rounding():
    mid = np.array([[0.0137]]); scale = np.array([[0.0419]])
    mid, scale = F.round_to_f16(mid), F.round_to_f16(scale)
    lib = F.round_to_f16(np.linspace(-1, 1, 16))[None]
    codes = np.arange(16, dtype=np.uint8)[None].repeat(8, axis=1)          # 128 weights of one group
    got = V.reconstruct(codes, np.zeros((1, 1), np.int64), mid, scale, lib)
    exact = mid[0, 0] + scale[0, 0] * lib[0, codes[0]]                     # exact in float64
    assert np.array_equal(got[0], exact.astype(np.float16).astype(np.float64))


def test_reconstruction_values_are_fp16():
    """Every reconstructed weight is an fp16 value (one rounding of mid + scale * entry)."""
    rng = np.random.default_rng(0)
    w = (rng.standard_t(4, size=(64, 256)) * 0.02).astype(np.float32)
    fit = V.v2a_fit(w, 4, threshold=1.0)
    wq = V.v2a_dense(fit, 256).astype(np.float32)
    assert np.array_equal(F.round_to_f16(wq.astype(np.float64)), wq.astype(np.float64))


def test_library_reduces_to_per_channel_codebooks_when_rows_equal_entries():
    """R = L rows: the start picks every row once, each row is its own cluster, and the
    library is exactly the set of per-channel codebooks (V2 with group scale and mid)."""
    rng = np.random.default_rng(1)
    z = rng.uniform(-1, 1, size=(V.LIB, 128)) * rng.uniform(0.2, 1.0, size=(V.LIB, 1))
    cbs = V.lloyd_rows(z, 16)
    lib = V.lib_fit(cbs)
    assert sorted(map(tuple, lib)) == sorted(map(tuple, cbs))


def test_libfit_lloyd_invariants():
    rng = np.random.default_rng(2)
    cbs = np.sort(rng.normal(size=(400, 4)) * rng.uniform(0.1, 1, size=(400, 1)), axis=1)
    trace = []
    lib = V.lib_fit(cbs, L=8, trace=trace)
    assert all(b <= a + 1e-12 for a, b in zip(trace, trace[1:]))          # the objective never rises
    a, d = V.library_assign(cbs, lib)
    assert np.array_equal(a, np.argmin(d, axis=1))                        # assignment = nearest
    lib2 = lib.copy()
    for l in range(8):                                                     # fixed point: centroid = member mean
        if (a == l).any():
            lib2[l] = cbs[a == l].mean(axis=0)
    np.testing.assert_allclose(lib2, lib, rtol=0, atol=1e-12)


def test_group_choice_brute_force_tiny():
    rng = np.random.default_rng(4)
    lib16 = F.round_to_f16(np.sort(rng.uniform(-1, 1, size=(3, 4)), axis=1))
    z = rng.uniform(-1, 1, size=(2, 256))
    li, codes = V.group_choice(z, lib16)
    for r, g in itertools.product(range(2), range(2)):
        zz = z[r, g * 128:(g + 1) * 128]
        errs = [sum(min((v - e) ** 2 for e in lib16[l]) for v in zz) for l in range(3)]
        assert li[r, g] == int(np.argmin(errs))
        for i, v in enumerate(zz):
            assert codes[r, g * 128 + i] == int(np.argmin([abs(v - e) for e in lib16[li[r, g]]]))


@pytest.mark.parametrize("n_bits", [2, 4])
def test_dense_plus_sparse_is_the_materialised_matrix(n_bits):
    rng = np.random.default_rng(5)
    w = (rng.standard_t(4, size=(48, 256)) * 0.02).astype(np.float32)
    w[3, 17] = 0.9; w[40, 200] = -0.7                        # planted outliers
    fit = V.v2a_fit(w, n_bits, threshold=6 * 0.02)
    assert int(fit["row_ptr"][-1]) >= 2
    W = V.v2a_matrix(fit, 256)
    # outlier positions come back to fp16 rounding of the residual
    assert abs(W[3, 17] - 0.9) < 1e-3 and abs(W[40, 200] + 0.7) < 1e-3
    err = np.linalg.norm(W - w) / np.linalg.norm(w)
    assert err < (0.12 if n_bits == 4 else 0.35)              # 4-bit is finer than 2-bit
    assert np.all(fit["lib_idx"] < V.LIB)
