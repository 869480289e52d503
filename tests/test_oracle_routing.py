"""Pins of the oracle's router: a hand-worked example, brute force, invariants."""
import numpy as np

from oracle import routing as R


def _rows(golden, tag):
    return [list(map(float, r[1:])) for r in golden("routing_tiny.txt") if r[0] == tag]


def test_routing_worked_example(golden):
    lg = np.array(_rows(golden, "logits"))
    ids = R.topk(lg, 2)
    assert ids.tolist() == [[int(v) for v in r] for r in _rows(golden, "ids")]
    counts, offsets, perm, inv = R.permutation(ids, 4)
    assert counts.tolist() == [int(v) for v in _rows(golden, "counts")[0]]
    assert offsets.tolist() == [int(v) for v in _rows(golden, "offsets")[0]]
    assert perm.tolist() == [int(v) for v in _rows(golden, "perm")[0]]
    assert inv.tolist() == [int(v) for v in _rows(golden, "inv")[0]]


def test_topk_brute_force_with_ties():
    rng = np.random.default_rng(7)
    for _ in range(30):
        T, E = 5, int(rng.integers(2, 40))
        k = int(rng.integers(1, E + 1))
        lg = rng.integers(-3, 4, size=(T, E)).astype(np.float32)   # many exact ties
        ids = R.topk(lg, k)
        for t in range(T):
            want = sorted(range(E), key=lambda e: (-float(lg[t, e]), e))[:k]
            assert ids[t].tolist() == want


def test_softmax_selected_equals_renormalised_full_softmax():
    rng = np.random.default_rng(8)
    lg = rng.normal(0, 3, (6, 20))
    ids = R.topk(lg, 5)
    w = R.softmax_selected(lg, ids)
    full = np.exp(lg - lg.max(1, keepdims=True))
    full /= full.sum(1, keepdims=True)
    sel = np.take_along_axis(full, ids.astype(int), 1)
    assert np.allclose(w, sel / sel.sum(1, keepdims=True), rtol=1e-14, atol=0)
    assert np.allclose(w.sum(1), 1.0, rtol=1e-14)
    assert np.all(np.diff(w, axis=1) <= 0)           # descending logit -> descending weight


def test_permutation_invariants():
    rng = np.random.default_rng(9)
    for E, T, k in ((7, 13, 3), (64, 16, 8), (256, 64, 8), (5, 1, 5)):
        lg = rng.normal(size=(T, E))
        ids = R.topk(lg, k)
        counts, offsets, perm, inv = R.permutation(ids, E)
        assert counts.sum() == T * k and offsets[0] == 0 and offsets[-1] == T * k
        assert np.array_equal(np.sort(perm), np.arange(T * k))          # bijection
        assert np.array_equal(inv[perm], np.arange(T * k))              # inv o perm = id
        flat = ids.reshape(-1)
        for e in range(E):
            seg = perm[offsets[e]:offsets[e + 1]]
            assert np.all(flat[seg] == e)
            assert np.all(np.diff(seg) > 0)                              # stable


def test_logits_brute_force():
    rng = np.random.default_rng(10)
    x = rng.normal(size=(3, 5))
    wr = rng.normal(size=(4, 5)).astype(np.float32)
    b = rng.normal(size=4).astype(np.float32)
    lg = R.router_logits(x, wr, b)
    for t in range(3):
        for e in range(4):
            s = sum(float(x[t, h]) * float(wr[e, h]) for h in range(5)) + float(b[e])
            assert abs(lg[t, e] - s) < 1e-12


def test_near_ties():
    lg = np.array([[1.0, 1.0, 0.0], [2.0, 1.0, 0.0]])
    assert R.near_ties(lg, 1).tolist() == [True, False]
