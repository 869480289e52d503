"""Oracle: router logits, top-k with softmax gate weights, and the token permutation.

TEST INFRASTRUCTURE ONLY (see ``oracle/__init__``).

[GATE] "A file is a census; a decode step is a sample": each token reads the
trunk plus the top-k of E experts (8 of 288, 8 of 256). The workload's
router is a top-8 softmax router with an optional per-expert logit bias.

Readings: logits = x . W_r^T + bias; the k largest logits are
selected, ties going to the lower expert index, in descending-logit order;
gate weights are the softmax over the k selected logits (identical to the
full softmax renormalised over them). The permutation is a stable sort of
the pairs p = t k + j by expert: perm[slot] = p, inv[p] = slot, with
counts[e] and offsets = exclusive scan of counts (E + 1 entries).
"""
from __future__ import annotations

import numpy as np


def router_logits(x, wr, bias=None):
    """x [T, H], wr [E, H] -> float64 [T, E]."""
    lg = np.asarray(x, dtype=np.float64) @ np.asarray(wr, dtype=np.float64).T
    if bias is not None:
        lg = lg + np.asarray(bias, dtype=np.float64)[None, :]
    return lg


def topk(logits, k: int):
    """-> ids int32 [T, k] (descending logit, ties to the lower expert)."""
    lg = np.asarray(logits)
    T, E = lg.shape
    ids = np.empty((T, k), dtype=np.int32)
    eidx = np.arange(E)
    for t in range(T):
        order = np.lexsort((eidx, -lg[t].astype(np.float64)))
        ids[t] = order[:k]
    return ids


def softmax_selected(logits, ids):
    """Softmax over the selected logits of each token, float64 [T, k]."""
    lg = np.asarray(logits, dtype=np.float64)
    sel = np.take_along_axis(lg, ids.astype(np.int64), axis=1)
    z = np.exp(sel - sel.max(axis=1, keepdims=True))
    return z / z.sum(axis=1, keepdims=True)


def permutation(ids, num_experts: int):
    """Stable grouping of the (token, slot) pairs by expert.

    Returns counts int32 [E], offsets int32 [E+1], perm int32 [T*k], inv int32 [T*k].
    """
    flat = np.asarray(ids, dtype=np.int64).reshape(-1)
    counts = np.bincount(flat, minlength=num_experts).astype(np.int32)
    offsets = np.zeros(num_experts + 1, dtype=np.int32)
    offsets[1:] = np.cumsum(counts)
    perm = np.argsort(flat, kind="stable").astype(np.int32)
    inv = np.empty_like(perm)
    inv[perm] = np.arange(perm.size, dtype=np.int32)
    return counts, offsets, perm, inv


def near_ties(logits, k: int, rel: float = 1e-4):
    """Tokens whose k-th and (k+1)-th largest logits are within rel * max(1, |l|):
    for them more than one top-k set is a correct selection."""
    lg = np.sort(np.asarray(logits, dtype=np.float64), axis=1)[:, ::-1]
    if k >= lg.shape[1]:
        return np.zeros(lg.shape[0], dtype=bool)
    a, b = lg[:, k - 1], lg[:, k]
    return (a - b) <= rel * np.maximum(1.0, np.abs(a))
