"""Oracle: the 4-bit codebook-plus-outlier format (CB4).

TEST INFRASTRUCTURE ONLY (see ``oracle/__init__``).

Follows [XFP]:
* 离群值提取 (outlier extraction): weights farther than a threshold from the
  mean mu go to a sparse fp16 term; their place in the bulk matrix is
  back-filled with mu before any codebook is fitted.
* Lloyd 迭代: a scalar k-means (Lloyd-Max) codebook of 2^N entries initialised
  at the CDF-uniform quantiles (equal probability mass per initial entry), then
  alternating nearest-entry assignment and conditional-mean update, 20 rounds
  as the MoE setting uses.
* V2 / SqueezeLLM-style dense + sparse decomposition: W = W_codebook + W_outlier,
  the forward pass being the dense codebook term plus the sparse term.
* 子字节打包: N = 4 packs 8 indices per 32-bit word; a 128-weight group spans
  16 lanes of such words (LANES_PER_GROUP = 128 / 8).

Readings where the pages are silent or differ from the workload:
* The workload fits one 16-entry fp16 codebook per 128-weight group of a row
  (not per channel, not a shared library), with the threshold |w - mu| > 6 sigma
  for the nominal sigma = 0.02 and mu = 0, and stores outliers in CSR per
  matrix instead of int64 (row, col) triples.
* The (i + 0.5)/16 quantile of the 128 sorted group values is the order
  statistic at index 8 i + 4.
* Assignment ties go to the lower index; an empty cluster keeps its entry; the
  conditional mean sums members in ascending position order in float64.
* After the last round the entries are rounded to fp16 and every weight is
  assigned once more to the nearest fp16 entry; an outlier stores the fp16
  residual w - entry(idx) at its position, so dense + sparse ~= w.
"""
from __future__ import annotations

import numpy as np

from .formats import round_to_f16, pack_nibbles, unpack_nibbles

GROUP = 128
ENTRIES = 16
LLOYD_ROUNDS = 20


def _nearest(g, c):
    """g [..., 128], c [..., 16] -> index of the nearest entry (first on ties)."""
    d = np.abs(g[..., :, None] - c[..., None, :])
    return np.argmin(d, axis=-1)


def lloyd_codebooks(groups, rounds: int = LLOYD_ROUNDS):
    """groups: float64 [G, 128] -> float64 entries [G, 16] after ``rounds`` Lloyd rounds."""
    g = np.asarray(groups, dtype=np.float64)
    srt = np.sort(g, axis=-1)
    q_idx = (np.arange(ENTRIES) * 2 + 1) * GROUP // (2 * ENTRIES)   # floor((i + 0.5) / 16 * 128)
    c = srt[:, q_idx].copy()
    zero = np.zeros(g.shape[:-1] + (1,), dtype=np.float64)
    for _ in range(rounds):
        a = _nearest(g, c)
        for j in range(ENTRIES):
            member = a == j
            vals = np.where(member, g, 0.0)
            s = np.cumsum(np.concatenate([zero, vals], axis=-1), axis=-1)[:, -1]   # ascending order
            n = member.sum(axis=-1)
            c[:, j] = np.where(n > 0, s / np.maximum(n, 1), c[:, j])
    return c


def cb4_fit(w, threshold: float, mu: float = 0.0, rounds: int = LLOYD_ROUNDS):
    """Fit CB4 to one matrix.

    w: float32 [N, K], K % 128 == 0. Returns a dict with
      idx      uint8 [N, K/2]  (packed 4-bit indices, even position in the low nibble)
      cb       uint16 [N, K/128, 16]  fp16 bits of the entries
      cb_val   float64 [N, K/128, 16]  the same entries as values
      row_ptr  int32 [N+1], col int32 [nnz], val float64 [nnz] (fp16 values)
    """
    w = np.asarray(w, dtype=np.float32)
    N, K = w.shape
    assert K % GROUP == 0
    w64 = w.astype(np.float64)
    out_mask = np.abs(w64 - mu) > threshold
    bulk = np.where(out_mask, mu, w64)
    groups = bulk.reshape(N * (K // GROUP), GROUP)
    c = lloyd_codebooks(groups, rounds)
    c16 = round_to_f16(c)
    a = _nearest(groups, c16).astype(np.uint8)
    idx = pack_nibbles(a.reshape(N, K))
    c16r = c16.reshape(N, K // GROUP, ENTRIES)
    rows, cols = np.nonzero(out_mask)
    dense_at = c16r[rows, cols // GROUP, a.reshape(N, K)[rows, cols]]
    val = round_to_f16(w64[rows, cols] - dense_at)
    row_ptr = np.zeros(N + 1, dtype=np.int32)
    np.add.at(row_ptr, rows + 1, 1)
    row_ptr = np.cumsum(row_ptr).astype(np.int32)
    return dict(idx=idx, cb=c16r.astype(np.float16).view(np.uint16), cb_val=c16r,
                row_ptr=row_ptr, col=cols.astype(np.int32), val=val)


def cb4_dense(idx, cb_val):
    """Dense codebook term: W_cb[r, c] = entry(r, c // 128, idx[r, c]); float64."""
    a = unpack_nibbles(idx).astype(np.int64)
    N, K = a.shape
    grp = np.broadcast_to(np.arange(K) // GROUP, (N, K))
    return cb_val[np.arange(N)[:, None], grp, a]


def cb4_sparse(row_ptr, col, val, n: int, k: int):
    """Sparse outlier term as a dense float64 [n, k] matrix (for small checks)."""
    out = np.zeros((n, k), dtype=np.float64)
    rows = np.repeat(np.arange(n), np.diff(row_ptr))
    out[rows, col] = val
    return out


def cb4_matvec(x, idx, cb_val, row_ptr, col, val):
    """y = (W_cb + W_out) x^T for x [T, K] float64 -> [T, N]: dense term plus sparse term."""
    x = np.asarray(x, dtype=np.float64)
    dense = cb4_dense(idx, cb_val)
    y = x @ dense.T
    n = dense.shape[0]
    rows = np.repeat(np.arange(n), np.diff(row_ptr))
    contrib = x[:, col] * val[None, :]          # [T, nnz]
    ys = np.zeros_like(y)
    np.add.at(ys.T, rows, contrib.T)
    return y + ys


def bits_per_weight_v2a(n_bits: int, lib_index_bits: int = 5, scale_bits: int = 16,
                        mid_bits: int = 16, group: int = GROUP) -> float:
    """[XFP] V2a: effective bits = N + (library index + scale + mid-point bits) / 128."""
    return n_bits + (lib_index_bits + scale_bits + mid_bits) / group


def bits_per_weight_cb4(group: int = GROUP, entries: int = ENTRIES, entry_bits: int = 16) -> float:
    """This workload's CB4: 4-bit index + a 16-entry fp16 codebook per 128 weights."""
    return 4 + entries * entry_bits / group
