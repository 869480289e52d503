"""Oracle: the V2a shared codebook library (codebook-plus-outlier weights whose
codebooks come from one small library per matrix).

TEST INFRASTRUCTURE ONLY (see ``oracle/__init__``).

Follows [XFP] section V2a：共享码本库 and the sections it builds on:
* one library of L = 32 fp16 codebooks of 2^N entries per layer matrix, N in {2, 4}
  (128 must be a multiple of the values per 32-bit word: 16 for N = 2, 8 for N = 4);
* per 128-weight group a 5-bit library index, a 16-bit scale and a 16-bit mid-point,
  so the effective width is N + (5 + 16 + 16) / 128 = N + 37/128 bits per weight
  (outlier residuals not counted);
* LibFit: per-channel Lloyd codebooks first (the V2 way), then Lloyd iterations over
  the codebooks themselves condense them into the L library entries ("a codebook of
  codebooks"); 20 rounds as the MoE setting uses (XFP_MOE_LLOYD_ITERS = 20);
* the outliers leave the bulk first and are kept as a sparse fp16 residual term
  (离群值提取), and the codebooks start at CDF-uniform quantiles (Lloyd 迭代).

Readings where the page is silent (its reconstruction formula is lost):
* group g of a row has mid_g = fp16((max + min) / 2) and scale_g = fp16((max - min) / 2)
  of its bulk values (outliers back-filled with mu); the normalised values are
  z = (w - mid_g) / scale_g, or 0 when scale_g = 0;
* a weight is reconstructed as fp16(mid_g + scale_g * lib[l_g][c]) rounded once
  (nearest, ties to even);
* per-channel codebooks: Lloyd over the row's K normalised values with 2^N entries,
  started at the sorted values at positions floor((2i + 1) K / 2^(N+1)), ties to the
  lower entry, member means summed in ascending position in float64, an empty entry
  kept;
* library: Lloyd over the R per-channel codebooks as vectors of 2^N entries, squared
  Euclidean distance summed in entry order, ties to the lower library index, member
  means summed in ascending row order, an empty entry kept; started at the codebooks
  of rank floor((2i + 1) R / (2 L)) when the rows are ordered by codebook span (largest
  entry minus smallest, ties by row); rounded to fp16 after the last round; R >= L;
* a group takes the library codebook with the least sum over its 128 positions (in
  order) of the squared distance to the nearest entry, ties to the lower index; each
  weight takes its nearest entry of that codebook (ties to the lower entry);
* the library index is stored in one byte; codes are packed low bits first (N = 4:
  two per byte, even position in the low nibble; N = 2: four per byte, position j at
  bits 2 (j % 4)); outliers: CSR per matrix with value fp16(w - reconstruction).
"""
from __future__ import annotations

import numpy as np

from .formats import round_to_f16

GROUP = 128
LIB = 32
ROUNDS = 20


def lloyd_rows(values, n: int, rounds: int = ROUNDS):
    """Scalar Lloyd per row: values float64 [R, K] -> entries float64 [R, n]."""
    v = np.asarray(values, dtype=np.float64)
    R, K = v.shape
    srt = np.sort(v, axis=-1)
    q = (2 * np.arange(n) + 1) * K // (2 * n)
    c = srt[:, q].copy()
    for _ in range(rounds):
        a = np.argmin(np.abs(v[:, :, None] - c[:, None, :]), axis=-1)
        for j in range(n):
            m = a == j
            s = np.cumsum(np.where(m, v, 0.0), axis=-1)[:, -1]
            cnt = m.sum(axis=-1)
            c[:, j] = np.where(cnt > 0, s / np.maximum(cnt, 1), c[:, j])
    return c


def library_init(cbs, L: int = LIB):
    """Starting library: the codebooks of rank floor((2i + 1) R / (2 L)) by span."""
    R = cbs.shape[0]
    span = cbs.max(axis=1) - cbs.min(axis=1)
    order = np.lexsort((np.arange(R), span))
    return cbs[order[(2 * np.arange(L) + 1) * R // (2 * L)]].copy()


def library_assign(cbs, lib):
    """Nearest library codebook of each row codebook (squared distance, ties lower)."""
    d = np.zeros((cbs.shape[0], lib.shape[0]))
    for j in range(cbs.shape[1]):
        d += (cbs[:, None, j] - lib[None, :, j]) ** 2
    return np.argmin(d, axis=1), d


def lib_fit(cbs, L: int = LIB, rounds: int = ROUNDS, trace=None):
    """LibFit: Lloyd over the per-channel codebooks [R, n] -> library float64 [L, n]
    (before the fp16 rounding).  ``trace`` (a list) receives the objective per round."""
    cbs = np.asarray(cbs, dtype=np.float64)
    R, n = cbs.shape
    assert R >= L
    lib = library_init(cbs, L)
    for _ in range(rounds):
        a, d = library_assign(cbs, lib)
        if trace is not None:
            trace.append(float(d[np.arange(R), a].sum()))
        for l in range(L):
            m = a == l
            if m.any():
                lib[l] = np.cumsum(cbs[m], axis=0)[-1] / m.sum()
    return lib


def group_stats(bulk):
    """bulk float64 [R, K] -> (mid, scale) float64 [R, K/128], both fp16 values."""
    R, K = bulk.shape
    g = bulk.reshape(R, K // GROUP, GROUP)
    lo, hi = g.min(axis=-1), g.max(axis=-1)
    return round_to_f16((hi + lo) / 2), round_to_f16((hi - lo) / 2)


def normalise(bulk, mid, scale):
    R, K = bulk.shape
    g = bulk.reshape(R, K // GROUP, GROUP)
    with np.errstate(divide="ignore", invalid="ignore"):
        z = np.where(scale[..., None] > 0, (g - mid[..., None]) / scale[..., None], 0.0)
    return z.reshape(R, K)


def group_choice(z, lib16):
    """Library index per group and code per weight: z [R, K], lib16 [L, n]."""
    R, K = z.shape
    g = z.reshape(R, K // GROUP, GROUP)
    L, n = lib16.shape
    err = np.zeros((R, K // GROUP, L))
    for l in range(L):
        d = np.min((g[..., None] - lib16[l][None, None, None, :]) ** 2, axis=-1)   # [R, G, 128]
        err[..., l] = np.cumsum(d, axis=-1)[..., -1]
    li = np.argmin(err, axis=-1)
    ent = lib16[li]                                                   # [R, G, n]
    codes = np.argmin(np.abs(g[..., None] - ent[:, :, None, :]), axis=-1)
    return li.astype(np.uint8), codes.reshape(R, K).astype(np.uint8)


def pack_codes(codes, n_bits: int):
    """codes uint8 [R, K] -> bytes [R, K * n_bits / 8], low bits first."""
    c = np.asarray(codes, dtype=np.uint8)
    per = 8 // n_bits
    R, K = c.shape
    c = c.reshape(R, K // per, per).astype(np.uint16)
    out = np.zeros((R, K // per), dtype=np.uint16)
    for j in range(per):
        out |= c[..., j] << (n_bits * j)
    return out.astype(np.uint8)


def unpack_codes(packed, n_bits: int, K: int):
    p = np.asarray(packed, dtype=np.uint8)
    per = 8 // n_bits
    mask = (1 << n_bits) - 1
    out = np.empty(p.shape[:-1] + (p.shape[-1], per), dtype=np.uint8)
    for j in range(per):
        out[..., j] = (p >> (n_bits * j)) & mask
    return out.reshape(p.shape[:-1] + (K,))


def reconstruct(codes, li, mid, scale, lib16):
    """Dense term: fp16(mid + scale * lib16[l][c]) per weight, as float64 [R, K]."""
    R, K = codes.shape
    grp = np.arange(K) // GROUP
    e = lib16[li[:, grp], codes]                         # [R, K]
    return round_to_f16(mid[:, grp] + scale[:, grp] * e)


def v2a_fit(w, n_bits: int, threshold: float, mu: float = 0.0, L: int = LIB, rounds: int = ROUNDS):
    """Fit V2a to one matrix w float32 [R, K].  Returns a dict:
      codes    uint8 [R, K * n_bits / 8] packed codes
      lib_idx  uint8 [R, K/128];  mid, scale  float64 [R, K/128] (fp16 values)
      lib      uint16 [L, 2^n_bits] fp16 bits;  lib_val float64 [L, 2^n_bits]
      row_ptr  int32 [R + 1], col int32 [nnz], val float64 [nnz] (fp16 residuals)
    """
    assert n_bits in (2, 4)
    w = np.asarray(w, dtype=np.float32)
    R, K = w.shape
    assert K % GROUP == 0
    w64 = w.astype(np.float64)
    out_mask = np.abs(w64 - mu) > threshold
    bulk = np.where(out_mask, mu, w64)
    mid, scale = group_stats(bulk)
    z = normalise(bulk, mid, scale)
    cbs = lloyd_rows(z, 1 << n_bits, rounds)
    lib16 = round_to_f16(lib_fit(cbs, L, rounds))
    li, codes = group_choice(z, lib16)
    dense = reconstruct(codes, li, mid, scale, lib16)
    rows, cols = np.nonzero(out_mask)
    val = round_to_f16(w64[rows, cols] - dense[rows, cols])
    row_ptr = np.zeros(R + 1, dtype=np.int32)
    np.add.at(row_ptr, rows + 1, 1)
    row_ptr = np.cumsum(row_ptr).astype(np.int32)
    return dict(codes=pack_codes(codes, n_bits), lib_idx=li, mid=mid, scale=scale,
                lib=lib16.astype(np.float16).view(np.uint16), lib_val=lib16, n_bits=n_bits,
                row_ptr=row_ptr, col=cols.astype(np.int32), val=val)


def v2a_dense(fit, K: int):
    codes = unpack_codes(fit["codes"], fit["n_bits"], K)
    return reconstruct(codes, fit["lib_idx"], fit["mid"], fit["scale"], fit["lib_val"])


def v2a_matrix(fit, K: int):
    """Dense plus sparse term as one float64 [R, K] matrix."""
    W = v2a_dense(fit, K).copy()
    R = W.shape[0]
    rows = np.repeat(np.arange(R), np.diff(fit["row_ptr"]))
    W[rows, fit["col"]] += fit["val"]
    return W


def bits_per_weight(n_bits: int, lib_index_bits: int = 5, scale_bits: int = 16, mid_bits: int = 16) -> float:
    """[XFP] V2a: N + (library index + scale + mid-point bits) / 128."""
    return n_bits + (lib_index_bits + scale_bits + mid_bits) / GROUP


def library_bytes(n_bits: int, L: int = LIB) -> int:
    """[XFP] V2a: an L = 32, N = 4 library is 32 x 16 x 2 bytes = 1 KB."""
    return L * (1 << n_bits) * 2
