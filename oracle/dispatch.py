"""Token permutation into per-expert segments and the gated combine (oracle).

Test infrastructure only (see the package docstring).

The pages give the semantics y = sum_j gate_j * ffn_{idx_j}(h) with no token
ever dropped ([report-walkthrough] section 3.2 pseudocode and section 3.4:
no capacity factor, every token reaches all K experts) and a dispatch /
expert MLP / combine split of the forward block ([report-walkthrough]
section 4.1).  They give no layout.  The layout used (a reading of
the pages): rows grouped by expert in ascending expert order, and within an
expert in ascending token order (a stable sort by expert); the x rows are
quantised first and their codes gathered (1x128 tiles lie inside one token
row, so quantise-then-gather equals gather-then-quantise bit for bit).
"""
from __future__ import annotations

import numpy as np

from .fp8 import round_bf16


def permute(idx, E: int):
    """Stable counting sort of the (token, slot) pairs by expert.

    idx int [T, K].  Returns (load [E], offsets [E+1], tok_of [T*K],
    row_of [T*K]) as int32: rows offsets[e] .. offsets[e+1]-1 belong to
    expert e in ascending token order; tok_of[row] is the token of a row and
    row_of[t*K + k] the row of pair (t, k)."""
    idx = np.asarray(idx, dtype=np.int64)
    T, K = idx.shape
    pairs = sorted((int(idx[t, k]), t, k) for t in range(T) for k in range(K))
    load = np.zeros(E, dtype=np.int32)
    for e, _, _ in pairs:
        load[e] += 1
    offsets = np.zeros(E + 1, dtype=np.int32)
    offsets[1:] = np.cumsum(load)
    tok_of = np.zeros(T * K, dtype=np.int32)
    row_of = np.zeros(T * K, dtype=np.int32)
    for row, (e, t, k) in enumerate(pairs):
        tok_of[row] = t
        row_of[t * K + k] = row
    return load, offsets, tok_of, row_of


def unpermute_rows(rows, row_of, T: int, K: int):
    """Inverse of the gather: out[t, k] = rows[row_of[t*K + k]]."""
    rows = np.asarray(rows)
    r = np.asarray(row_of, dtype=np.int64).reshape(T, K)
    return rows[r]


def combine(yperm, row_of, w, yshared=None):
    """out[t] = sum_k w[t,k] * yperm[row_of[t,k]] (+ yshared[t]), float64.

    yperm [T*K, H] and yshared [T, H] hold the values the layer stored (bf16
    values); w [T, K] fp32 gates.  Summation is exact-order float64."""
    w64 = np.asarray(w, dtype=np.float64)
    T, K = w64.shape
    y = np.asarray(yperm, dtype=np.float64)
    r = np.asarray(row_of, dtype=np.int64).reshape(T, K)
    out = np.zeros((T, y.shape[1]), dtype=np.float64)
    for k in range(K):
        out += w64[:, k:k + 1] * y[r[:, k]]
    if yshared is not None:
        out += np.asarray(yshared, dtype=np.float64)
    return out


def combine_by_rank(yperm, row_of, w, rank, yshared=None):
    """Node-limited combine: out[t] = sum over the ranks r that token t selected
    of bf16( sum_{k : rank[t,k] = r} w[t,k] * yperm[row_of[t,k]] ) (+ yshared[t]),
    float64 sums.

    [report-walkthrough] section 3.4 sends a token at most once to each node it
    selected; section 4.1 has the node compute the token's experts there and
    accumulate their results while the combine forwards them back.  Each rank's
    gated partial sum is the row that crosses back; it is stored in bf16, the
    precision in which the layer stores the expert rows it sums, and the source
    adds the partials.
    rank int [T, K]: the rank of each slot's expert."""
    w64 = np.asarray(w, dtype=np.float64)
    T, K = w64.shape
    y = np.asarray(yperm, dtype=np.float64)
    r = np.asarray(row_of, dtype=np.int64).reshape(T, K)
    rk = np.asarray(rank, dtype=np.int64).reshape(T, K)
    out = np.zeros((T, y.shape[1]), dtype=np.float64)
    for t in range(T):
        for dest in sorted(set(int(v) for v in rk[t])):
            part = np.zeros(y.shape[1], dtype=np.float64)
            for k in range(K):
                if rk[t, k] == dest:
                    part += w64[t, k] * y[r[t, k]]
            out[t] += round_bf16(part)
    if yshared is not None:
        out += np.asarray(yshared, dtype=np.float64)
    return out
