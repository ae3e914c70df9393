"""Backward FP8 grouped GEMMs of the expert FFN (oracle) -- test infrastructure only.

[repro-guide] section 3 config: gemm_fprop, gemm_dgrad and gemm_wgrad all in
fp8 (e4m3), inputs quantised tile-wise 1x128, weights block-wise 128x128;
[infra-answer]: E4M3 in both the forward and the backward pass, with the
products formed as promoted partial sums because the tensor cores do not
apply per-tile scales.

For one expert with forward Y = X W^T (X [M, K], W [N, K]):

dgrad   dX = dY W            contraction over N.  dY is an input, quantised
                             1x128 along N (its rows); W keeps its 128x128
                             blocks, read transposed.  Promotion every 128 of N:
    dX[m, k] = sum_nb  s_dY[m, nb] * s_W[nb, k // 128] * sum_{n in nb} dY_q[m, n] W_q[n, k]

wgrad   dW = dY^T X          contraction over the expert's M rows.  Reading:
                             the 1x128 input tiling is applied along the
                             contraction, i.e. to columns of dY and of X --
                             tiles of 128 consecutive rows of one column
                             (128x1), never crossing the expert's row range
                             (the last tile of a ragged range is shorter).
    dW[n, k] = sum_mb  s_dY[mb, n] * s_X[mb, k] * sum_{m in mb} dY_q[m, n] X_q[m, k]

The scale rule is the forward one (amax / 448 in fp32, amax 0 -> 1, codes
e4m3 round-to-nearest-even with saturation).  Every partial sum over one
128-wide block is exact in float64 (as in the forward oracle), so dX and dW
are the float64 products of the dequantised operands up to the order of the
final additions.
"""
from __future__ import annotations

import numpy as np

from .fp8 import _quant_tiles, e4m3_decode


def quant_128x1(x, offsets) -> tuple[np.ndarray, np.ndarray, np.ndarray]:
    """Column tiles of 128 consecutive rows inside each group's row range.

    x [M, C] (bf16 or fp32 values), offsets int [G+1] (row ranges).
    Returns codes uint8 [M, C], scales float32 [n_tiles, C] and the first row
    of every tile int64 [n_tiles + 1] (the last entry is M)."""
    x32 = np.asarray(x, dtype=np.float32)
    M, C = x32.shape
    offsets = np.asarray(offsets, dtype=np.int64)
    starts = []
    for g in range(offsets.shape[0] - 1):
        starts.extend(range(int(offsets[g]), int(offsets[g + 1]), 128))
    starts.append(int(offsets[-1]))
    tile_rows = np.asarray(starts, dtype=np.int64)
    codes = np.zeros((M, C), dtype=np.uint8)
    scales = np.zeros((len(starts) - 1, C), dtype=np.float32)
    for t in range(len(starts) - 1):
        r0, r1 = tile_rows[t], tile_rows[t + 1]
        q, s = _quant_tiles(np.ascontiguousarray(x32[r0:r1].T))      # [C, rows of the tile]
        codes[r0:r1] = q.T
        scales[t] = s
    return codes, scales, tile_rows


def dgrad_blockscaled(dyq, sdy, wq, sw) -> np.ndarray:
    """dX = dY W with promotion every 128 of N, float64 [M, K].

    dyq uint8 [M, N], sdy fp32 [M, N/128] (1x128 tiles); wq uint8 [N, K],
    sw fp32 [N/128, K/128] (128x128 blocks)."""
    dY = e4m3_decode(dyq)
    W = e4m3_decode(wq)
    M, N = dY.shape
    K = W.shape[1]
    assert N % 128 == 0 and K % 128 == 0 and W.shape[0] == N
    sdy64 = np.asarray(sdy, dtype=np.float64)
    sw64 = np.asarray(sw, dtype=np.float64)
    dX = np.zeros((M, K), dtype=np.float64)
    for nb in range(N // 128):
        ns = slice(nb * 128, (nb + 1) * 128)
        P = dY[:, ns] @ W[ns, :]                                 # exact partial sum
        s_k = np.repeat(sw64[nb, :], 128)                        # weight scale of each output column
        dX += (sdy64[:, nb:nb + 1] * s_k[None, :]) * P
    return dX


def wgrad_blockscaled(dyq, sdy, xq, sx, tile_rows, r0: int, r1: int) -> np.ndarray:
    """dW = dY^T X over rows r0..r1-1 (one expert) with promotion per 128x1 tile.

    dyq [M, N], xq [M, K] codes; sdy [n_tiles, N], sx [n_tiles, K] scales and
    tile_rows [n_tiles + 1] from quant_128x1 of both operands with the same
    row ranges.  Returns float64 [N, K]."""
    dY = e4m3_decode(dyq)
    X = e4m3_decode(xq)
    N, K = dY.shape[1], X.shape[1]
    sdy64 = np.asarray(sdy, dtype=np.float64)
    sx64 = np.asarray(sx, dtype=np.float64)
    dW = np.zeros((N, K), dtype=np.float64)
    tile_rows = np.asarray(tile_rows, dtype=np.int64)
    for t in range(tile_rows.shape[0] - 1):
        a, b = int(tile_rows[t]), int(tile_rows[t + 1])
        if a < r0 or b > r1:
            continue
        P = dY[a:b].T @ X[a:b]                                   # exact partial sum over <= 128 rows
        dW += (sdy64[t][:, None] * sx64[t][None, :]) * P
    return dW
