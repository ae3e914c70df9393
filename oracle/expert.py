"""Block-scaled FP8 GEMM with promotion every 128 of K, SwiGLU, requant (oracle).

Test infrastructure only (see the package docstring).

[report-walkthrough] section 4.3: GEMM inputs are quantised per block with
their own scales and accumulation stays in higher precision.  [infra-answer]:
the per-tile (1x128) / per-group (128x128) scales are not supported by the
tensor cores, so the product is formed as partial sums that are promoted.
Reading: for every 128-wide block kb of K,
    P_kb[m, n] = sum_{k in kb} decode(qa[m, k]) * decode(qb[n, k])
    C[m, n]   += sA[m, kb] * sB[n // 128, kb] * P_kb[m, n].
P_kb is exact in float64 (products of two E4M3 values have at most 8
significant bits and exponents in [-18, 17], so 128 of them sum exactly
within 53 bits), so C is the float64 dot product of the dequantised operands
up to the order of the final float64 additions.

SwiGLU ([infra-answer]: SwiGLU is one of the recomputed operators;
[arch-overview]: expert intermediate 2048): act = silu(g) * u with
silu(g) = g / (1 + exp(-g)); g is the first I rows of the expert's
up-projection W13 and u the next I rows; no bias terms.
"""
from __future__ import annotations

import numpy as np

from .fp8 import e4m3_decode, quant_1x128, round_bf16


def gemm_blockscaled(aq, sa, bq, sb) -> np.ndarray:
    """C = A . B^T with per-128-K promotion, float64.

    aq uint8 [M, K], sa fp32 [M, K/128]; bq uint8 [N, K], sb fp32 [N/128, K/128]."""
    A = e4m3_decode(aq)
    B = e4m3_decode(bq)
    M, K = A.shape
    N = B.shape[0]
    assert K % 128 == 0 and N % 128 == 0 and B.shape[1] == K
    sa64 = np.asarray(sa, dtype=np.float64)
    sb64 = np.asarray(sb, dtype=np.float64)
    C = np.zeros((M, N), dtype=np.float64)
    for kb in range(K // 128):
        ks = slice(kb * 128, (kb + 1) * 128)
        P = A[:, ks] @ B[:, ks].T                       # exact partial sum
        s_n = np.repeat(sb64[:, kb], 128)               # scale of each output column's block
        C += (sa64[:, kb:kb + 1] * s_n[None, :]) * P
    return C


def grouped_gemm_blockscaled(offsets, aq, sa, bq, sb) -> np.ndarray:
    """Rows offsets[g]..offsets[g+1]-1 of A times B[g]^T, float64 [M, N].

    bq uint8 [G, N, K], sb fp32 [G, N/128, K/128]."""
    offsets = np.asarray(offsets, dtype=np.int64)
    G = offsets.shape[0] - 1
    M = aq.shape[0]
    N = bq.shape[1]
    C = np.zeros((M, N), dtype=np.float64)
    for g in range(G):
        r0, r1 = int(offsets[g]), int(offsets[g + 1])
        if r1 > r0:
            C[r0:r1] = gemm_blockscaled(aq[r0:r1], sa[r0:r1], bq[g], sb[g])
    return C


def silu(g) -> np.ndarray:
    g = np.asarray(g, dtype=np.float64)
    return g / (1.0 + np.exp(-g))


def swiglu(gu) -> np.ndarray:
    """act = silu(gate) * up; gu [M, 2I] holds gate columns then up columns."""
    gu = np.asarray(gu, dtype=np.float64)
    I = gu.shape[1] // 2
    return silu(gu[:, :I]) * gu[:, I:]


def swiglu_requant(gu):
    """SwiGLU in float64, rounded to fp32 (the precision the kernel decides
    the codes in), then 1x128 quantisation.  Returns (codes, scales, act64)."""
    act = swiglu(gu)
    codes, scales = quant_1x128(act.astype(np.float32))
    return codes, scales, act


def expert_ffn(aq, sa, w13q, s13, w2q, s2):
    """One expert (or the shared expert) on already-quantised input rows.

    aq/sa: the rows' 1x128 codes and scales; w13q [2I, H] / s13, w2q [H, I] /
    s2: 128x128 block-quantised weights.  Returns (y float64 rounded to bf16,
    y float64 unrounded).  The intermediate activation is requantised 1x128."""
    gu = gemm_blockscaled(aq, sa, w13q, s13)
    actq, acts, _ = swiglu_requant(gu)
    y = gemm_blockscaled(actq, acts, w2q, s2)
    return round_bf16(y), y
