"""The whole DeepSeekMoE layer forward, and its per-token form (oracle).

Test infrastructure only (see the package docstring).

Forward order ([report-walkthrough] section 3.2 pseudocode, with the FP8
recipe of section 4.3 and [repro-guide] section 3):
  1. s = sigmoid(x W_r^T); group-limited top-K on s + b; gates from s.
  2. x quantised to E4M3 per 1x128 tile; rows gathered per expert.
  3. per expert: G = xq W13^T (promoted per 128 of K), act = silu(g) * u,
     act requantised per 1x128 tile, y = actq W2^T, stored as bf16.
  4. shared expert: the same FFN on every token, stored as bf16.
  5. out[t] = sum_k w[t,k] y_{t,k} + y_shared[t], stored as bf16.
  6. load = bincount(idx) drives the bias update (separate call).
The layer input x is the already-normalised hidden state; there is no
residual add here (a reading: the pages place the norm and residual outside
the MoE FFN).
"""
from __future__ import annotations

from dataclasses import dataclass, field
from typing import Callable

import numpy as np

from .dispatch import combine, permute
from .expert import expert_ffn
from .fp8 import quant_128x128, quant_1x128, round_bf16
from .routing import expert_load, router_scores, select_experts


@dataclass
class LayerWeights:
    """Block-quantised expert weights, produced on demand.

    master(kind, e) returns one master weight as an array-like of bf16
    values: kind "w13" -> [2I, H], "w2" -> [H, I]; e = -1 is the shared
    expert.  Quantised blocks are cached per (kind, e)."""
    master: Callable[[str, int], np.ndarray]
    cache: dict = field(default_factory=dict)

    def get(self, kind: str, e: int):
        key = (kind, e)
        if key not in self.cache:
            self.cache[key] = quant_128x128(np.asarray(self.master(kind, e), dtype=np.float32))
        return self.cache[key]


def quantize_layer_weights(w13, w2, sh13, sh2) -> LayerWeights:
    """LayerWeights over in-memory master weights w13 [E,2I,H], w2 [E,H,I],
    sh13 [2I,H], sh2 [H,I]."""
    def master(kind, e):
        if kind == "w13":
            return sh13 if e < 0 else w13[e]
        return sh2 if e < 0 else w2[e]
    return LayerWeights(master)


def moe_forward(x, w_router, bias, weights: LayerWeights, n_group: int, topk_group: int,
                K: int, rho: float, offset=None, with_shared: bool = True) -> dict:
    """The full layer on every token.  Returns every intermediate."""
    x32 = np.asarray(x, dtype=np.float32)
    T, H = x32.shape
    E = np.asarray(w_router).shape[0]
    s64 = router_scores(x32, w_router, offset)
    s32 = s64.astype(np.float32)
    idx, w = select_experts(s32, bias, n_group, topk_group, K, rho)
    load = expert_load(idx, E)
    _, offsets, tok_of, row_of = permute(idx, E)
    xq, xs = quant_1x128(x32)
    aq, as_ = xq[tok_of], xs[tok_of]
    yperm = np.zeros((T * K, H), dtype=np.float64)
    for e in range(E):
        r0, r1 = int(offsets[e]), int(offsets[e + 1])
        if r1 > r0:
            w13q, s13 = weights.get("w13", e)
            w2q, s2 = weights.get("w2", e)
            yperm[r0:r1], _ = expert_ffn(aq[r0:r1], as_[r0:r1], w13q, s13, w2q, s2)
    ysh = None
    if with_shared:
        w13q, s13 = weights.get("w13", -1)
        w2q, s2 = weights.get("w2", -1)
        ysh, _ = expert_ffn(xq, xs, w13q, s13, w2q, s2)
    out64 = combine(yperm, row_of, w, ysh)
    return dict(s64=s64, s32=s32, idx=idx, w=w, load=load, offsets=offsets, tok_of=tok_of,
                row_of=row_of, xq=xq, xs=xs, aq=aq, as_=as_, yperm=yperm, ysh=ysh,
                out64=out64, out=round_bf16(out64))


def moe_forward_tokens(x_rows, w_router, bias, weights: LayerWeights, n_group: int,
                       topk_group: int, K: int, rho: float, offset=None,
                       with_shared: bool = True, idx=None) -> dict:
    """The layer's output for a few tokens only.

    Every step of the layer acts on one token row at a time (routing, 1x128
    tiles, GEMM rows, combine), so a token's output does not depend on the
    other tokens of the batch.  `idx` may pin the routing (for tokens whose
    top-K is a near tie); otherwise it is computed here."""
    x32 = np.asarray(x_rows, dtype=np.float32)
    n = x32.shape[0]
    s64 = router_scores(x32, w_router, offset)
    s32 = s64.astype(np.float32)
    sel_idx, w = select_experts(s32, bias, n_group, topk_group, K, rho)
    if idx is not None:
        idx = np.asarray(idx, dtype=np.int32)
        s_sel = np.take_along_axis(s32, idx.astype(np.int64), axis=1).astype(np.float64)
        w = ((rho * s_sel) / s_sel.sum(axis=1, keepdims=True)).astype(np.float32)
    else:
        idx = sel_idx
    xq, xs = quant_1x128(x32)
    out64 = np.zeros_like(x32, dtype=np.float64)
    ys = np.zeros((n, K, x32.shape[1]), dtype=np.float64)
    for t in range(n):
        for k in range(K):
            e = int(idx[t, k])
            w13q, s13 = weights.get("w13", e)
            w2q, s2 = weights.get("w2", e)
            ys[t, k], _ = expert_ffn(xq[t:t + 1], xs[t:t + 1], w13q, s13, w2q, s2)
            out64[t] += float(w[t, k]) * ys[t, k]
    ysh = None
    if with_shared:
        w13q, s13 = weights.get("w13", -1)
        w2q, s2 = weights.get("w2", -1)
        ysh, _ = expert_ffn(xq, xs, w13q, s13, w2q, s2)
        out64 += ysh
    return dict(s64=s64, s32=s32, idx=idx, w=w, xq=xq, xs=xs, ys=ys, ysh=ysh,
                out64=out64, out=round_bf16(out64))
