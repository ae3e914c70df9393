"""Helpers shared by the GPU parity tests (no arithmetic of the layer here)."""
import numpy as np
import torch

# normwise relative tolerance for floating-point outputs of the FP8 path
# (the target the pages' FP8 recipe is held to in this repository: 1e-3 against
# the float64 oracle on the same quantised values)
TOL_NORMWISE = 1e-3


def np_(t: torch.Tensor) -> np.ndarray:
    t = t.detach().cpu()
    if t.dtype == torch.bfloat16:
        t = t.float()
    return t.numpy()


def normwise(got, ref) -> float:
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    den = np.linalg.norm(ref)
    return float(np.linalg.norm(got - ref) / (den if den > 0 else 1.0))


def bf16_ulp(v) -> np.ndarray:
    """Spacing of the bf16 grid at |v| (8 significant bits)."""
    a = np.abs(np.asarray(v, dtype=np.float64))
    e = np.floor(np.log2(np.maximum(a, 2.0 ** -126)))
    return 2.0 ** (e - 7)


def cuda(t: torch.Tensor) -> torch.Tensor:
    return t.contiguous().cuda()


def router_logit_tol(x, w_router, pieces: int = 3):
    """Per-token bound on the router-logit error of an fp32 accumulation of the
    H-term dot products (computed as `pieces` * H exact products): a random walk
    of per-add roundings of at most half an fp32 ulp of the running magnitude,
    taken at 8 standard deviations, with the running magnitude bounded by
    sum_h |x_h w_eh| (the largest over experts).  Returns float64 [T]."""
    x64 = np.abs(np.asarray(x, dtype=np.float64))
    w64 = np.abs(np.asarray(w_router, dtype=np.float64))
    mag = (x64 @ w64.T).max(axis=1)
    n = pieces * x64.shape[1]
    return 8.0 * np.sqrt(n) * 2.0 ** -24 * mag


def same_expert_sets(idx_a, idx_b):
    """Per token: the two routing tables select the same set of experts."""
    a = np.sort(np.asarray(idx_a), axis=1)
    b = np.sort(np.asarray(idx_b), axis=1)
    return np.all(a == b, axis=1)


def order_is_valid(idx, s32, b32):
    """Per token: the table lists its experts by descending s + b (fp32), ties
    to the lower index -- the order rule, checked on the given affinities."""
    idx = np.asarray(idx, dtype=np.int64)
    r = (np.asarray(s32, dtype=np.float32) + np.asarray(b32, dtype=np.float32)).astype(np.float32)
    v = np.take_along_axis(r, idx, axis=1).astype(np.float64)
    ok = (v[:, :-1] > v[:, 1:]) | ((v[:, :-1] == v[:, 1:]) & (idx[:, :-1] < idx[:, 1:]))
    return np.all(ok, axis=1)


def _e4m3_midpoints() -> np.ndarray:
    """The rounding boundaries of E4M3 (OCP OFP8) magnitudes: midpoints between
    consecutive finite values 0, k 2^-9 (k = 1..7), 2^e (1 + m/8) (e = -6..8,
    up to 448).  Values above 448 saturate, so there is no boundary beyond."""
    vals = [k * 2.0 ** -9 for k in range(8)]
    vals += [2.0 ** e * (1 + m / 8) for e in range(-6, 9) for m in range(8) if 2.0 ** e * (1 + m / 8) <= 448]
    vals = np.array(sorted(vals))
    return (vals[1:] + vals[:-1]) / 2


_MIDPOINTS = _e4m3_midpoints()


def e4m3_boundary_distance(t) -> np.ndarray:
    """|t| distance to the nearest E4M3 rounding boundary (float64)."""
    a = np.abs(np.asarray(t, dtype=np.float64))
    i = np.clip(np.searchsorted(_MIDPOINTS, a), 1, len(_MIDPOINTS) - 1)
    return np.minimum(np.abs(a - _MIDPOINTS[i - 1]), np.abs(a - _MIDPOINTS[i]))


def gemm_error_bound(mag, KB: int) -> np.ndarray:
    """Bound on the fp32 error of one promoted FP8 GEMM element against float64:
    the 128-product partial of each K block summed in fp32 (at most 128 roundings
    of 2^-23 relative, allowing truncation), the product of the two scales (one
    rounding) and KB fused multiply-adds (2^-24 each), each relative to the
    magnitude sum mag = sum_kb |sA sB| sum_k |qa qb|; doubled as a margin."""
    return 2.0 * (256 + 1 + KB) * 2.0 ** -24 * np.asarray(mag, dtype=np.float64)


def swiglu_error_bound(g, u, eg, eu) -> np.ndarray:
    """Bound on |act_gpu - act| for act = silu(g) u = g / (1 + exp(-g)) u when the
    kernel computes it in fp32 from inputs within eg, eu of g, u: first-order
    propagation (|d silu/dg| <= 1.1, d act/du = silu(g)) plus the kernel's own
    error: __expf(-g) within 2 + 1.173 |g| ulps of exp(-g) (entering through the
    denominator with weight exp(-g) / (1 + exp(-g))), __fdividef within 2 ulps,
    the addition and the final product half an ulp each (ulp <= 2^-23 |value|)."""
    g = np.asarray(g, dtype=np.float64)
    u = np.asarray(u, dtype=np.float64)
    with np.errstate(over="ignore"):
        e = np.exp(-g)
    w = np.where(np.isfinite(e), e / (1.0 + e), 1.0)
    silu = g / (1.0 + e)
    act = silu * u
    func = np.abs(act) * ((2.0 + 1.173 * np.abs(g)) * w + 2.0 + 1.0) * 2.0 ** -23
    return 1.1 * np.abs(u) * eg + np.abs(silu) * eu + 1.1 * eg * eu + func
