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
