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
