"""Parallel evaluation of the oracle's expert FFNs for the full-size parity tests.

Test infrastructure.  The full-size checks compare whole expert segments and
dozens of sampled tokens with the float64 oracle, which has to quantise every
expert it touches (about 3 s of numpy per DeepSeek-V3 expert).  This module
farms those expert FFNs out to a process pool started with the "spawn"
method (never forked: the test process holds a CUDA context).

Each worker regenerates the expert's master weights from their seeds with
`synth` (on the device the layer drew them on; a CUDA draw in a worker is the
same Philox stream as in the parent), quantises them with the oracle and runs
`oracle.expert_ffn` on the rows it is given.  Nothing here computes any part
of the layer itself.
"""
from __future__ import annotations

import atexit
import multiprocessing as mp
import os

import numpy as np

_POOL = None


def _workers() -> int:
    n = os.cpu_count() or 2
    try:
        import psutil
        mem_gb = psutil.virtual_memory().available / 2 ** 30
        n = min(n, max(1, int(mem_gb // 6)))     # the float64 quantiser peaks at a few GB
    except Exception:
        pass
    return max(1, min(16, n))


def _init():
    from threadpoolctl import threadpool_limits
    threadpool_limits(2)


def pool():
    global _POOL
    if _POOL is None:
        _POOL = mp.get_context("spawn").Pool(_workers(), initializer=_init)
        atexit.register(_POOL.terminate)
    return _POOL


def _master(shape, kind: str, e: int, device: str) -> np.ndarray:
    import synth
    H, I = shape.H, shape.I
    if e < 0:
        tid = synth.SH13 if kind == "w13" else synth.SH2
    else:
        tid = synth.W13 if kind == "w13" else synth.W2
    rows, cols = (2 * I, H) if kind == "w13" else (H, I)
    w = synth.expert_weight(rows, cols, shape.w_std, synth.seed_of(shape, tid, max(e, 0)), device=device)
    return w.float().cpu().numpy()


def _ffn_task(args):
    shape, e, xq, xs, device = args
    import oracle
    q13, s13 = oracle.quant_128x128(_master(shape, "w13", e, device))
    q2, s2 = oracle.quant_128x128(_master(shape, "w2", e, device))
    y16, _ = oracle.expert_ffn(xq, xs, q13, s13, q2, s2)
    return e, y16.astype(np.float32)      # bf16-rounded values are exact in fp32


def expert_outputs(shape, jobs: dict, device: str = "cuda") -> dict:
    """jobs: {expert e (-1 = shared): (xq uint8 [n, H], xs fp32 [n, H/128])}.
    Returns {e: y float32 [n, H]}, the oracle's bf16-rounded expert outputs."""
    tasks = [(shape, int(e), xq, xs, device) for e, (xq, xs) in jobs.items()]
    return dict(pool().imap_unordered(_ffn_task, tasks))
