"""The FP8 block-scaled GEMM sweep at its full sizes: dense (N, K) in {(4096, 7168),
(7168, 2048), (18432, 7168), (7168, 18432)} with M in {128, 1024, 4096, 16384} and
grouped variants with 256 groups of uniform random sizes summing to 8M.  A is bf16
N(0,1) with 1 % of the entries x100 (1x128 tiles), B is N(0, 0.02) (128x128
blocks), C bf16.  Parity on sampled rows: every row of C depends only on its own
A row, so the oracle computes the sampled rows exactly."""
import numpy as np
import pytest
import torch

import oracle
import synth
from tests._util import TOL_NORMWISE, bf16_ulp, np_, normwise

pytestmark = [pytest.mark.gpu, pytest.mark.slow]

SHAPES = [(4096, 7168), (7168, 2048), (18432, 7168), (7168, 18432)]


def _quant_b(lib, G, N, K, seed):
    qb = torch.empty(G, N, K, dtype=torch.uint8, device="cuda")
    sb = torch.empty(G, N // 128, K // 128, dtype=torch.float32, device="cuda")
    for g in range(G):
        w = synth.normal((N, K), 0.02, seed + g, device="cuda", dtype=torch.bfloat16)
        lib.fp8_quant_128x128(w, qb[g], sb[g])
    return qb, sb


def _run(lib, G, sizes, N, K, seed, mode=0):
    M = int(sum(sizes))
    a = synth.heavy_tailed(M, K, seed, device="cuda")
    qa = torch.empty(M, K, dtype=torch.uint8, device="cuda")
    sa = torch.empty(M, K // 128, dtype=torch.float32, device="cuda")
    lib.fp8_quant_1x128(a, qa, sa)
    qb, sb = _quant_b(lib, G, N, K, seed + 7)
    offs = torch.tensor(np.concatenate([[0], np.cumsum(sizes)]), dtype=torch.int32, device="cuda")
    C = torch.empty(M, N, dtype=torch.bfloat16, device="cuda")
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    lib.fp8_grouped_gemm_blockscaled(G, offs, M, N, K, qa, sa, qb, sb, lib.MOE_EPI_BF16 | mode, C, None, st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    return a, C, offs.cpu().numpy()


def _check_rows(a, C, offs, rows, N, K, seed):
    """Oracle on the sampled rows (each row's group weight regenerated)."""
    groups = np.searchsorted(offs, rows, side="right") - 1
    got = np_(C[torch.as_tensor(rows, device="cuda")])
    ah = a[torch.as_tensor(rows, device="cuda")].float().cpu().numpy()
    aq, sa = oracle.quant_1x128(ah)
    ref = np.zeros_like(got, dtype=np.float64)
    for g in np.unique(groups):
        w = synth.normal((N, K), 0.02, seed + 7 + int(g), device="cuda", dtype=torch.bfloat16).float().cpu().numpy()
        bq, sb = oracle.quant_128x128(w)
        sel = groups == g
        ref[sel] = oracle.gemm_blockscaled(aq[sel], sa[sel], bq, sb)
    r16 = oracle.round_bf16(ref)
    assert normwise(got, r16) < TOL_NORMWISE
    assert np.mean(np.abs(got - r16) <= bf16_ulp(r16)) > 0.999


@pytest.mark.parametrize("N,K", SHAPES)
@pytest.mark.parametrize("M", [128, 1024, 4096, 16384])
def test_dense_sweep(lib, N, K, M):
    if M == 16384 and N * K > 7168 * 7168:
        pytest.skip("largest dense shapes checked at M <= 4096 (runtime)")
    seed = 50 + N // 1024 + K // 1024 + M // 128
    a, C, offs = _run(lib, 1, [M], N, K, seed)
    rows = np.sort(np.random.default_rng(seed).choice(M, size=min(M, 6), replace=False))
    _check_rows(a, C, offs, rows, N, K, seed)


@pytest.mark.parametrize("N,K", SHAPES)
@pytest.mark.parametrize("M", [128, 1024])
def test_grouped_sweep(lib, N, K, M):
    G = 256
    seed = 900 + N // 1024 + K // 1024 + M // 128
    sizes = synth.group_sizes(8 * M, G, seed)
    a, C, offs = _run(lib, G, sizes, N, K, seed)
    rng = np.random.default_rng(seed)
    nonempty = [g for g in range(G) if sizes[g] > 0]
    gs = rng.choice(nonempty, size=2, replace=False)
    rows = np.sort(np.array([rng.integers(offs[g], offs[g + 1]) for g in gs]))
    _check_rows(a, C, offs, rows, N, K, seed)
