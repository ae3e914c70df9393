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


def _check_rows(a, C, offs, rows, N, K, seed, n_blocks=None):
    """Oracle on the sampled rows (each row's group weight regenerated).  With
    n_blocks, only those 128-column blocks of C are compared: a 128x128 weight
    block is quantised on its own, so quantising just the rows of B behind
    those columns gives the oracle's values there exactly."""
    groups = np.searchsorted(offs, rows, side="right") - 1
    got = np_(C[torch.as_tensor(rows, device="cuda")])
    ah = a[torch.as_tensor(rows, device="cuda")].float().cpu().numpy()
    aq, sa = oracle.quant_1x128(ah)
    blocks = list(range(N // 128)) if n_blocks is None else sorted(set(int(b) for b in n_blocks))
    cols = np.concatenate([np.arange(128 * b, 128 * b + 128) for b in blocks])
    ref = np.zeros((len(rows), len(cols)), dtype=np.float64)
    for g in np.unique(groups):
        w = synth.normal((N, K), 0.02, seed + 7 + int(g), device="cuda", dtype=torch.bfloat16)[
            torch.as_tensor(cols, device="cuda")].float().cpu().numpy()
        bq, sb = oracle.quant_128x128(w)
        sel = groups == g
        ref[sel] = oracle.gemm_blockscaled(aq[sel], sa[sel], bq, sb)
    r16 = oracle.round_bf16(ref)
    g = got[:, cols]
    assert normwise(g, r16) < TOL_NORMWISE
    assert np.mean(np.abs(g - r16) <= bf16_ulp(r16)) > 0.999


@pytest.mark.parametrize("N,K", SHAPES)
@pytest.mark.parametrize("M", [128, 1024, 4096, 16384])
def test_dense_sweep(lib, N, K, M):
    seed = 50 + N // 1024 + K // 1024 + M // 128
    a, C, offs = _run(lib, 1, [M], N, K, seed)
    rng = np.random.default_rng(seed)
    rows = np.sort(rng.choice(M, size=min(M, 6), replace=False))
    # six 128-column blocks: the first, the last and four drawn at random
    nb = N // 128
    blocks = [0, nb - 1] + list(rng.choice(nb, size=min(nb, 4), replace=False))
    _check_rows(a, C, offs, rows, N, K, seed, blocks)


GROUPED = [(N, K, M) for N, K in SHAPES for M in (128, 1024, 4096)] + [(7168, 2048, 16384)]


@pytest.mark.parametrize("N,K,M", GROUPED)
def test_grouped_sweep(lib, N, K, M):
    """256 groups of uniform random sizes summing to 8M: one row in every 8th
    non-empty group (ragged group boundaries included), each on the first, the
    last and one random 128-column block."""
    G = 256
    seed = 900 + N // 1024 + K // 1024 + M // 128
    sizes = synth.group_sizes(8 * M, G, seed)
    a, C, offs = _run(lib, G, sizes, N, K, seed)
    rng = np.random.default_rng(seed)
    nonempty = [g for g in range(G) if sizes[g] > 0]
    gs = nonempty[int(rng.integers(8))::8]
    # alternate the first row, the last row and a random row of the group
    rows = []
    for i, g in enumerate(gs):
        lo, hi = int(offs[g]), int(offs[g + 1])
        rows.append((lo, hi - 1, int(rng.integers(lo, hi)))[i % 3])
    nb = N // 128
    _check_rows(a, C, offs, np.array(sorted(rows)), N, K, seed, [0, nb - 1, int(rng.integers(nb))])
