"""Backward weight gradient in FP8 on the GPU against the float64 oracle: the
128x1 grouped quantiser (bit-exact codes and scales, transposed and padded
layout) and the grouped wgrad GEMM (per element within the fp32 accumulation
bound of the promoted sum), on ragged groups including empty and one-row
experts, and on one expert of the DeepSeek-V3 size."""
import numpy as np
import pytest
import torch

import synth
from oracle.backward import quant_128x1, wgrad_blockscaled
from tests._util import cuda, gemm_error_bound, normwise, np_, TOL_NORMWISE

pytestmark = pytest.mark.gpu


def _quant_gpu(lib, x, offs):
    M, C = x.shape
    G = len(offs) - 1
    p_cap, t_cap = lib.wgrad_capacities(M, G)
    q = torch.full((C, p_cap), 0xAB, dtype=torch.uint8, device="cuda")
    s = torch.full((t_cap, C), -1.0, dtype=torch.float32, device="cuda")
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    goffs = cuda(torch.tensor(offs, dtype=torch.int32))
    lib.fp8_quant_128x1_grouped(cuda(x), goffs, q, s, st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    return q, s, goffs


CASES = [  # group sizes, N (columns of dY), K (columns of X)
    ([0, 1, 130, 257, 64, 0, 300], 256, 384),
    ([128, 128], 384, 256),
    ([5] * 20 + [0, 700], 128, 512),
]


@pytest.mark.parametrize("sizes,N,K", CASES)
def test_quant_128x1_bitexact(lib, sizes, N, K):
    offs = np.concatenate([[0], np.cumsum(sizes)]).astype(np.int64)
    M = int(offs[-1])
    x = synth.heavy_tailed(M, K, 31 + M)
    q, s, _ = _quant_gpu(lib, x, offs)
    rq, rs, rows = quant_128x1(x.float().numpy(), offs)
    q, s = np_(q), np_(s)
    for t in range(len(rows) - 1):
        a, b = int(rows[t]), int(rows[t + 1])
        assert np.array_equal(q[:, 128 * t:128 * t + (b - a)], rq[a:b].T)
        assert not q[:, 128 * t + (b - a):128 * (t + 1)].any()          # padding rows are code 0
        assert np.array_equal(s[t], rs[t])


def _wgrad_check(lib, sizes, N, K, seed):
    offs = np.concatenate([[0], np.cumsum(sizes)]).astype(np.int64)
    M, G = int(offs[-1]), len(sizes)
    dy = synth.heavy_tailed(M, N, seed)
    x = synth.activations(M, K, seed + 1)
    dq, ds, goffs = _quant_gpu(lib, dy, offs)
    xq, xs, _ = _quant_gpu(lib, x, offs)
    dW = torch.full((G, N, K), float("nan"), dtype=torch.float32, device="cuda")
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    lib.fp8_grouped_gemm_wgrad(goffs, M, dq, ds, xq, xs, dW, st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    got = np_(dW)
    rdq, rds, rows = quant_128x1(dy.float().numpy(), offs)
    rxq, rxs, _ = quant_128x1(x.float().numpy(), offs)
    for g in range(G):
        r0, r1 = int(offs[g]), int(offs[g + 1])
        ref = wgrad_blockscaled(rdq, rds, rxq, rxs, rows, r0, r1)
        if r1 == r0:
            assert not got[g].any()                         # an empty expert's gradient is zero
            continue
        mag = wgrad_blockscaled(rdq & 0x7F, rds, rxq & 0x7F, rxs, rows, r0, r1)
        kb = int(((rows[:-1] >= r0) & (rows[:-1] < r1)).sum())
        assert np.all(np.abs(got[g] - ref) <= gemm_error_bound(mag, kb)), f"group {g}"
        assert normwise(got[g], ref) < TOL_NORMWISE


@pytest.mark.parametrize("sizes,N,K", CASES)
def test_wgrad_matches_oracle(lib, sizes, N, K):
    _wgrad_check(lib, sizes, N, K, seed=50 + N + K)


@pytest.mark.slow
def test_wgrad_dsv3_expert(lib):
    """One routed expert of the DeepSeek-V3 layer with a ragged 300-row load:
    the gradient of its W13 (dY [300, 2I = 4096], X [300, H = 7168]) and of
    its W2 (dY [300, H], act [300, I = 2048]), next to an empty expert."""
    _wgrad_check(lib, [300, 0], 4096, 7168, seed=7)
    _wgrad_check(lib, [0, 300], 7168, 2048, seed=8)
