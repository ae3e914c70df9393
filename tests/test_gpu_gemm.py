"""GPU parity of the grouped FP8 block-scaled GEMM (tcgen05) against the float64
oracle, through the C ABI.  Operands are drawn by `synth` in bf16 and quantised
independently by each side (the quantisers agree bit for bit, see
test_gpu_kernels), so both sides multiply the same E4M3 codes and scales."""
import numpy as np
import pytest
import torch

import oracle
import synth
from tests._util import TOL_NORMWISE, bf16_ulp, cuda, normwise, np_

pytestmark = pytest.mark.gpu


def _operands(sizes, N, K, seed, heavy=True, m_extra=0):
    M = int(sum(sizes)) + m_extra
    G = len(sizes)
    a = synth.heavy_tailed(M, K, seed) if heavy else synth.activations(M, K, seed)
    b = synth.normal((G * N, K), 0.02, seed + 1, dtype=torch.bfloat16).reshape(G, N, K)
    aq, sa = oracle.quant_1x128(a.float().numpy())
    bq = np.empty((G, N, K), np.uint8)
    sb = np.empty((G, N // 128, K // 128), np.float32)
    for g in range(G):
        bq[g], sb[g] = oracle.quant_128x128(b[g].float().numpy())
    offs = np.concatenate([[0], np.cumsum(sizes)]).astype(np.int32)
    return a, b, aq, sa, bq, sb, offs, M


def _gpu_operands(lib, a, b):
    M, K = a.shape
    G, N, _ = b.shape
    dev = dict(device="cuda")
    qa = torch.empty(M, K, dtype=torch.uint8, **dev)
    sa = torch.empty(M, K // 128, dtype=torch.float32, **dev)
    lib.fp8_quant_1x128(cuda(a), qa, sa)
    qb = torch.empty(G, N, K, dtype=torch.uint8, **dev)
    sb = torch.empty(G, N // 128, K // 128, dtype=torch.float32, **dev)
    lib.fp8_quant_128x128(cuda(b), qb, sb)
    return qa, sa, qb, sb


GEMM_CASES = [  # sizes, N, K
    ([200], 512, 1024),                         # dense, ragged M tile, 8 K blocks (ring wraps)
    ([0, 130, 1, 257, 40], 384, 256),           # empty group, 1-row group, N tail of 128
    ([5] * 40, 256, 384),                       # many small groups
    (list(range(0, 300, 7)), 768, 512),         # 43 groups, > 148 tiles: persistent loop
    ([128, 128, 256], 256, 128),                # exact tiles, single K block
    ([600, 0, 255, 256, 1], 512, 384),          # several 256-row pair tiles, ragged
    ([90, 3, 300, 2100], 512, 256),             # large last group: its tiles are interleaved in two chunks
]


TILE_MODES = {"pair": 0x200, "single": 0x100}   # CTA-pair tiles or one-SM tiles


@pytest.mark.parametrize("sizes,N,K", GEMM_CASES)
@pytest.mark.parametrize("epi", ["f32", "bf16"])
@pytest.mark.parametrize("mode", list(TILE_MODES))
def test_grouped_gemm(lib, sizes, N, K, epi, mode):
    a, b, aq, sa, bq, sb, offs, M = _operands(sizes, N, K, seed=len(sizes) * 7 + N + K, m_extra=3)
    qa, qsa, qb, qsb = _gpu_operands(lib, a, b)
    ref = oracle.grouped_gemm_blockscaled(offs, aq, sa, bq, sb)
    dt = torch.float32 if epi == "f32" else torch.bfloat16
    sentinel = 7.0
    C = torch.full((M, N), sentinel, dtype=dt, device="cuda")
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    e = (lib.MOE_EPI_F32 if epi == "f32" else lib.MOE_EPI_BF16) | TILE_MODES[mode]
    lib.fp8_grouped_gemm_blockscaled(len(sizes), cuda(torch.from_numpy(offs)), M, N, K, qa, qsa, qb, qsb,
                                     e, C, None, st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    got = np_(C)
    used = int(offs[-1])
    assert np.all(got[used:] == sentinel)             # rows outside every group untouched
    g, r = got[:used], ref[:used]
    if epi == "bf16":
        r = oracle.round_bf16(r)
    assert normwise(g, r) < TOL_NORMWISE
    # element-wise: fp32 accumulation error is far below a bf16 ulp
    tol = 1e-4 * np.abs(r) + 1e-5 * np.abs(r).max() + (bf16_ulp(r) if epi == "bf16" else 0)
    assert np.all(np.abs(g - r) <= tol)


@pytest.mark.parametrize("mode", list(TILE_MODES))
def test_integer_exact_gemm(lib, mode):
    """Integer-valued codes with unit-friendly scales: the result is an exact
    integer matrix on both sides (fp32 sums of integers below 2^24)."""
    rng = np.random.default_rng(0)
    M, N, K = 256, 256, 512
    ai = rng.integers(-8, 9, (M, K)).astype(np.float32)
    bi = rng.integers(-8, 9, (N, K)).astype(np.float32)
    # place 448 in every tile/block so the scale is exactly 1
    ai[:, ::128] = 448.0
    bi[0::128, ::128] = 448.0
    a = torch.from_numpy(ai).to(torch.bfloat16)
    b = torch.from_numpy(bi).to(torch.bfloat16).reshape(1, N, K)
    qa, qsa, qb, qsb = _gpu_operands(lib, a, b)
    assert torch.all(qsa == 1.0) and torch.all(qsb == 1.0)
    C = torch.empty(M, N, dtype=torch.float32, device="cuda")
    offs = torch.tensor([0, M], dtype=torch.int32, device="cuda")
    lib.fp8_grouped_gemm_blockscaled(1, offs, M, N, K, qa, qsa, qb, qsb, lib.MOE_EPI_F32 | TILE_MODES[mode], C)
    torch.cuda.synchronize()
    exact = ai.astype(np.int64) @ bi.astype(np.int64).T
    assert np.array_equal(np_(C).astype(np.int64), exact)


@pytest.mark.parametrize("sizes,I,K", [([70, 0, 150], 256, 384), ([1], 128, 128), ([300] * 3, 512, 1024),
                                       ([50, 1100], 256, 256), ([257, 511, 3, 0, 129], 256, 256)])
@pytest.mark.parametrize("mode", list(TILE_MODES))
def test_grouped_gemm_swiglu_requant(lib, sizes, I, K, mode):
    N = 2 * I
    a, b, aq, sa, bq, sb, offs, M = _operands(sizes, N, K, seed=91 + I, heavy=False)
    qa, qsa, qb, qsb = _gpu_operands(lib, a, b)
    q = torch.empty(M, I, dtype=torch.uint8, device="cuda")
    s = torch.empty(M, I // 128, dtype=torch.float32, device="cuda")
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    lib.fp8_grouped_gemm_blockscaled(len(sizes), cuda(torch.from_numpy(offs)), M, N, K, qa, qsa, qb, qsb,
                                     lib.MOE_EPI_SWIGLU_REQUANT | TILE_MODES[mode], q, s, st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    gu = oracle.grouped_gemm_blockscaled(offs, aq, sa, bq, sb)
    rq, rs, act = oracle.swiglu_requant(gu)
    gq, gs = np_(q), np_(s)
    # the scales follow the fp32 amax of act, which differs from float64 by rounding only
    assert np.max(np.abs(gs - rs) / rs) < 1e-4
    same = (gq == rq)
    assert same.mean() > 0.99
    deq_g = oracle.dequant_1x128(gq, gs)
    deq_r = oracle.dequant_1x128(rq, rs)
    step = np.abs(deq_r) * 2 ** -3 + np.repeat(rs, 128, 1) * 2 ** -9
    assert np.all(np.abs(deq_g - deq_r) <= step * 1.01)
    assert normwise(deq_g, deq_r) < TOL_NORMWISE * 10
    assert normwise(deq_g, act) < 0.05


@pytest.mark.parametrize("mode", list(TILE_MODES))
def test_bad_offsets_flagged(lib, mode):
    M, N, K = 64, 256, 128
    qa = torch.zeros(M, K, dtype=torch.uint8, device="cuda")
    qsa = torch.ones(M, 1, dtype=torch.float32, device="cuda")
    qb = torch.zeros(2, N, K, dtype=torch.uint8, device="cuda")
    qsb = torch.ones(2, 2, 1, dtype=torch.float32, device="cuda")
    C = torch.full((M, N), 3.0, dtype=torch.float32, device="cuda")
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    offs = torch.tensor([0, 40, 20], dtype=torch.int32, device="cuda")   # decreasing
    lib.fp8_grouped_gemm_blockscaled(2, offs, M, N, K, qa, qsa, qb, qsb, lib.MOE_EPI_F32 | TILE_MODES[mode], C,
                                     None, st)
    torch.cuda.synchronize()
    assert int(st.item()) & lib.MOE_FLAG_BAD_OFFSETS
    assert torch.all(C == 3.0)


@pytest.mark.parametrize("mode", list(TILE_MODES))
def test_dgrad_through_the_grouped_gemm(lib, mode):
    """Backward dgrad dX = dY . W per expert runs on the forward kernel with the
    weights quantised transposed: 128x128 block codes and scales transpose
    exactly, so B = W^T [K, N] with contraction over N reproduces the oracle's
    dgrad (promotion per 128 of N)."""
    from oracle.backward import dgrad_blockscaled
    sizes, N, K = [70, 0, 150], 256, 384            # forward Y [M, N] = X [M, K] W^T, W [N, K]
    G = len(sizes)
    M = sum(sizes)
    offs = np.concatenate([[0], np.cumsum(sizes)]).astype(np.int32)
    dy = synth.heavy_tailed(M, N, 41)
    w = synth.normal((G * N, K), 0.02, 42, dtype=torch.bfloat16).reshape(G, N, K)
    dyq, sdy = oracle.quant_1x128(dy.float().numpy())
    ref = np.zeros((M, K))
    wq_ref = []
    for g in range(G):
        wq, sw = oracle.quant_128x128(w[g].float().numpy())
        wq_ref.append((wq, sw))
        r0, r1 = offs[g], offs[g + 1]
        if r1 > r0:
            ref[r0:r1] = dgrad_blockscaled(dyq[r0:r1], sdy[r0:r1], wq, sw)
    qdy = torch.empty(M, N, dtype=torch.uint8, device="cuda")
    qsdy = torch.empty(M, N // 128, dtype=torch.float32, device="cuda")
    lib.fp8_quant_1x128(cuda(dy), qdy, qsdy)
    wt = cuda(w.transpose(1, 2))                          # [G, K, N]
    qwt = torch.empty(G, K, N, dtype=torch.uint8, device="cuda")
    swt = torch.empty(G, K // 128, N // 128, dtype=torch.float32, device="cuda")
    lib.fp8_quant_128x128(wt, qwt, swt)
    for g in range(G):                                    # transposed quantisation is exact
        assert np.array_equal(np_(qwt[g]), wq_ref[g][0].T) and np.array_equal(np_(swt[g]), wq_ref[g][1].T)
    dx = torch.zeros(M, K, dtype=torch.float32, device="cuda")
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    lib.fp8_grouped_gemm_blockscaled(G, cuda(torch.from_numpy(offs)), M, K, N, qdy, qsdy, qwt, swt,
                                     lib.MOE_EPI_F32 | TILE_MODES[mode], dx, None, st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    got = np_(dx)
    assert normwise(got, ref) < TOL_NORMWISE
    assert np.all(np.abs(got - ref) <= 1e-4 * np.abs(ref) + 1e-5 * np.abs(ref).max())
