"""GPU parity of the grouped FP8 block-scaled GEMM (tcgen05) against the float64
oracle, through the C ABI.  Operands are drawn by `synth` in bf16 and quantised
independently by each side (the quantisers agree bit for bit, see
test_gpu_kernels), so both sides multiply the same E4M3 codes and scales."""
import numpy as np
import pytest
import torch

import oracle
import synth
from tests._util import (TOL_NORMWISE, bf16_ulp, cuda, e4m3_boundary_distance, gemm_error_bound, normwise, np_,
                         swiglu_error_bound)

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
    # element-wise: within the fp32 accumulation bound of the promoted sum (plus
    # one bf16 rounding for the bf16 epilogue)
    mag = oracle.grouped_gemm_blockscaled(offs, aq & 0x7F, sa, bq & 0x7F, sb)[:used]
    tol = gemm_error_bound(mag, K // 128) + (bf16_ulp(r) if epi == "bf16" else 0)
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


SWIGLU_CASES = [([70, 0, 150], 256, 384), ([1], 128, 128), ([300] * 3, 512, 1024), ([50, 1100], 256, 256),
                ([257, 511, 3, 0, 129], 256, 256)]


def _swiglu_gpu(lib, sizes, I, K, mode, seed):
    N = 2 * I
    a, b, aq, sa, bq, sb, offs, M = _operands(sizes, N, K, seed=seed, heavy=False)
    qa, qsa, qb, qsb = _gpu_operands(lib, a, b)
    q = torch.empty(M, I, dtype=torch.uint8, device="cuda")
    s = torch.empty(M, I // 128, dtype=torch.float32, device="cuda")
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    goffs = cuda(torch.from_numpy(offs))
    lib.fp8_grouped_gemm_blockscaled(len(sizes), goffs, M, N, K, qa, qsa, qb, qsb,
                                     lib.MOE_EPI_SWIGLU_REQUANT | TILE_MODES[mode], q, s, st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    return (aq, sa, bq, sb, offs, M), (qa, qsa, qb, qsb, goffs), q, s


@pytest.mark.parametrize("sizes,I,K", SWIGLU_CASES)
@pytest.mark.parametrize("mode", list(TILE_MODES))
def test_grouped_gemm_swiglu_requant(lib, sizes, I, K, mode):
    """Fused SwiGLU + 1x128 requant against the oracle, to the bound its error
    analysis gives: the GPU's gate/up values differ from float64 by at most the
    fp32 accumulation bound of the promoted GEMM (gemm_error_bound), the act
    by that propagated through silu(g) u plus the kernel's __expf/__fdividef
    error (swiglu_error_bound), the tile scale by the act error of the tile's
    largest element, and the quotient act/scale by both plus 1.5 ulps of the
    reciprocal.  Every code whose oracle quotient lies farther than that from
    an E4M3 rounding boundary must be identical; the rest may be a neighbour."""
    (aq, sa, bq, sb, offs, M), _, q, s = _swiglu_gpu(lib, sizes, I, K, mode, 91 + I)
    gu = oracle.grouped_gemm_blockscaled(offs, aq, sa, bq, sb)
    mag = oracle.grouped_gemm_blockscaled(offs, aq & 0x7F, sa, bq & 0x7F, sb)
    eps = gemm_error_bound(mag, K // 128)
    rq, rs, act = oracle.swiglu_requant(gu)
    used = int(offs[-1])
    gq, gs = np_(q)[:used], np_(s)[:used]
    rq, rs, act, gu, eps = rq[:used], rs[:used], act[:used], gu[:used], eps[:used]
    dact = swiglu_error_bound(gu[:, :I], gu[:, I:], eps[:, :I], eps[:, I:])
    amax = np.abs(act).reshape(used, I // 128, 128).max(-1)
    damax = dact.reshape(used, I // 128, 128).max(-1)
    ds = damax / np.maximum(amax, 1e-300) + 2.0 ** -23          # relative scale bound
    assert np.all(np.abs(gs.astype(np.float64) - rs) <= rs * ds)
    t = act / np.repeat(rs.astype(np.float64), 128, 1)
    band = dact / np.repeat(rs.astype(np.float64), 128, 1) + np.abs(t) * (np.repeat(ds, 128, 1) + 2.0 ** -22)
    outside = e4m3_boundary_distance(t) > band
    same = gq == rq
    assert np.all(same[outside]), f"{int((~same & outside).sum())} codes differ away from a rounding boundary"
    deq_g = oracle.dequant_1x128(gq, gs)
    deq_r = oracle.dequant_1x128(rq, rs)
    step = np.abs(deq_r) * 2 ** -3 + np.repeat(rs, 128, 1) * 2 ** -9
    assert np.all(np.abs(deq_g - deq_r) <= step * (1 + 1e-6))          # the rest: neighbours
    print(f"identical codes {same.mean():.7f}, band {1 - outside.mean():.2e}")
    # the band is a worst case; codes actually differ only where the quotient
    # sits within a few fp32 ulps of a boundary (measured: >= 0.999995 identical)
    assert same.mean() > 0.9999
    assert normwise(deq_g, deq_r) < TOL_NORMWISE


@pytest.mark.parametrize("sizes,I,K", SWIGLU_CASES[:3])
def test_fused_requant_matches_division_rule(lib, sizes, I, K):
    """The fused epilogue requantises with the reciprocal of the tile scale; the
    stand-alone swiglu_requant divides (the quantisation rule).  Given the same
    fp32 gate/up values (the F32 epilogue of the same GEMM, whose promotion is
    the same code), scales agree bit for bit and codes differ only where the
    quotient lies within 2^-21 of an E4M3 rounding boundary.  Prints the
    measured mismatch rate."""
    (aq, sa, bq, sb, offs, M), (qa, qsa, qb, qsb, goffs), q, s = _swiglu_gpu(lib, sizes, I, K, "single", 91 + I)
    gu = torch.empty(M, 2 * I, dtype=torch.float32, device="cuda")
    lib.fp8_grouped_gemm_blockscaled(len(sizes), goffs, M, 2 * I, K, qa, qsa, qb, qsb,
                                     lib.MOE_EPI_F32 | TILE_MODES["single"], gu)
    qe = torch.empty(M, I, dtype=torch.uint8, device="cuda")
    se = torch.empty(M, I // 128, dtype=torch.float32, device="cuda")
    lib.swiglu_requant(gu, qe, se)
    torch.cuda.synchronize()
    used = int(offs[-1])
    assert torch.equal(s[:used], se[:used])
    diff = (np_(q) != np_(qe))[:used]
    rate = float(diff.mean())
    print(f"reciprocal vs division: {int(diff.sum())} of {diff.size} codes differ ({rate:.2e})")
    if diff.any():
        g = np_(gu)[:used].astype(np.float64)
        act32 = oracle.swiglu(g).astype(np.float32).astype(np.float64)   # near-boundary test only
        t = act32 / np.repeat(np_(se)[:used].astype(np.float64), 128, 1)
        near = e4m3_boundary_distance(t) <= np.abs(t) * 2.0 ** -21 + swiglu_error_bound(g[:, :I], g[:, I:], 0, 0) / \
            np.repeat(np_(se)[:used].astype(np.float64), 128, 1)
        assert np.all(near[diff])
    assert rate < 1e-4


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
