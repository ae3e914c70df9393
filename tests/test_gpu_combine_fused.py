"""GPU parity of the combine fused into the second grouped GEMM: each row's
bf16 value times its gate is added into its token's fp32 output row at the L2,
in no fixed order, and moe_combine_finish rounds the sums to bf16.

References: the plain grouped GEMM's bf16 rows combined by the float64 oracle
(the additions differ from that exact sum only by fp32 rounding, bounded by
the number of terms per output), and, for the layer, the materialised path."""
import numpy as np
import pytest
import torch

import oracle
import synth
from tests._util import TOL_NORMWISE, bf16_ulp, cuda, normwise, np_
from tests.test_gpu_gemm import _gpu_operands, _operands

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("sizes,N,K,T", [
    ([40, 0, 130, 1, 257], 256, 256, 100),     # empty and 1-row groups
    ([300, 300, 300, 300], 512, 384, 400),      # three rows per token on average
])
def test_combine_gemm(lib, sizes, N, K, T):
    a, b, aq, sa, bq, sb, offs, M = _operands(sizes, N, K, seed=31 + N, m_extra=2)
    qa, qsa, qb, qsb = _gpu_operands(lib, a, b)
    rng = np.random.default_rng(N + K)
    tok = rng.integers(0, T, M).astype(np.int32)
    gate = rng.uniform(0.05, 1.0, M).astype(np.float32)
    goffs = cuda(torch.from_numpy(offs))
    # plain GEMM rows (bf16), then the float64 combine of those rows
    C = torch.empty(M, N, dtype=torch.bfloat16, device="cuda")
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    lib.fp8_grouped_gemm_blockscaled(len(sizes), goffs, M, N, K, qa, qsa, qb, qsb, lib.MOE_EPI_BF16 | 0x100, C,
                                     None, st)
    acc = torch.zeros(T, N, dtype=torch.float32, device="cuda")
    lib.fp8_grouped_gemm_blockscaled_combine(len(sizes), goffs, M, N, K, qa, qsa, qb, qsb,
                                             cuda(torch.from_numpy(tok)), cuda(torch.from_numpy(gate)), acc, st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    used = int(offs[-1])
    y = np_(C).astype(np.float64)[:used]
    ref = np.zeros((T, N))
    mag = np.zeros((T, N))
    cnt = np.zeros(T)
    for m in range(used):
        ref[tok[m]] += np.float64(gate[m]) * y[m]
        mag[tok[m]] += np.abs(np.float64(gate[m]) * y[m])
        cnt[tok[m]] += 1
    got = np_(acc).astype(np.float64)
    # fp32: one rounding of each product and of each addition
    bound = (cnt[:, None] + 1) * 2.0 ** -24 * mag * 1.01 + 1e-30
    assert np.all(np.abs(got - ref) <= bound)


def test_combine_gemm_bad_token(lib):
    sizes, N, K, T = [50, 60], 256, 256, 20
    a, b, aq, sa, bq, sb, offs, M = _operands(sizes, N, K, seed=3)
    qa, qsa, qb, qsb = _gpu_operands(lib, a, b)
    tok = np.arange(M, dtype=np.int32) % T
    tok[7] = T                          # outside the output: flagged, skipped
    acc = torch.zeros(T, N, dtype=torch.float32, device="cuda")
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    lib.fp8_grouped_gemm_blockscaled_combine(len(sizes), cuda(torch.from_numpy(offs)), M, N, K, qa, qsa, qb, qsb,
                                             cuda(torch.from_numpy(tok)), cuda(torch.ones(M)), acc, st)
    torch.cuda.synchronize()
    assert int(st.item()) & lib.MOE_FLAG_BAD_INDEX
    assert bool(torch.isfinite(acc).all())


def test_combine_finish(lib):
    n = 8 * 1000
    acc = synth.normal((n,), 3.0, 44, device="cuda")
    acc[:8] = torch.tensor([1.0 + 2.0 ** -8, 1.0 + 3 * 2.0 ** -8, -0.0, float("inf"), 1e-40, 65504.0, 3.0e38, -2.5])
    keep = acc.clone()
    out = torch.empty(n, dtype=torch.bfloat16, device="cuda")
    f32 = torch.empty(n, dtype=torch.float32, device="cuda")
    lib.moe_combine_finish(acc, out, f32, True)
    torch.cuda.synchronize()
    assert np.array_equal(np_(out.float()), oracle.round_bf16(np_(keep).astype(np.float64)).astype(np.float32))
    assert torch.equal(f32, keep)
    assert not bool(acc.any())


@pytest.mark.parametrize("shape", [synth.MID, pytest.param(synth.DSV3, marks=pytest.mark.slow)])
def test_layer_fused_combine(lib, shape):
    """The layer with the combine inside W2: its fp32 output within the fp32
    rounding of the materialised path's fixed-order sum, the bf16 output equal
    to it except where that rounding crosses a bf16 rounding boundary (one ulp),
    and both against the float64 oracle as the layer tests require."""
    from tests.test_gpu_layer import build_layer
    dev = "cuda" if shape is synth.DSV3 else "cpu"
    lay_m, master, wr, b = build_layer(lib, shape, device=dev)
    lay_f = lib.MoELayer(shape.T, shape.H, shape.E, shape.K, shape.n_group, shape.topk_group, shape.I, shape.rho,
                         lay_m.w_router, b.cuda().contiguous(), lay_m.qw, fused_combine=True)
    x = cuda(synth.activations(shape.T, shape.H, synth.seed_of(shape, synth.X), shape.x_outlier_frac, device=dev))
    om = lay_m.forward(x, out_f32=True).clone()
    fm = lay_m.out_f32.clone()
    for rep in range(2):                         # the accumulator is re-armed by each forward
        of = lay_f.forward(x, out_f32=True).clone()
        ff = lay_f.out_f32.clone()
        torch.cuda.synchronize()
        assert int(lay_f.status.item()) == 0
        assert torch.equal(lay_f.topk_idx, lay_m.topk_idx)
        yk = np_(lay_m.yperm).astype(np.float64)
        w = np_(lay_m.topk_w).astype(np.float64)
        r = np_(lay_m.row_of).reshape(shape.T, shape.K)
        mag = np.abs(np_(lay_m.ysh).astype(np.float64))
        for k in range(shape.K):
            mag += np.abs(w[:, k:k + 1] * yk[r[:, k]])
        bound = 2 * (shape.K + 2) * 2.0 ** -24 * mag + 1e-30
        assert np.all(np.abs(np_(ff).astype(np.float64) - np_(fm).astype(np.float64)) <= bound)
        g, ref = np_(of).astype(np.float64), np_(om).astype(np.float64)
        # g = bf16(ff), ref = bf16(fm): half an ulp of each rounding plus |ff - fm|
        assert np.all(np.abs(g - ref) <= 0.5 * bf16_ulp(g) + 0.5 * bf16_ulp(ref) + bound)
        assert np.mean(g == ref) > 0.99
        assert normwise(g, ref) < TOL_NORMWISE
