"""The expert-parallel layer on one GPU (one rank, no process group): with every
expert local, per-slot dispatch and combine reduce to permutations and the output
must be bit-identical to the single-GPU layer's; node-limited dispatch must equal
the oracle's per-rank combine of the layer's expert rows; the placement and plan
kernels against their definitions."""
import numpy as np
import pytest
import torch

import synth
from tests._util import cuda, np_
from tests.test_gpu_layer import build_layer

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("shape", [synth.TINY, synth.MID])
def test_ep_layer_one_rank_same_bits_as_layer(lib, shape):
    from sparse_moe_layer_group_b200.ep import EPMoELayer
    layer, master, wr, b = build_layer(lib, shape, device="cpu")
    ep = EPMoELayer(shape.T, shape.H, shape.E, shape.K, shape.n_group, shape.topk_group, shape.I, shape.rho,
                    layer.w_router, layer.e_bias, layer.qw, dedupe=False, placement="cyclic")
    x = cuda(synth.activations(shape.T, shape.H, synth.seed_of(shape, synth.X), shape.x_outlier_frac))
    ref = layer.forward(x).clone()
    got = ep.forward(x)
    torch.cuda.synchronize()
    assert int(ep.status.item()) == 0
    assert torch.equal(got, ref)
    assert torch.equal(ep.topk_idx, layer.topk_idx)
    # the bias update from the (here single-rank) global loads: same bits as the layer's
    b_ep, b_layer = layer.e_bias.clone(), layer.e_bias.clone()
    ep.bias_update(0.001, bias=b_ep)
    layer.bias_update(0.001, bias=b_layer)
    torch.cuda.synchronize()
    assert torch.equal(ep.load_all, layer.load)
    assert torch.equal(b_ep, b_layer)


@pytest.mark.parametrize("shape", [synth.TINY, synth.MID])
def test_ep_layer_one_rank_node_limited(lib, shape):
    """Node-limited dispatch on one rank: every token sends one row carrying its
    K slots, the rank returns their gated sum in bf16, and the output is the
    oracle's combine_by_rank of the single-GPU layer's expert rows (fp32 on the
    GPU, float64 in the oracle: within one bf16 ulp)."""
    import oracle
    from sparse_moe_layer_group_b200.ep import EPMoELayer
    from tests._util import bf16_ulp, normwise, TOL_NORMWISE
    layer, master, wr, b = build_layer(lib, shape, device="cpu")
    ep = EPMoELayer(shape.T, shape.H, shape.E, shape.K, shape.n_group, shape.topk_group, shape.I, shape.rho,
                    layer.w_router, layer.e_bias, layer.qw, dedupe=True, placement="block")
    x = cuda(synth.activations(shape.T, shape.H, synth.seed_of(shape, synth.X), shape.x_outlier_frac))
    layer.forward(x)
    got = ep.forward(x)
    torch.cuda.synchronize()
    assert int(ep.status.item()) == 0
    assert torch.equal(ep.topk_idx, layer.topk_idx)
    assert int(ep.send_load.sum()) == shape.T            # one row per token
    T, K = shape.T, shape.K
    ref = oracle.round_bf16(oracle.combine_by_rank(np_(layer.yperm).astype(np.float64), np_(layer.row_of),
                                                   np_(layer.topk_w), np.zeros((T, K), dtype=np.int64),
                                                   np_(layer.ysh).astype(np.float64)))
    g = np_(got).astype(np.float64)
    assert normwise(g, ref) < TOL_NORMWISE
    assert np.mean(np.abs(g - ref) <= bf16_ulp(ref)) > 0.999


def test_ep_plan_and_scatter_rows(lib):
    """moe_ep_plan against its definition (both placements, repeated ranks, a bad
    index) and moe_ep_scatter_rows against a row scatter."""
    T, E, K, world = 300, 64, 8, 8
    idx = synth.topk_indices(T, E, K, 9).contiguous()
    idx[7, 3] = 99                                            # out of range: flagged, not sent
    w = torch.rand(T, K, generator=synth.gen(10, "cpu"))
    for placement in (lib.MOE_EP_CYCLIC, lib.MOE_EP_BLOCK):
        dest = torch.empty(T * K, dtype=torch.int32, device="cuda")
        mid = torch.empty(T * K, K, dtype=torch.int32, device="cuda")
        mw = torch.empty(T * K, K, dtype=torch.float32, device="cuda")
        st = torch.zeros(1, dtype=torch.int32, device="cuda")
        lib.abi.moe_ep_plan(cuda(idx), cuda(w), E, world, placement, dest, mid, mw, st)
        torch.cuda.synchronize()
        assert int(st.item()) & lib.MOE_FLAG_BAD_INDEX
        e = idx.numpy().astype(np.int64)
        ok = (e >= 0) & (e < E)
        El = E // world
        rk = np.where(ok, e // El if placement == lib.MOE_EP_BLOCK else e % world, -1)
        lk = np.where(ok, e % El if placement == lib.MOE_EP_BLOCK else e // world, -1)
        want_d = np.full(T * K, -1)
        want_m = np.full((T * K, K), -1)
        want_w = np.zeros((T * K, K), dtype=np.float32)
        for t in range(T):
            for k in range(K):
                if rk[t, k] < 0 or rk[t, k] in rk[t, :k]:
                    continue
                want_d[t * K + k] = rk[t, k]
                on = rk[t] == rk[t, k]
                want_m[t * K + k, on] = lk[t, on]
                want_w[t * K + k, on] = w.numpy()[t, on]
        assert np.array_equal(np_(dest), want_d)
        assert np.array_equal(np_(mid), want_m)
        assert np.array_equal(np_(mw), want_w)
    # row scatter: 5 int32 per row into a permutation's order, one row skipped
    n, width = 1000, 5
    vals = torch.randint(-1000, 1000, (n, width), dtype=torch.int32, generator=synth.gen(11, "cpu"))
    perm = torch.randperm(n, generator=synth.gen(12, "cpu")).to(torch.int32)
    perm[3] = -1
    out = torch.full((n, width), -9, dtype=torch.int32, device="cuda")
    lib.abi.moe_ep_scatter_rows(cuda(perm), cuda(vals), out)
    torch.cuda.synchronize()
    want = np.full((n, width), -9)
    p = perm.numpy()
    want[p[p >= 0]] = vals.numpy()[p >= 0]
    assert np.array_equal(np_(out), want)


def test_ep_split_and_scatter(lib):
    n, E, world = 1000, 256, 8
    idx = synth.topk_indices(125, E, 8, 3).reshape(-1).contiguous()
    idx[17] = 300                                            # out of range: flagged, -1
    dest = torch.empty(n, dtype=torch.int32, device="cuda")
    loc = torch.empty(n, dtype=torch.int32, device="cuda")
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    lib.moe_ep_split(cuda(idx), E, world, dest, loc, st)
    perm = torch.randperm(n, generator=synth.gen(4, "cpu")).to(torch.int32)
    perm[5] = -1                                              # skipped entry
    out = torch.full((n,), -9, dtype=torch.int32, device="cuda")
    lib.moe_ep_scatter(cuda(perm), cuda(torch.arange(n, dtype=torch.int32)), out)
    torch.cuda.synchronize()
    e = idx.numpy().astype(np.int64)
    ok = (e >= 0) & (e < E)
    assert int(st.item()) & lib.MOE_FLAG_BAD_INDEX
    assert np.array_equal(np_(dest)[ok], e[ok] % world) and np.array_equal(np_(loc)[ok], e[ok] // world)
    assert np_(dest)[17] == -1 and np_(loc)[17] == -1
    want = np.full(n, -9)
    p = perm.numpy()
    want[p[p >= 0]] = np.arange(n)[p >= 0]
    assert np.array_equal(np_(out), want)
