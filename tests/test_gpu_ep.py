"""The expert-parallel layer on one GPU (one rank, no process group): with every
expert local, dispatch and combine reduce to permutations, and the output must be
bit-identical to the single-GPU layer's; the placement kernels against their
definition."""
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
                    layer.w_router, layer.e_bias, layer.qw)
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
