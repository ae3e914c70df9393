"""End-to-end layer parity on the GPU (all kernels chained through the C ABI)
against the float64 oracle: full parity on small shapes, sampled tokens at the
DeepSeek-V3 shape (T=4096, H=7168, 256+1 experts, top-8, I=2048) and the
decode shape (T=128) in the launch configuration bench.py times."""
import numpy as np
import pytest
import torch

import oracle
import synth
from tests._util import TOL_NORMWISE, bf16_ulp, cuda, normwise, np_
from tests.test_gpu_kernels import check_routing, routing_tol

pytestmark = pytest.mark.gpu


def build_layer(lib, shape, device="cuda", T=None, offset=None):
    """Layer with synth weights drawn on `device` (per expert, regenerable)."""
    T = shape.T if T is None else T
    H, E, I = shape.H, shape.E, shape.I

    def master(kind, e):
        tid = (synth.SH13 if kind == "w13" else synth.SH2) if e < 0 else (synth.W13 if kind == "w13" else synth.W2)
        rows, cols = (2 * I, H) if kind == "w13" else (H, I)
        return synth.expert_weight(rows, cols, shape.w_std, synth.seed_of(shape, tid, max(e, 0)), device=device)

    qw = lib.QuantWeights.from_master(master, E, H, I, device="cuda")
    wr = synth.router_weights(E, H, shape.wr_std, synth.seed_of(shape, synth.WR), device=device)
    b = synth.expert_bias(E, shape.bias_range, synth.seed_of(shape, synth.BIAS), device=device)
    layer = lib.MoELayer(T, H, E, shape.K, shape.n_group, shape.topk_group, I, shape.rho,
                         wr.cuda().contiguous(), b.cuda().contiguous(), qw,
                         router_offset=None if offset is None else offset.cuda())
    return layer, master, wr, b


def _oracle_weights(master):
    def host_master(kind, e):
        return master(kind, e).float().cpu().numpy()
    return oracle.LayerWeights(host_master)


@pytest.mark.parametrize("shape", [synth.TINY, synth.MID])
def test_layer_full_parity(lib, shape):
    layer, master, wr, b = build_layer(lib, shape, device="cpu")
    x = synth.activations(shape.T, shape.H, synth.seed_of(shape, synth.X), shape.x_outlier_frac)
    out = layer.forward(cuda(x), out_f32=True)
    torch.cuda.synchronize()
    assert int(layer.status.item()) == 0
    ref = oracle.moe_forward(x.float().numpy(), wr.numpy(), b.numpy(), _oracle_weights(master),
                             shape.n_group, shape.topk_group, shape.K, shape.rho)
    same = check_routing(np_(layer.topk_idx), np_(layer.scores), ref["idx"], ref["s32"], b.numpy(), shape.n_group,
                         shape.topk_group, shape.K, routing_tol(x.float().numpy(), wr.numpy()))
    if same.all():
        assert np.array_equal(np_(layer.load), ref["load"])
        assert np.array_equal(np_(layer.offsets), ref["offsets"])
        assert np.array_equal(np_(layer.tok_of), ref["tok_of"])
    assert np.array_equal(np_(layer.xq), ref["xq"]) and np.array_equal(np_(layer.xs), ref["xs"])
    g = np_(out)[same]
    r = ref["out"][same]
    assert normwise(g, r) < TOL_NORMWISE
    assert normwise(np_(layer.out_f32)[same], ref["out64"][same]) < TOL_NORMWISE
    assert normwise(np_(layer.ysh), ref["ysh"]) < TOL_NORMWISE


def _sampled_parity(lib, shape, T, n_samples, seed):
    layer, master, wr, b = build_layer(lib, shape, device="cuda", T=T)
    x = synth.activations(T, shape.H, synth.seed_of(shape, synth.X), shape.x_outlier_frac, device="cuda")
    out = layer.forward(x)
    torch.cuda.synchronize()
    assert int(layer.status.item()) == 0
    xh = x.float().cpu().numpy()
    # routing of every token by the oracle (float64 router, fp32 decisions)
    s32 = oracle.router_scores(xh, wr.cpu().numpy()).astype(np.float32)
    ridx, rw = oracle.select_experts(s32, b.cpu().numpy(), shape.n_group, shape.topk_group, shape.K, shape.rho)
    same = check_routing(np_(layer.topk_idx), np_(layer.scores), ridx, s32, b.cpu().numpy(), shape.n_group,
                         shape.topk_group, shape.K, routing_tol(xh, wr.cpu().numpy()), min_same=0.97)
    # invariants that hold at any size
    load = np_(layer.load)
    assert load.sum() == T * shape.K
    assert np.array_equal(np_(layer.offsets), np.concatenate([[0], np.cumsum(load)]))
    # sampled tokens, one by one (rows of every step are independent)
    rng = np.random.default_rng(seed)
    cand = np.where(same)[0]
    pick = np.sort(rng.choice(cand, size=n_samples, replace=False))
    W = _oracle_weights(master)
    ref = oracle.moe_forward_tokens(xh[pick], wr.cpu().numpy(), b.cpu().numpy(), W, shape.n_group,
                                    shape.topk_group, shape.K, shape.rho)
    assert np.array_equal(ref["idx"], np_(layer.topk_idx)[pick])
    g = np_(out)[pick]
    assert normwise(g, ref["out"]) < TOL_NORMWISE
    assert np.mean(np.abs(g - ref["out"]) <= bf16_ulp(ref["out"])) > 0.99


@pytest.mark.slow
def test_layer_dsv3_sampled_tokens(lib):
    _sampled_parity(lib, synth.DSV3, synth.DSV3.T, 2, 0)


@pytest.mark.slow
def test_layer_decode_sampled_tokens(lib):
    _sampled_parity(lib, synth.DECODE, synth.DECODE.T, 2, 1)


def test_layer_single_token(lib):
    shape = synth.MID
    layer, master, wr, b = build_layer(lib, shape, device="cpu", T=1)
    x = synth.activations(1, shape.H, 5)
    out = layer.forward(cuda(x))
    torch.cuda.synchronize()
    ref = oracle.moe_forward_tokens(x.float().numpy(), wr.numpy(), b.numpy(), _oracle_weights(master),
                                    shape.n_group, shape.topk_group, shape.K, shape.rho)
    assert np.array_equal(np_(layer.topk_idx), ref["idx"])
    assert normwise(np_(out), ref["out"]) < TOL_NORMWISE


def test_layer_caller_owned_output(lib):
    """forward(out=buf) writes the same bits into the caller's buffer."""
    shape = synth.TINY
    layer, master, wr, b = build_layer(lib, shape, device="cpu")
    x = cuda(synth.activations(shape.T, shape.H, synth.seed_of(shape, synth.X), shape.x_outlier_frac))
    ref = layer.forward(x).clone()
    buf = torch.full_like(ref, float("nan"))
    got = layer.forward(x, out=buf)
    torch.cuda.synchronize()
    assert got.data_ptr() == buf.data_ptr()
    assert torch.equal(buf, ref)
    with pytest.raises(ValueError):
        layer.forward(x, out=torch.empty(shape.T, shape.H, dtype=torch.float32, device="cuda"))
