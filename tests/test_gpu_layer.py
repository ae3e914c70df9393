"""End-to-end layer parity on the GPU (all kernels chained through the C ABI)
against the float64 oracle: full parity on small shapes; at the DeepSeek-V3
shape (T=4096, H=7168, 256+1 experts, top-8, I=2048) and the decode shape
(T=128), in the launch configuration bench.py times, whole expert segments,
shared-expert rows and 64 sampled tokens."""
import numpy as np
import pytest
import torch

import oracle
import synth
from tests import _oracle_pool
from tests._util import TOL_NORMWISE, bf16_ulp, cuda, normwise, np_
from tests.test_gpu_kernels import check_routing, routing_tol

pytestmark = pytest.mark.gpu


def build_layer(lib, shape, device="cuda", T=None, offset=None, gather=False):
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
                         router_offset=None if offset is None else offset.cuda(), gather=gather)
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


def _segment_experts(load, n_top: int = 4) -> list:
    """Experts whose whole output segments are compared: the n_top most loaded
    (several M tiles), the most loaded of the rest whose load is not a multiple
    of 128 (a ragged last M tile) and the least loaded non-empty one."""
    load = np.asarray(load)
    order = [int(e) for e in np.argsort(-load, kind="stable") if load[e] > 0]
    pick = order[:n_top]
    ragged = [e for e in order if load[e] % 128 != 0 and e not in pick]
    pick += ragged[:1]
    rest = [e for e in order[::-1] if e not in pick]
    pick += rest[:1]
    return pick


def _index_of(sorted_tokens, t) -> int:
    i = int(np.searchsorted(sorted_tokens, t))
    assert sorted_tokens[i] == t
    return i


def check_layer_against_oracle(layer, shape, x, wr, b, n_tokens: int, seed: int, offset=None,
                               segments: bool = True, n_shared_rows: int = 256, out=None):
    """Full-size parity of one forward already run on `layer` with input x:
    routing of every token, the expert loads and offsets, the quantised input,
    whole expert segments of yperm (segments=True), n_shared_rows rows of the
    shared expert and n_tokens sampled tokens of the output, all against the
    float64 oracle (expert FFNs evaluated in a process pool)."""
    T, E, K = x.shape[0], shape.E, shape.K
    xh = x.float().cpu().numpy()
    wrh, bh = wr.cpu().numpy(), np.asarray(b.cpu().numpy() if hasattr(b, "cpu") else b)
    offh = None if offset is None else offset.cpu().numpy()
    s32 = oracle.router_scores(xh, wrh, offh).astype(np.float32)
    ridx, rw = oracle.select_experts(s32, bh, shape.n_group, shape.topk_group, K, shape.rho)
    gidx = np_(layer.topk_idx)
    same = check_routing(gidx, None, ridx, s32, bh, shape.n_group, shape.topk_group, K,
                         routing_tol(xh, wrh), min_same=0.97)
    # gates from the GPU's fp32 affinities (a few ulps from the oracle's)
    assert np.allclose(np_(layer.topk_w)[same], rw[same], rtol=1e-4, atol=0)
    load = np_(layer.load)
    assert load.sum() == T * K
    assert np.array_equal(np_(layer.offsets), np.concatenate([[0], np.cumsum(load)]))
    xq, xs = oracle.quant_1x128(xh)
    assert np.array_equal(np_(layer.xq), xq) and np.array_equal(np_(layer.xs), xs)
    rload, roffs, rtok, _ = oracle.permute(ridx, E)
    if same.all():
        assert np.array_equal(load, rload)
        assert np.array_equal(np_(layer.tok_of), rtok)
    rng = np.random.default_rng(seed)
    seg = _segment_experts(rload) if segments else []
    pick = np.sort(rng.choice(np.where(same)[0], size=min(n_tokens, int(same.sum())), replace=False))
    sh_rows = np.sort(rng.choice(T, size=min(n_shared_rows, T), replace=False))
    toks = {e: set(int(t) for t in rtok[roffs[e]:roffs[e + 1]]) for e in seg}
    for t in pick:
        for k in range(K):
            toks.setdefault(int(ridx[t, k]), set()).add(int(t))
    toks[-1] = set(int(t) for t in sh_rows) | set(int(t) for t in pick)
    toks = {e: np.array(sorted(v), dtype=np.int64) for e, v in toks.items()}
    ys = _oracle_pool.expert_outputs(shape, {e: (xq[v], xs[v]) for e, v in toks.items()},
                                     device=str(x.device.type))
    grow = np_(layer.row_of).reshape(T, K)
    ulp_frac = lambda g, r: float(np.mean(np.abs(g - r) <= bf16_ulp(r)))
    # whole expert segments (rows of tokens whose routing is identical)
    for e in seg:
        st = [int(t) for t in toks[e] if same[t]]
        rows = [int(grow[t, int(np.where(gidx[t] == e)[0][0])]) for t in st]
        g = np_(layer.yperm[torch.as_tensor(rows, device=layer.yperm.device)])
        r = ys[e][[_index_of(toks[e], t) for t in st]]
        assert normwise(g, r) < TOL_NORMWISE, f"expert {e} (load {rload[e]})"
        assert ulp_frac(g, r) > 0.99, f"expert {e} (load {rload[e]})"
    # shared expert rows (both column chunks of its tiles)
    g = np_(layer.ysh[torch.as_tensor(sh_rows, device=layer.ysh.device)])
    r = ys[-1][[_index_of(toks[-1], t) for t in sh_rows]]
    assert normwise(g, r) < TOL_NORMWISE
    assert ulp_frac(g, r) > 0.99
    # sampled tokens of the output: the oracle's combine of the oracle's expert rows
    yk = np.stack([np.stack([ys[int(ridx[t, k])][_index_of(toks[int(ridx[t, k])], t)] for k in range(K)])
                   for t in pick]).reshape(len(pick) * K, -1)
    ysh = ys[-1][[_index_of(toks[-1], t) for t in pick]]
    ref = oracle.round_bf16(oracle.combine(yk, np.arange(len(pick) * K), rw[pick], ysh))
    got = np_((layer.out if out is None else out)[torch.as_tensor(pick, device=layer.out.device)])
    assert normwise(got, ref) < TOL_NORMWISE
    assert ulp_frac(got, ref) > 0.99
    return same, pick


@pytest.mark.slow
@pytest.mark.parametrize("shape", [synth.DSV3, synth.DECODE])
def test_layer_full_size(lib, shape):
    """The bench's workloads (DeepSeek-V3 T=4096 and decode T=128) in the launch
    configuration bench.py times: whole segments of the four most loaded
    experts, of a ragged one and of the least loaded one, 256 rows of the
    shared expert and 64 sampled tokens of the output."""
    layer, master, wr, b = build_layer(lib, shape, device="cuda")
    x = synth.activations(shape.T, shape.H, synth.seed_of(shape, synth.X), shape.x_outlier_frac, device="cuda")
    layer.forward(x)
    torch.cuda.synchronize()
    assert int(layer.status.item()) == 0
    check_layer_against_oracle(layer, shape, x, wr, b, n_tokens=64, seed=0)


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


@pytest.mark.parametrize("shape", [synth.TINY, synth.MID, pytest.param(synth.DSV3, marks=pytest.mark.slow)])
def test_layer_gather_equals_materialised(lib, shape):
    """The forward whose W13 gathers its A rows through tok_of and the default
    forward over the materialised permuted copy give the same bits at every
    stage: the gather changes where the GEMM reads a row, not its arithmetic."""
    dev = "cuda" if shape is synth.DSV3 else "cpu"
    lay_g, master, wr, b = build_layer(lib, shape, device=dev, gather=True)
    lay_m = lib.MoELayer(shape.T, shape.H, shape.E, shape.K, shape.n_group, shape.topk_group, shape.I, shape.rho,
                         lay_g.w_router, b.cuda().contiguous(), lay_g.qw, gather=False)
    assert lay_g.aq is None and lay_m.aq is not None
    x = synth.activations(shape.T, shape.H, synth.seed_of(shape, synth.X), shape.x_outlier_frac, device=dev)
    x = cuda(x)
    og = lay_g.forward(x).clone()
    om = lay_m.forward(x).clone()
    torch.cuda.synchronize()
    assert int(lay_g.status.item()) == 0 and int(lay_m.status.item()) == 0
    for name in ("topk_idx", "load", "offsets", "tok_of", "row_of", "xq", "xs", "actq", "acts", "yperm"):
        assert torch.equal(getattr(lay_g, name), getattr(lay_m, name)), name
    assert torch.equal(og, om)


def test_layer_cuda_graph_replay(lib):
    """A captured forward + bias update replays the same kernels: same output
    bits as the eager forward, on new input written into the captured buffer,
    and the same bias update."""
    shape = synth.MID
    layer, master, wr, b = build_layer(lib, shape, device="cpu")
    xs = [cuda(synth.activations(shape.T, shape.H, 100 + i, shape.x_outlier_frac)) for i in range(2)]
    eager, bias_eager = [], []
    for x in xs:
        bb = layer.e_bias.clone()
        eager.append(layer.forward(x).clone())
        layer.bias_update(0.001, bias=bb)
        bias_eager.append(bb)
    x_static = xs[0].clone()
    b_graph = layer.e_bias.clone()
    graph = layer.capture_graph(x_static, gamma=0.001, bias=b_graph)
    for i, x in enumerate(xs):
        x_static.copy_(x)
        b_graph.copy_(layer.e_bias)
        graph.replay()
        torch.cuda.synchronize()
        assert torch.equal(layer.out, eager[i])
        assert torch.equal(b_graph, bias_eager[i])
    assert int(layer.status.item()) == 0


@pytest.mark.parametrize("shape", [synth.MID, pytest.param(synth.DSV3, marks=pytest.mark.slow)])
def test_layer_one_call_forward_and_host_runner(lib, shape):
    """moe_layer_forward (the whole forward and the bias update behind one C
    call) gives the Python-chained forward's bits; moe_layer_run_host on three
    host batches gives each batch's forward output in its host buffer."""
    dev = "cuda" if shape is synth.DSV3 else "cpu"
    layer, master, wr, b = build_layer(lib, shape, device=dev)
    xs = [synth.activations(shape.T, shape.H, 200 + i, shape.x_outlier_frac, device=dev) for i in range(3)]
    ref, ref_b = [], []
    for x in xs:
        bb = layer.e_bias.clone()
        ref.append(layer.forward(cuda(x)).clone())
        layer.bias_update(0.001, bias=bb)
        ref_b.append(bb)
    torch.cuda.synchronize()
    # one call on the device
    b1 = layer.e_bias.clone()
    out1 = torch.empty_like(ref[0])
    layer.forward_native(cuda(xs[0]), out=out1, bias_out=b1, gamma=0.001)
    torch.cuda.synchronize()
    assert int(layer.status.item()) == 0
    assert torch.equal(out1, ref[0]) and torch.equal(b1, ref_b[0])
    # host batches: uploads, forwards and downloads overlapped, every output in place
    x_host = [x.cpu().pin_memory() for x in xs]
    out_host = [torch.full((shape.T, shape.H), float("nan"), dtype=torch.bfloat16).pin_memory() for _ in xs]
    x_dev = [torch.empty_like(ref[0]) for _ in range(2)]
    out_dev = [torch.empty_like(ref[0]) for _ in range(2)]
    layer.run_host(x_host, out_host, x_dev, out_dev)
    # a second call right behind the first, on the same device buffers: its
    # uploads wait for the first call's forwards
    out_host2 = [torch.full_like(o, float("nan")).pin_memory() for o in out_host]
    layer.run_host(x_host[::-1], out_host2, x_dev, out_dev)
    torch.cuda.synchronize()
    for i in range(3):
        assert torch.equal(out_host[i], ref[i].cpu()), f"batch {i}"
        assert torch.equal(out_host2[i], ref[2 - i].cpu()), f"second call, batch {i}"
