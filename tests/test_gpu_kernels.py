"""GPU parity of the memory-bound kernels through the C ABI against the oracle:
quantisers, router, selection, permutation, SwiGLU requant, combine, bias update."""
import numpy as np
import pytest
import torch

import oracle
import synth
from tests._util import (TOL_NORMWISE, bf16_ulp, cuda, e4m3_boundary_distance, normwise, np_, order_is_valid,
                         router_logit_tol, same_expert_sets, swiglu_error_bound)

pytestmark = pytest.mark.gpu


def _nan_eq(a, b):
    a = np.asarray(a)
    b = np.asarray(b)
    both = np.isnan(a) & np.isnan(b)
    return np.array_equal(np.where(both, 0, a), np.where(both, 0, b))


# ---------------------------------------------------------------- quant 1x128
@pytest.mark.parametrize("rows,cols,outl", [(1, 128, 0.0), (7, 384, 0.0), (300, 512, 0.01),
                                            (1031, 7168, 0.001), (4096, 7168, 0.001)])
def test_quant_1x128_bitexact(lib, rows, cols, outl):
    x = synth.activations(rows, cols, 11 + rows, outlier_frac=outl)
    q = torch.empty(rows, cols, dtype=torch.uint8, device="cuda")
    s = torch.empty(rows, cols // 128, dtype=torch.float32, device="cuda")
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    lib.fp8_quant_1x128(cuda(x), q, s, st)
    torch.cuda.synchronize()
    rq, rs = oracle.quant_1x128(x.float().numpy())
    assert np.array_equal(np_(q), rq)
    assert np.array_equal(np_(s), rs)
    assert int(st.item()) == 0


def test_quant_1x128_edge_tiles(lib):
    x = np.zeros((4, 512), dtype=np.float32)
    x[1, :128] = np.float32(896.0)                      # amax -> exactly 448 after scaling
    x[1, 5] = -3.0
    x[2, 130] = np.nan                                   # non-finite tile 1 of row 2
    x[3, 256:384] = np.linspace(-2 ** -120, 2 ** -120, 128)   # tiny values: subnormal scale
    x[3, 384:] = synth.activations(1, 128, 3).float().numpy() * 100
    xb = torch.from_numpy(x).to(torch.bfloat16)
    q = torch.empty(4, 512, dtype=torch.uint8, device="cuda")
    s = torch.empty(4, 4, dtype=torch.float32, device="cuda")
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    lib.fp8_quant_1x128(cuda(xb), q, s, st)
    torch.cuda.synchronize()
    rq, rs = oracle.quant_1x128(xb.float().numpy())
    assert np.array_equal(np_(q), rq)
    assert _nan_eq(np_(s), rs)
    assert int(st.item()) & lib.MOE_FLAG_NONFINITE
    assert np_(s)[0, 0] == 1.0 and not np_(q)[0].any()


def test_quant_128x128_bitexact(lib):
    w = synth.expert_weight(3 * 256, 384, 0.006, 5).reshape(3, 256, 384)
    q = torch.empty(3, 256, 384, dtype=torch.uint8, device="cuda")
    s = torch.empty(3, 2, 3, dtype=torch.float32, device="cuda")
    lib.fp8_quant_128x128(cuda(w), q, s)
    torch.cuda.synchronize()
    for b in range(3):
        rq, rs = oracle.quant_128x128(w[b].float().numpy())
        assert np.array_equal(np_(q[b]), rq)
        assert np.array_equal(np_(s[b]), rs)


# ---------------------------------------------------------------- routing
SEL_CASES = [  # T, E, K, n_group, topk_group, tie_frac
    (64, 16, 4, 4, 2, 0.0), (64, 16, 4, 4, 2, 0.4), (333, 256, 8, 8, 4, 0.05), (50, 64, 6, 8, 8, 0.2),
    (17, 32, 32, 1, 1, 0.0), (9, 96, 5, 32, 3, 0.1), (1, 256, 8, 8, 4, 0.0),
]


@pytest.mark.parametrize("T,E,K,ng,kg,ties", SEL_CASES)
def test_route_select_bitexact(lib, T, E, K, ng, kg, ties):
    s = synth.scores(T, E, 100 + T + E, tie_frac=ties)
    b = synth.expert_bias(E, 0.05, 7)
    d = lib.dims(T, 128, E, K, ng, kg, 128, 2.5)
    idx = torch.empty(T, K, dtype=torch.int32, device="cuda")
    w = torch.empty(T, K, dtype=torch.float32, device="cuda")
    lib.moe_route_select(d, cuda(s), cuda(b), idx, w)
    torch.cuda.synchronize()
    ridx, rw = oracle.select_experts(s.numpy(), b.numpy(), ng, kg, K, 2.5)
    assert np.array_equal(np_(idx), ridx)
    assert np.array_equal(np_(w), rw)


@pytest.mark.parametrize("shape", [synth.TINY, synth.MID])
def test_router_scores_close_to_float64(lib, shape):
    T, H, E = shape.T, shape.H, shape.E
    x = synth.activations(T, H, synth.seed_of(shape, synth.X), shape.x_outlier_frac)
    wr = synth.router_weights(E, H, shape.wr_std, synth.seed_of(shape, synth.WR))
    b = synth.expert_bias(E, shape.bias_range, synth.seed_of(shape, synth.BIAS))
    off = synth.zipf_offset(E, 0.05, 9)
    d = lib.dims(T, H, E, shape.K, shape.n_group, shape.topk_group, shape.I, shape.rho)
    idx = torch.empty(T, shape.K, dtype=torch.int32, device="cuda")
    w = torch.empty(T, shape.K, dtype=torch.float32, device="cuda")
    sc = torch.empty(T, E, dtype=torch.float32, device="cuda")
    ws = torch.empty(lib.workspace_size(d), dtype=torch.uint8, device="cuda")
    lib.moe_route(d, cuda(x), cuda(wr), cuda(b), cuda(off), idx, w, sc, ws)
    torch.cuda.synchronize()
    ref = oracle.router_scores(x.float().numpy(), wr.numpy(), off.numpy())
    # fp32 accumulation: |d logit| within the random-walk bound, ds = s (1 - s) d logit
    tol = router_logit_tol(x.float().numpy(), wr.numpy())[:, None] * ref * (1 - ref)
    assert np.all(np.abs(np_(sc) - ref) <= tol + 2 ** -24 * ref)


def _near_tie_tokens(s32, b32, ng, kg, K, tol):
    """Tokens whose selected set could change under an affinity perturbation of
    at most `tol` (absolute, per token or scalar): a gap below 2 tol (4 tol for
    the two-value group scores) at the group boundary (topk_group-th vs next
    group) or at the K-th expert among the kept groups' experts."""
    r = (s32 + b32).astype(np.float32).astype(np.float64)
    T, E = r.shape
    tol = np.broadcast_to(np.asarray(tol, dtype=np.float64), (T,))
    gs = E // ng
    srt = -np.sort(-r.reshape(T, ng, gs), axis=-1)
    gsc = srt[..., 0] + (srt[..., 1] if gs > 1 else 0)
    tie = np.zeros(T, dtype=bool)
    gorder = np.argsort(-gsc, axis=1, kind="stable")
    gsort = np.take_along_axis(gsc, gorder, axis=1)
    if kg < ng:
        tie |= (gsort[:, kg - 1] - gsort[:, kg]) <= 4 * tol + 1e-7
    keep = np.zeros((T, ng), dtype=bool)
    np.put_along_axis(keep, gorder[:, :kg], True, axis=1)
    masked = np.where(np.repeat(keep, gs, axis=1), r, -np.inf)
    rs = -np.sort(-masked, axis=1)
    if K < kg * gs:
        tie |= (rs[:, K - 1] - rs[:, K]) <= 2 * tol + 1e-7
    return tie


def routing_tol(x, w_router):
    """Per-token bound on |s_gpu - s| (s(1-s) <= 1/4 times the logit bound)."""
    return 0.25 * router_logit_tol(x, w_router)


def check_routing(gpu_idx, gpu_s, ref_idx, ref_s32, bias, ng, kg, K, tol, min_same=0.9):
    """Sets equal for every token without a near tie; the GPU's order valid on
    its own affinities; returns the mask of tokens with an identical table."""
    tie = _near_tie_tokens(ref_s32, bias, ng, kg, K, tol)
    sets = same_expert_sets(gpu_idx, ref_idx)
    bad = ~(sets | tie)
    assert not bad.any(), f"{int(bad.sum())} tokens select a different set without a near tie"
    if gpu_s is not None:
        assert order_is_valid(gpu_idx, gpu_s, bias).all()
    same = np.all(np.asarray(gpu_idx) == np.asarray(ref_idx), axis=1)
    assert same.mean() > min_same
    return same


@pytest.mark.parametrize("shape", [synth.TINY, synth.MID])
def test_route_end_to_end(lib, shape):
    T, H, E, K = shape.T, shape.H, shape.E, shape.K
    x = synth.activations(T, H, synth.seed_of(shape, synth.X), shape.x_outlier_frac)
    wr = synth.router_weights(E, H, shape.wr_std, synth.seed_of(shape, synth.WR))
    b = synth.expert_bias(E, shape.bias_range, synth.seed_of(shape, synth.BIAS))
    d = lib.dims(T, H, E, K, shape.n_group, shape.topk_group, shape.I, shape.rho)
    idx = torch.empty(T, K, dtype=torch.int32, device="cuda")
    w = torch.empty(T, K, dtype=torch.float32, device="cuda")
    ws = torch.empty(lib.workspace_size(d), dtype=torch.uint8, device="cuda")
    lib.moe_route(d, cuda(x), cuda(wr), cuda(b), None, idx, w, None, ws)
    torch.cuda.synchronize()
    s64 = oracle.router_scores(x.float().numpy(), wr.numpy())
    s32 = s64.astype(np.float32)
    ridx, rw = oracle.select_experts(s32, b.numpy(), shape.n_group, shape.topk_group, K, shape.rho)
    same = check_routing(np_(idx), None, ridx, s32, b.numpy(), shape.n_group, shape.topk_group, K,
                         routing_tol(x.float().numpy(), wr.numpy()))
    assert np.allclose(np_(w)[same], rw[same], rtol=1e-4, atol=0)


@pytest.mark.parametrize("shape", [synth.TINY, synth.MID])
def test_route_pieces_same_bits_as_route(lib, shape):
    """Routing with the router weights split once (moe_router_split +
    moe_route_pieces) gives the same bits as moe_route, which splits per call."""
    T, H, E, K = shape.T, shape.H, shape.E, shape.K
    x = cuda(synth.activations(T, H, synth.seed_of(shape, synth.X), shape.x_outlier_frac))
    wr = cuda(synth.router_weights(E, H, shape.wr_std, synth.seed_of(shape, synth.WR)))
    b = cuda(synth.expert_bias(E, shape.bias_range, synth.seed_of(shape, synth.BIAS)))
    d = lib.dims(T, H, E, K, shape.n_group, shape.topk_group, shape.I, shape.rho)
    ws = torch.empty(lib.workspace_size(d), dtype=torch.uint8, device="cuda")
    outs = []
    pieces = torch.empty(lib.moe_router_pieces_bytes(E, H) // 2, dtype=torch.bfloat16, device="cuda")
    lib.moe_router_split(wr, pieces)
    for use_pieces in (False, True):
        idx = torch.empty(T, K, dtype=torch.int32, device="cuda")
        w = torch.empty(T, K, dtype=torch.float32, device="cuda")
        sc = torch.empty(T, E, dtype=torch.float32, device="cuda")
        if use_pieces:
            lib.moe_route_pieces(d, x, pieces, b, None, idx, w, sc, ws)
        else:
            lib.moe_route(d, x, wr, b, None, idx, w, sc, ws)
        outs.append((idx, w, sc))
    torch.cuda.synchronize()
    for a, c in zip(*outs):
        assert torch.equal(a, c)
    # the pieces add up to W_r exactly
    p = pieces.reshape(3, E, H).double()
    assert torch.equal(p[0] + p[1] + p[2], wr.double())


def test_route_empty_batch(lib):
    d = lib.dims(0, 256, 16, 4, 4, 2, 128, 2.5)
    lib.moe_route(d, None, None, None, None, None, None)   # T == 0: no launch, OK


# ---------------------------------------------------------------- permutation
@pytest.mark.parametrize("T,E,K,skew", [(1, 16, 4, 0.0), (64, 16, 4, 0.0), (300, 32, 4, 3.0),
                                        (4096, 256, 8, 0.0), (1000, 256, 8, 6.0), (129, 8, 8, 0.0)])
def test_permute_bitexact(lib, T, E, K, skew):
    H = 256
    idx = synth.topk_indices(T, E, K, 40 + T, skew=skew)
    x = synth.activations(T, H, 41)
    xq, xs = oracle.quant_1x128(x.float().numpy())
    d = lib.dims(T, H, E, K, 1, 1, 128, 2.5)
    dev = dict(device="cuda")
    load = torch.empty(E, dtype=torch.int32, **dev)
    offs = torch.empty(E + 1, dtype=torch.int32, **dev)
    tok_of = torch.empty(T * K, dtype=torch.int32, **dev)
    row_of = torch.empty(T * K, dtype=torch.int32, **dev)
    aq = torch.empty(T * K, H, dtype=torch.uint8, **dev)
    as_ = torch.empty(T * K, H // 128, dtype=torch.float32, **dev)
    ws = torch.empty(lib.workspace_size(d), dtype=torch.uint8, **dev)
    st = torch.zeros(1, dtype=torch.int32, **dev)
    lib.moe_permute(d, cuda(idx), cuda(torch.from_numpy(xq)), cuda(torch.from_numpy(xs)), load, offs, tok_of,
                    row_of, aq, as_, ws, st)
    torch.cuda.synchronize()
    rl, ro, rt, rr = oracle.permute(idx.numpy(), E)
    assert np.array_equal(np_(load), rl)
    assert np.array_equal(np_(offs), ro)
    assert np.array_equal(np_(tok_of), rt)
    assert np.array_equal(np_(row_of), rr)
    assert np.array_equal(np_(aq), xq[rt])
    assert np.array_equal(np_(as_), xs[rt])
    assert int(st.item()) == 0


def test_permute_all_tokens_same_experts_and_bad_index(lib):
    T, E, K = 200, 16, 4
    idx = torch.arange(K, dtype=torch.int32).repeat(T, 1)
    idx[5, 2] = 99                      # out of range: flagged and skipped
    d = lib.dims(T, 128, E, K, 1, 1, 128, 2.5)
    dev = dict(device="cuda")
    load = torch.empty(E, dtype=torch.int32, **dev)
    offs = torch.empty(E + 1, dtype=torch.int32, **dev)
    tok_of = torch.full((T * K,), -7, dtype=torch.int32, **dev)
    row_of = torch.empty(T * K, dtype=torch.int32, **dev)
    ws = torch.empty(lib.workspace_size(d), dtype=torch.uint8, **dev)
    st = torch.zeros(1, dtype=torch.int32, **dev)
    lib.moe_permute(d, cuda(idx), None, None, load, offs, tok_of, row_of, None, None, ws, st)
    torch.cuda.synchronize()
    assert int(st.item()) & lib.MOE_FLAG_BAD_INDEX
    assert np_(row_of)[5 * K + 2] == -1
    assert list(np_(load)[:4]) == [T, T, T - 1, T] and not np_(load)[4:].any()
    assert np_(offs)[-1] == T * K - 1
    # expert 2's rows skip token 5 and keep ascending token order
    seg = np_(tok_of)[np_(offs)[2]:np_(offs)[3]]
    assert list(seg) == [t for t in range(T) if t != 5]


# ---------------------------------------------------------------- SwiGLU requant
def test_swiglu_requant_stand_alone(lib):
    """Stand-alone SwiGLU + requant (exact division) on a given fp32 gate|up
    matrix: the act differs from float64 only by the kernel's __expf/__fdividef
    error (swiglu_error_bound with exact inputs), the scale by the act error of
    the tile's largest element; every code whose quotient lies farther than
    that from an E4M3 rounding boundary is identical, the rest neighbours."""
    M, I = 333, 512
    gu = synth.normal((M, 2 * I), 3.0, 77)
    q = torch.empty(M, I, dtype=torch.uint8, device="cuda")
    s = torch.empty(M, I // 128, dtype=torch.float32, device="cuda")
    lib.swiglu_requant(cuda(gu), q, s)
    torch.cuda.synchronize()
    g64 = gu.numpy().astype(np.float64)
    rq, rs, act = oracle.swiglu_requant(g64)
    gq, gs = np_(q), np_(s)
    dact = swiglu_error_bound(g64[:, :I], g64[:, I:], 0.0, 0.0)
    amax = np.abs(act).reshape(M, I // 128, 128).max(-1)
    ds = dact.reshape(M, I // 128, 128).max(-1) / amax + 2.0 ** -23
    assert np.all(np.abs(gs.astype(np.float64) - rs) <= rs * ds)
    rs_e = np.repeat(rs.astype(np.float64), 128, 1)
    t = act / rs_e
    outside = e4m3_boundary_distance(t) > dact / rs_e + np.abs(t) * (np.repeat(ds, 128, 1) + 2.0 ** -23)
    same = gq == rq
    assert np.all(same[outside])
    deq_g = oracle.dequant_1x128(gq, gs)
    deq_r = oracle.dequant_1x128(rq, rs)
    step = np.abs(deq_r) * 2 ** -3 + np.repeat(rs, 128, 1) * 2 ** -9
    assert np.all(np.abs(deq_g - deq_r) <= step * (1 + 1e-6))
    print(f"identical codes {same.mean():.7f}, band {1 - outside.mean():.2e}")
    assert same.mean() > 0.9999
    assert normwise(deq_g, deq_r) < TOL_NORMWISE


# ---------------------------------------------------------------- combine
@pytest.mark.parametrize("T,H,E,K,shared", [(64, 256, 16, 4, True), (300, 512, 32, 4, False),
                                            (1000, 7168, 256, 8, True)])
def test_combine(lib, T, H, E, K, shared):
    idx = synth.topk_indices(T, E, K, 5)
    _, _, _, row_of = oracle.permute(idx.numpy(), E)
    yperm = synth.normal((T * K, H), 1.0, 6, dtype=torch.bfloat16)
    ysh = synth.normal((T, H), 1.0, 7, dtype=torch.bfloat16) if shared else None
    w = torch.rand(T, K, generator=synth.gen(8, "cpu"))
    d = lib.dims(T, H, E, K, 1, 1, 128, 2.5)
    out = torch.empty(T, H, dtype=torch.bfloat16, device="cuda")
    out32 = torch.empty(T, H, dtype=torch.float32, device="cuda")
    lib.moe_combine(d, cuda(yperm), cuda(torch.from_numpy(row_of)), cuda(w),
                    cuda(ysh) if shared else None, out, out32)
    torch.cuda.synchronize()
    ref = oracle.combine(yperm.float().numpy(), row_of, w.numpy(),
                         ysh.float().numpy() if shared else None)
    # fp32 accumulation error is bounded by the magnitudes summed, not the result
    mag = oracle.combine(np.abs(yperm.float().numpy()), row_of, np.abs(w.numpy()),
                         np.abs(ysh.float().numpy()) if shared else None)
    g32 = np_(out32)
    assert np.all(np.abs(g32 - ref) <= 4 * K * 2 ** -24 * mag)
    g16 = np_(out)
    r16 = oracle.round_bf16(ref)
    # the bf16 store may flip at a rounding boundary: one bf16 step at most
    assert np.all(np.abs(g16 - r16) <= bf16_ulp(r16) + 4 * K * 2 ** -24 * mag)
    assert normwise(g16, r16) < TOL_NORMWISE


# ---------------------------------------------------------------- bias update
def test_bias_update_bitexact(lib):
    E, T, K = 256, 4096, 8
    load = synth.topk_indices(T, E, K, 3, skew=2.0)
    lv = np.bincount(load.numpy().ravel(), minlength=E).astype(np.int32)
    lv[:5] = T * K // E                 # exactly average: unchanged
    b = synth.expert_bias(E, 0.01, 4)
    bg = cuda(b)
    lib.moe_bias_update(E, T, K, 0.001, cuda(torch.from_numpy(lv)), bg)
    torch.cuda.synchronize()
    ref = oracle.bias_update(b.numpy(), lv, T, K, 0.001)
    assert np.array_equal(np_(bg), ref)


# ---------------------------------------------------------------- balance statistics
@pytest.mark.parametrize("T,E,K,S", [(64, 16, 4, 16), (4096, 256, 8, 4096), (300, 32, 4, 100), (4096, 256, 8, 512)])
def test_balance_stats(lib, T, E, K, S):
    s = synth.scores(T, E, 61 + T)
    idx = synth.topk_indices(T, E, K, 62 + T, skew=1.5)
    load = np.bincount(idx.numpy().ravel(), minlength=E).astype(np.int32)
    d = lib.dims(T, 128, E, K, 1, 1, 128, 2.5)
    loss = torch.empty(T // S, dtype=torch.float64, device="cuda")
    ent = torch.empty(1, dtype=torch.float64, device="cuda")
    lib.moe_balance_stats(d, cuda(s), cuda(idx), cuda(torch.from_numpy(load)), S, 0.001, loss, ent)
    torch.cuda.synchronize()
    ref = oracle.seq_balance_loss(s.numpy(), idx.numpy(), S, 0.001)
    assert np.allclose(np_(loss), ref, rtol=1e-12, atol=0)
    assert abs(float(ent.item()) - oracle.load_entropy(load)) <= 1e-12 * oracle.load_entropy(load)
