"""Pins of the oracle's permutation, combine, promoted GEMM, SwiGLU and layer."""
import numpy as np
import pytest
import torch

import oracle
import synth


def test_permute_invariants_and_bruteforce():
    idx = synth.topk_indices(50, 12, 3, 0, skew=2.0).numpy()
    load, offs, tok_of, row_of = oracle.permute(idx, 12)
    T, K = idx.shape
    assert load.sum() == T * K and offs[0] == 0 and offs[-1] == T * K
    assert np.all(np.diff(offs) == load) and np.all(np.diff(offs) >= 0)
    assert np.array_equal(load, np.bincount(idx.ravel(), minlength=12))
    # every (t,k) appears exactly once
    assert sorted(row_of.tolist()) == list(range(T * K))
    # unpermute(permute) is the identity on token ids
    assert np.array_equal(oracle.unpermute_rows(tok_of, row_of, T, K),
                          np.repeat(np.arange(T)[:, None], K, 1))
    # brute force: numpy's stable argsort of the expert ids in (t,k) order
    order = np.argsort(idx.ravel(), kind="stable")
    assert np.array_equal(tok_of, order // K)
    for e in range(12):
        seg = tok_of[offs[e]:offs[e + 1]]
        assert np.all(np.diff(seg) > 0)                     # ascending tokens
        assert np.all(idx[seg].__eq__(e).any(1))


def test_permute_empty_and_degenerate():
    load, offs, tok_of, row_of = oracle.permute(np.zeros((0, 4), np.int32), 8)
    assert load.sum() == 0 and list(offs) == [0] * 9 and tok_of.size == 0
    idx = np.tile(np.arange(4, dtype=np.int32), (7, 1))     # every token -> experts 0..3
    load, offs, tok_of, _ = oracle.permute(idx, 8)
    assert list(load) == [7, 7, 7, 7, 0, 0, 0, 0]
    assert list(tok_of[:7]) == list(range(7))


def test_combine_one_hot_is_a_copy():
    y = np.arange(6 * 4, dtype=np.float64).reshape(6, 4)
    row_of = np.array([3, 0, 5, 1, 2, 4])
    w = np.array([[1, 0], [0, 1], [1, 0]], dtype=np.float32)
    out = oracle.combine(y, row_of, w)
    assert np.array_equal(out, np.stack([y[3], y[1], y[2]]))
    out2 = oracle.combine(y, row_of, w, yshared=np.ones((3, 4)))
    assert np.array_equal(out2, out + 1)


def _codes_of_small_integers(rng, shape, lo=-8, hi=8):
    ints = rng.integers(lo, hi + 1, shape)
    return oracle.e4m3_encode(ints.astype(np.float32)), ints


def test_gemm_exact_integer_case():
    """Integer codes (|v| <= 8) and unit scales: every product and sum is an
    integer, so C must equal the exact integer matrix product (Python ints)."""
    rng = np.random.default_rng(0)
    aq, ai = _codes_of_small_integers(rng, (37, 384))
    bq, bi = _codes_of_small_integers(rng, (256, 384))
    sa = np.ones((37, 3), np.float32)
    sb = np.ones((2, 3), np.float32)
    C = oracle.gemm_blockscaled(aq, sa, bq, sb)
    exact = np.array(ai, dtype=object) @ np.array(bi, dtype=object).T
    assert np.array_equal(C, exact.astype(np.float64))


def test_gemm_scales_enter_per_block():
    """Powers-of-two scales keep everything exact: compare with the exact
    integer sum of scale_a * scale_b * a * b over each 128-block."""
    rng = np.random.default_rng(1)
    aq, ai = _codes_of_small_integers(rng, (5, 256))
    bq, bi = _codes_of_small_integers(rng, (128, 256))
    sa = np.array([[2.0, 0.5]] * 5, np.float32)
    sb = np.array([[4.0, 0.25]], np.float32)
    C = oracle.gemm_blockscaled(aq, sa, bq, sb)
    ref = 8.0 * (ai[:, :128] @ bi[:, :128].T) + 0.125 * (ai[:, 128:] @ bi[:, 128:].T)
    assert np.array_equal(C, ref)


def test_gemm_matches_dense_float64_of_dequantised():
    """Promotion per 128 of K equals the plain float64 product of the
    dequantised operands up to the order of float64 additions."""
    rng = np.random.default_rng(2)
    a = synth.heavy_tailed(40, 512, 3).float().numpy()
    b = synth.normal((256, 512), 0.02, 4).numpy()
    aq, sa = oracle.quant_1x128(a)
    bq, sb = oracle.quant_128x128(b)
    C = oracle.gemm_blockscaled(aq, sa, bq, sb)
    A = torch.from_numpy(oracle.dequant_1x128(aq, sa))
    B = torch.from_numpy(oracle.dequant_128x128(bq, sb))
    ref = (A @ B.T).numpy()
    assert np.allclose(C, ref, rtol=1e-12, atol=1e-12 * np.abs(ref).max())
    # and the quantised product is close to the unquantised one
    full = a.astype(np.float64) @ b.astype(np.float64).T
    assert np.linalg.norm(C - full) / np.linalg.norm(full) < 0.05


def test_grouped_gemm_rows_follow_groups():
    rng = np.random.default_rng(5)
    offs = np.array([0, 3, 3, 10])
    aq, _ = _codes_of_small_integers(rng, (10, 128))
    bq = np.stack([_codes_of_small_integers(rng, (128, 128))[0] for _ in range(3)])
    sa = np.ones((10, 1), np.float32)
    sb = np.ones((3, 1, 1), np.float32)
    C = oracle.grouped_gemm_blockscaled(offs, aq, sa, bq, sb)
    assert np.array_equal(C[:3], oracle.gemm_blockscaled(aq[:3], sa[:3], bq[0], sb[0]))
    assert np.array_equal(C[3:], oracle.gemm_blockscaled(aq[3:], sa[3:], bq[2], sb[2]))


def test_silu_swiglu_closed_forms():
    assert oracle.silu(0.0) == 0.0
    assert abs(oracle.silu(40.0) - 40.0) < 1e-12
    assert abs(oracle.silu(-40.0)) < 1e-15
    g = np.linspace(-6, 6, 101)
    ref = torch.nn.functional.silu(torch.from_numpy(g)).numpy()
    assert np.allclose(oracle.silu(g), ref, rtol=1e-14, atol=1e-16)
    gu = np.concatenate([g[None], np.full((1, 101), 3.0)], 1)
    assert np.allclose(oracle.swiglu(gu), 3 * ref[None], rtol=1e-14)


def _tiny_layer(E=1, K=1, n_group=1, topk_group=1, T=8, H=128, I=128, seed=0):
    x = synth.activations(T, H, seed).float().numpy()
    wr = synth.router_weights(E, H, 0.02, seed + 1).numpy()
    bias = np.zeros(E, np.float32)
    w13 = np.stack([synth.expert_weight(2 * I, H, 0.02, seed + 10 + e).float().numpy() for e in range(E)])
    w2 = np.stack([synth.expert_weight(H, I, 0.02, seed + 50 + e).float().numpy() for e in range(E)])
    sh13 = synth.expert_weight(2 * I, H, 0.02, seed + 90).float().numpy()
    sh2 = synth.expert_weight(H, I, 0.02, seed + 91).float().numpy()
    W = oracle.quantize_layer_weights(w13, w2, sh13, sh2)
    return x, wr, bias, W, (w13, w2, sh13, sh2)


def test_layer_single_expert_reduces_to_two_dense_ffns():
    """E = K = 1, one group: every token goes to expert 0 with gate 2.5, so
    out = bf16(2.5 * bf16(FFN_0(x)) + bf16(FFN_shared(x))), each FFN written
    out here from dequantised operands with torch float64 ops."""
    x, wr, bias, W, (w13, w2, sh13, sh2) = _tiny_layer()
    res = oracle.moe_forward(x, wr, bias, W, 1, 1, 1, 2.5)
    assert np.all(res["idx"] == 0) and np.all(res["w"] == np.float32(2.5))

    def ffn(wq13, wq2):
        xq, xs = oracle.quant_1x128(x)
        X = torch.from_numpy(oracle.dequant_1x128(xq, xs))
        G = X @ torch.from_numpy(oracle.dequant_128x128(*wq13)).T
        I = G.shape[1] // 2
        act = (torch.nn.functional.silu(G[:, :I]) * G[:, I:]).float().numpy()
        aq, as_ = oracle.quant_1x128(act)
        Y = torch.from_numpy(oracle.dequant_1x128(aq, as_)) @ torch.from_numpy(oracle.dequant_128x128(*wq2)).T
        return Y.numpy()

    y0 = ffn(W.get("w13", 0), W.get("w2", 0))
    ysh = ffn(W.get("w13", -1), W.get("w2", -1))
    b16 = lambda v: torch.from_numpy(v).to(torch.bfloat16).double().numpy()
    ref = 2.5 * b16(y0) + b16(ysh)
    got = res["out64"]
    assert np.linalg.norm(got - ref) / np.linalg.norm(ref) < 1e-6
    assert np.allclose(res["yperm"], b16(y0), rtol=0, atol=np.abs(y0).max() * 2 ** -7)


def test_layer_tokens_equal_full_layer():
    """The per-token form equals the batch form row by row."""
    E, K = 8, 2
    x, wr, bias, W, _ = _tiny_layer(E=E, K=K, n_group=2, topk_group=1, T=12)
    full = oracle.moe_forward(x, wr, bias, W, 2, 1, K, 2.5)
    part = oracle.moe_forward_tokens(x[[1, 7, 11]], wr, bias, W, 2, 1, K, 2.5)
    assert np.array_equal(part["idx"], full["idx"][[1, 7, 11]])
    assert np.array_equal(part["out"], full["out"][[1, 7, 11]])


# ---------------------------------------------------------------- node-limited combine
def test_combine_by_rank_hand_example():
    """Three slots, two ranks.  Rank 0's partial 1 + 2^-8 lies exactly halfway
    between the bf16 neighbours 1 and 1 + 2^-7 and rounds to even (1.0); rank 1's
    partial 2^-8 is exact; the source's float64 sum is 1 + 2^-8.  The single
    combine of the same slots gives 1 + 2^-7."""
    y = np.array([[1.0], [2.0 ** -8], [2.0 ** -8]])
    row_of = np.array([0, 1, 2])
    w = np.ones((1, 3), dtype=np.float32)
    got = oracle.combine_by_rank(y, row_of, w, np.array([[0, 0, 1]]))
    assert got[0, 0] == 1.0 + 2.0 ** -8
    assert oracle.combine(y, row_of, w)[0, 0] == 1.0 + 2.0 ** -7


def test_combine_by_rank_reduces_to_the_combine():
    rng = np.random.default_rng(5)
    T, K, H = 6, 4, 16
    # bf16 rows and power-of-two gates: every product and every partial is exact in bf16
    y = rng.integers(-8, 8, (T * K, H)).astype(np.float64)
    w = (2.0 ** rng.integers(-3, 1, (T, K))).astype(np.float32)
    row_of = rng.permutation(T * K)
    ysh = oracle.round_bf16(rng.standard_normal((T, H)))
    distinct = np.tile(np.arange(K), (T, 1))
    assert np.array_equal(oracle.combine_by_rank(y, row_of, w, distinct, ysh), oracle.combine(y, row_of, w, ysh))
    # one rank for every slot: the partial is the whole gated sum, rounded once
    y2 = rng.standard_normal((T * K, H))
    same = np.zeros((T, K), dtype=np.int64)
    want = oracle.round_bf16(oracle.combine(y2, row_of, w)) + ysh
    assert np.array_equal(oracle.combine_by_rank(y2, row_of, w, same, ysh), want)
