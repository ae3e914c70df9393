"""Pins of the oracle's router, selection, gates, load and bias update."""
import itertools

import numpy as np
import pytest
import torch

import oracle
import synth


def _tiny_inputs(seed=0, ties=0.0):
    s = synth.scores(64, 16, seed, tie_frac=ties).numpy()
    b = synth.expert_bias(16, 0.01, seed + 1).numpy()
    return s, b


@pytest.mark.parametrize("ties", [0.0, 0.3])
def test_selection_matches_bruteforce_tiny(ties):
    """Exhaustive search over all C(4,2) group pairs and all C(8,4) expert
    subsets of the kept groups (the tiny workload: E=16, K=4, 4 groups, 2 kept)."""
    s, b = _tiny_inputs(ties=ties)
    idx, w = oracle.select_experts(s, b, 4, 2, 4, 2.5)
    for t in range(s.shape[0]):
        bi, bw = oracle.select_experts_bruteforce(s[t], b, 4, 2, 4, 2.5)
        assert list(idx[t]) == bi
        assert np.array_equal(w[t], np.array(bw, dtype=np.float32))


def test_ungrouped_reduces_to_plain_topk():
    """topk_group == n_group: plain top-K of s + b (torch.topk on distinct values)."""
    s = synth.scores(200, 64, 5).numpy()
    b = synth.expert_bias(64, 0.01, 6).numpy()
    idx, _ = oracle.select_experts(s, b, 8, 8, 6, 2.5)
    r = torch.from_numpy((s + b).astype(np.float32))
    ref = torch.topk(r, 6, dim=1, largest=True, sorted=True).indices.numpy()
    # distinct values (checked) make the top-K unique
    assert all(len(set(row)) == 64 for row in (s + b).astype(np.float32))
    assert np.array_equal(idx, ref)


def test_group_limit_respected_and_ties_to_lower_index():
    s = np.full((1, 16), 0.5, dtype=np.float32)
    b = np.zeros(16, dtype=np.float32)
    idx, w = oracle.select_experts(s, b, 4, 2, 4, 2.5)
    # all equal: groups 0 and 1 are kept, experts in ascending order
    assert list(idx[0]) == [0, 1, 2, 3]
    assert np.allclose(w, 2.5 / 4)
    # the group score uses the top-2 sum, not the top-1: group 3 has the
    # single largest value but group 1 has the larger top-2 sum
    s = np.full((1, 16), 0.1, dtype=np.float32)
    s[0, 12] = 0.9                # group 3: top2 = 0.9 + 0.1 = 1.0
    s[0, 4:6] = 0.6               # group 1: top2 = 1.2
    s[0, 8:10] = 0.55             # group 2: top2 = 1.1
    idx, _ = oracle.select_experts(s, b, 4, 2, 4, 2.5)
    assert sorted(set(i // 4 for i in idx[0])) == [1, 2]


def test_k_equals_e_gives_normalised_affinities():
    s = synth.scores(10, 8, 7).numpy()
    b = np.zeros(8, dtype=np.float32)
    idx, w = oracle.select_experts(s, b, 1, 1, 8, 2.5)
    for t in range(10):
        want = 2.5 * s[t].astype(np.float64) / s[t].astype(np.float64).sum()
        got = np.zeros(8)
        got[idx[t]] = w[t]
        assert np.allclose(got, want, rtol=1e-7, atol=0)


def test_gate_invariants():
    s, b = _tiny_inputs(3)
    idx, w = oracle.select_experts(s, b, 4, 2, 4, 2.5)
    assert (w >= 0).all()
    sums = w.astype(np.float64).sum(1)
    assert np.all(np.abs(sums - 2.5) <= 4 * np.spacing(np.float32(2.5)))
    # the bias ranks but never enters the gate: gates use s only
    for t in range(5):
        tot = s[t, idx[t]].astype(np.float64).sum()
        assert np.allclose(w[t], 2.5 * s[t, idx[t]] / tot, rtol=1e-7)
    # every token's experts are distinct
    assert all(len(set(r)) == 4 for r in idx)


def test_bias_changes_ranking_only():
    s = np.array([[0.50, 0.49, 0.48, 0.47]], dtype=np.float32)
    b = np.array([0.0, 0.0, 0.05, 0.0], dtype=np.float32)
    idx, w = oracle.select_experts(s, b, 1, 1, 2, 1.0)
    assert list(idx[0]) == [2, 0]                   # 0.53 > 0.50
    assert np.allclose(w[0], [0.48 / 0.98, 0.50 / 0.98], rtol=1e-6)


def test_router_scores_closed_form():
    x = np.zeros((2, 128), dtype=np.float32)
    wr = np.ones((3, 128), dtype=np.float32) * 0.5
    x[1, 0] = 2.0
    s = oracle.router_scores(x, wr)
    assert np.allclose(s[0], 0.5)
    assert np.allclose(s[1], 1 / (1 + np.exp(-1.0)))
    s2 = oracle.router_scores(x, wr, offset=np.array([0.0, 1.0, -1.0], dtype=np.float32))
    assert np.allclose(s2[0], 1 / (1 + np.exp(-np.array([0.0, 1.0, -1.0]))))
    # against torch's sigmoid of a float64 matmul on random data
    xb = synth.activations(8, 256, 1).float().numpy()
    w = synth.router_weights(16, 256, 0.02, 2).numpy()
    ref = torch.sigmoid(torch.from_numpy(xb).double() @ torch.from_numpy(w).double().T).numpy()
    assert np.allclose(oracle.router_scores(xb, w), ref, rtol=1e-13, atol=0)


def test_load_and_bias_update_hand_computed():
    idx = np.array([[0, 1], [0, 2], [0, 1], [3, 1]], dtype=np.int32)   # T=4, K=2, E=4
    load = oracle.expert_load(idx, 4)
    assert list(load) == [3, 3, 1, 1]                                  # mean 2
    b = np.array([0.0, 0.25, -0.5, 1.0], dtype=np.float32)
    nb = oracle.bias_update(b, load, 4, 2, 0.001)
    g = np.float32(0.001)
    assert nb[0] == np.float32(0 - g) and nb[1] == np.float32(np.float32(0.25) - g)
    assert nb[2] == np.float32(np.float32(-0.5) + g) and nb[3] == np.float32(np.float32(1.0) + g)
    # sign(0) = 0: an exactly average load leaves the bias unchanged
    nb2 = oracle.bias_update(b, np.array([2, 2, 2, 2]), 4, 2, 0.001)
    assert np.array_equal(nb2, b)
    # the mean need not be an integer: T*K/E = 3/2 -> load 1 under, load 2 over
    nb3 = oracle.bias_update(np.zeros(2, np.float32), np.array([1, 2]), 3, 1, 0.5)
    assert list(nb3) == [0.5, -0.5]


def test_seq_balance_loss_hand_computed():
    # one sequence of 2 tokens, E = 2, K = 1: token 0 -> expert 0, token 1 -> expert 0
    s = np.array([[0.8, 0.2], [0.6, 0.4]])
    idx = np.array([[0], [0]])
    # f = (1, 0), P = (0.7, 0.3): L = alpha * 0.7
    assert np.allclose(oracle.seq_balance_loss(s, idx, 2, 0.001), [0.0007], rtol=1e-15)
    # two sequences of one token each
    got = oracle.seq_balance_loss(s, np.array([[0], [1]]), 1, 1.0)
    assert np.allclose(got, [0.8, 0.4], rtol=1e-15)


def test_seq_balance_loss_closed_forms():
    # constant affinities c and any routing: sum_i f_i = 1, so L = alpha * c
    T, E, K = 64, 16, 4
    idx = synth.topk_indices(T, E, K, 3).numpy()
    s = np.full((T, E), 0.25)
    assert np.allclose(oracle.seq_balance_loss(s, idx, 16, 0.01), 0.0025, rtol=1e-14)
    # against a brute-force triple loop
    s = synth.scores(T, E, 9).numpy().astype(np.float64)
    want = []
    for q in range(4):
        acc = 0.0
        for i in range(E):
            cnt = sum(1 for t in range(16 * q, 16 * q + 16) for k in range(K) if idx[t, k] == i)
            mean = sum(s[t, i] for t in range(16 * q, 16 * q + 16)) / 16
            acc += cnt / (16 * K) * mean
        want.append(0.001 * acc)
    assert np.allclose(oracle.seq_balance_loss(s, idx, 16, 0.001), want, rtol=1e-13)


def test_load_entropy_closed_forms():
    assert abs(oracle.load_entropy(np.full(256, 128)) - np.log(256)) < 1e-12
    assert oracle.load_entropy(np.array([0, 0, 5, 0])) == 0.0
    assert abs(oracle.load_entropy(np.array([1, 1, 2])) - (-(0.25 * np.log(0.25) * 2 + 0.5 * np.log(0.5)))) < 1e-15
