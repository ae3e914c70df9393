"""Router, group-limited top-K selection, gates and the bias update (oracle).

Test infrastructure only (see the package docstring).

What the pages fix ([report-walkthrough] section 3.2, its router/bias
pseudocode, and [repro-guide] section 3 config):
  s      = sigmoid(h . W_router)            affinities, sigmoid not softmax
  idx    = topk(s + b, K)                   the bias only ranks
  gate   = normalize(s.gather(idx))         gate values come from s, no bias
  y      = sum_j gate_j * ffn_{idx_j}(h)
  load   = bincount(idx), target = T*K/N_r
  b_i   -= gamma if load_i is over target, += gamma if under
with norm_topk_prob = true and routed_scaling_factor = 2.5.  Node-limited
routing ([report-walkthrough] section 3.4): each token is sent to at most M
nodes, chosen by the sum of the highest affinities of the experts on each
node; here a "node" is one of n_group equal expert groups, M = topk_group.

Readings where the pages are silent:
* the group score is the sum of the top min(2, E/n_group) values of s + b in
  the group, added in fp32;
* ties go to the lower index (groups and experts); output order is
  descending s + b, then ascending expert index;
* s + b is one fp32 addition; every ranking decision is taken on fp32
  values, the precision the GPU kernel decides in;
* normalize: w_k = (rho * s_k) / sum_{j in top-K} s_j, evaluated in float64
  from the fp32 affinities and rounded once to fp32;
* bias update: b_i += gamma * sign(T*K/E - load_i) with sign(0) = 0
  (dead band eps = 0), each update one fp32 addition.
"""
from __future__ import annotations

import itertools

import numpy as np


def router_scores(x, w_router, offset=None) -> np.ndarray:
    """Affinities s = sigmoid(x . W_r^T (+ offset)) in float64.

    x [T, H] (bf16 values), w_router [E, H] fp32, offset [E] fp32 or None
    (the skewed-routing workload's per-expert logit offset)."""
    x64 = np.asarray(x, dtype=np.float64)
    w64 = np.asarray(w_router, dtype=np.float64)
    logits = x64 @ w64.T
    if offset is not None:
        logits = logits + np.asarray(offset, dtype=np.float64)[None, :]
    return 1.0 / (1.0 + np.exp(-logits))


def _group_scores(r32: np.ndarray, n_group: int) -> np.ndarray:
    """fp32 sum of the top min(2, group size) values of each group."""
    T, E = r32.shape
    gs = E // n_group
    grp = np.sort(r32.reshape(T, n_group, gs), axis=-1)[..., ::-1]   # descending
    if gs == 1:
        return grp[..., 0].astype(np.float32)
    return (grp[..., 0] + grp[..., 1]).astype(np.float32)            # one fp32 add


def select_experts(s32, bias32, n_group: int, topk_group: int, K: int, rho: float):
    """Group-limited, bias-ranked top-K and normalised, scaled gates.

    s32 [T, E] fp32 affinities, bias32 [E] fp32.
    Returns idx int32 [T, K] (descending s+b, ties to lower index) and
    w fp32 [T, K]."""
    s32 = np.asarray(s32, dtype=np.float32)
    b32 = np.asarray(bias32, dtype=np.float32)
    T, E = s32.shape
    assert E % n_group == 0 and 1 <= topk_group <= n_group
    gs = E // n_group
    assert topk_group * gs >= K
    r = (s32 + b32[None, :]).astype(np.float32)                      # one fp32 add
    gscore = _group_scores(r, n_group)
    # stable sort on the negated key: larger first, equal keys keep index order
    gorder = np.argsort(-gscore, axis=1, kind="stable")[:, :topk_group]
    keep = np.zeros((T, n_group), dtype=bool)
    np.put_along_axis(keep, gorder, True, axis=1)
    keep_e = np.repeat(keep, gs, axis=1)
    masked = np.where(keep_e, r.astype(np.float64), -np.inf)
    idx = np.argsort(-masked, axis=1, kind="stable")[:, :K]
    s_sel = np.take_along_axis(s32, idx, axis=1).astype(np.float64)
    w = (rho * s_sel) / s_sel.sum(axis=1, keepdims=True)
    return idx.astype(np.int32), w.astype(np.float32)


def select_experts_bruteforce(s32_row, bias32, n_group: int, topk_group: int, K: int, rho: float):
    """Same selection for ONE token by exhaustive search (small E only).

    Groups: among all topk_group-subsets of groups, the chosen one is the
    subset whose (score, -index) pairs sorted descending are lexicographically
    largest.  Experts: among all K-subsets of the kept groups' experts, the
    chosen one is the lexicographically largest by sorted (r, -index) pairs.
    Returns (idx list in output order, w list)."""
    s = np.asarray(s32_row, dtype=np.float32)
    b = np.asarray(bias32, dtype=np.float32)
    E = s.shape[0]
    gs = E // n_group
    r = [np.float32(s[e] + b[e]) for e in range(E)]
    gscore = []
    for g in range(n_group):
        vals = sorted((r[e] for e in range(g * gs, (g + 1) * gs)), reverse=True)
        gscore.append(vals[0] if gs == 1 else np.float32(vals[0] + vals[1]))

    def key_of(items, val):
        return sorted(((val[i], -i) for i in items), reverse=True)

    best_g = max(itertools.combinations(range(n_group), topk_group),
                 key=lambda c: key_of(c, gscore))
    allowed = [e for g in best_g for e in range(g * gs, (g + 1) * gs)]
    best = max(itertools.combinations(allowed, K), key=lambda c: key_of(c, r))
    order = [-negi for _, negi in key_of(best, r)]
    tot = sum(float(s[e]) for e in order)
    w = [np.float32(rho * float(s[e]) / tot) for e in order]
    return order, w


def expert_load(idx, E: int) -> np.ndarray:
    """load[e] = number of (token, slot) pairs routed to expert e (bincount)."""
    flat = np.asarray(idx, dtype=np.int64).reshape(-1)
    return np.bincount(flat, minlength=E).astype(np.int32)


def bias_update(bias32, load, T: int, K: int, gamma: float) -> np.ndarray:
    """b_e += gamma * sign(T*K/E - load_e), sign(0) = 0, one fp32 add each.

    The comparison with the mean T*K/E is made exactly in integers
    (T*K versus E*load_e)."""
    b = np.asarray(bias32, dtype=np.float32).copy()
    load = np.asarray(load, dtype=np.int64)
    E = b.shape[0]
    g32 = np.float32(gamma)
    for e in range(E):
        diff = T * K - E * int(load[e])
        if diff > 0:        # under-loaded: raise its bias
            b[e] = np.float32(b[e] + g32)
        elif diff < 0:      # over-loaded: lower it
            b[e] = np.float32(b[e] - g32)
    return b


def seq_balance_loss(s, idx, seq_len: int, alpha: float) -> np.ndarray:
    """Sequence-wise balance loss, one value per sequence ([report-walkthrough]
    section 3.3: per sequence, the sum over experts of each expert's share of the
    sequence's assignments times its mean affinity over the sequence, times a
    small coefficient alpha; aux_loss_alpha 0.001 in [repro-guide] section 3).

    Reading (the pages give no normalisation): for a sequence of S tokens,
        f_i = (#slots of the sequence routed to i) / (S * K)
        P_i = (1 / S) * sum_t s[t, i]        (the sigmoid affinities)
        L   = alpha * sum_i f_i * P_i
    s [T, E] affinities, idx [T, K]; T must be a multiple of seq_len.
    Returns float64 [T / seq_len]."""
    s = np.asarray(s, dtype=np.float64)
    idx = np.asarray(idx, dtype=np.int64)
    T, E = s.shape
    K = idx.shape[1]
    assert T % seq_len == 0
    out = np.zeros(T // seq_len)
    for q in range(T // seq_len):
        rows = slice(q * seq_len, (q + 1) * seq_len)
        f = np.bincount(idx[rows].reshape(-1), minlength=E) / (seq_len * K)
        P = s[rows].sum(axis=0) / seq_len
        out[q] = alpha * float(np.sum(f * P))
    return out


def load_entropy(load) -> float:
    """Entropy (natural log) of the expert-load distribution p_i = load_i / sum(load),
    with 0 log 0 = 0: log(E) for perfectly even loads, 0 when one expert takes all."""
    load = np.asarray(load, dtype=np.float64)
    tot = load.sum()
    if tot <= 0:
        return 0.0
    p = load[load > 0] / tot
    return float(-np.sum(p * np.log(p)))
