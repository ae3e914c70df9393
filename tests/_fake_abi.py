"""A CPU stand-in of the library binding, built from the oracle, for testing host
logic that chains the calls (the expert-parallel layer's dispatch and combine)
on CPU ranks without a GPU.  Test infrastructure only.

Every function has the name and arguments of the binding's function and writes
its outputs in place into CPU tensors; the arithmetic is the oracle's, so a
chain of these calls reproduces the oracle's layer bit for bit."""
import numpy as np
import torch

import oracle
from sparse_moe_layer_group_b200._abi import (MOE_EP_BLOCK, MOE_EP_CYCLIC, MOE_EPI_BF16, MOE_EPI_F32,  # noqa: F401
                                              MOE_EPI_SWIGLU_REQUANT, dims)

_WR = {}


def workspace_size(d):
    return 256


def moe_router_pieces_bytes(E, H):
    return 3 * E * H * 2


def moe_router_split(w_router, w_pieces, stream=None):
    _WR[w_pieces.data_ptr()] = w_router.detach().clone()


def moe_route_pieces(d, x, w_pieces, e_bias, router_offset, topk_idx, topk_w, scores=None, ws=None,
                     status=None, stream=None):
    wr = _WR[w_pieces.data_ptr()].numpy()
    off = None if router_offset is None else router_offset.numpy()
    s32 = oracle.router_scores(x.float().numpy(), wr, off).astype(np.float32)
    idx, w = oracle.select_experts(s32, e_bias.numpy(), d.n_group, d.topk_group, d.K, d.routed_scaling_factor)
    topk_idx.copy_(torch.from_numpy(idx.astype(np.int32)))
    topk_w.copy_(torch.from_numpy(w.astype(np.float32)))
    if scores is not None:
        scores.copy_(torch.from_numpy(s32))


def fp8_quant_1x128(x, q, scales, status=None, stream=None):
    cq, cs = oracle.quant_1x128(x.float().numpy())
    q.copy_(torch.from_numpy(cq))
    scales.copy_(torch.from_numpy(cs))


def moe_ep_split(topk_idx, E, world, dest_rank, local_idx, status=None, stream=None):
    e = topk_idx.reshape(-1).numpy().astype(np.int64)
    dest_rank.copy_(torch.from_numpy((e % world).astype(np.int32)))
    local_idx.copy_(torch.from_numpy((e // world).astype(np.int32)))


def _permute_skipping(idx, E):
    """oracle.permute over the entries in [0, E); the others get row_of = -1
    (the library's treatment of an index it does not dispatch)."""
    T, K = idx.shape
    ok = (idx >= 0) & (idx < E)
    if ok.all():
        return oracle.permute(idx, E)
    pairs = sorted((int(idx[t, k]), t, k) for t in range(T) for k in range(K) if ok[t, k])
    load = np.bincount([e for e, _, _ in pairs], minlength=E).astype(np.int32)
    offs = np.concatenate([[0], np.cumsum(load)]).astype(np.int32)
    tok = np.zeros(T * K, dtype=np.int32)
    row = np.full(T * K, -1, dtype=np.int32)
    for r, (_, t, k) in enumerate(pairs):
        tok[r] = t
        row[t * K + k] = r
    return load, offs, tok[:len(pairs)], row


def moe_permute(d, topk_idx, xq, xs, expert_load, expert_offsets, tok_of, row_of, aq, as_, ws, status=None,
                stream=None):
    idx = topk_idx.reshape(d.T, d.K).numpy()
    load, offs, tok, row = _permute_skipping(idx, d.E)
    expert_load.copy_(torch.from_numpy(load))
    expert_offsets.copy_(torch.from_numpy(offs))
    tok_of[:len(tok)].copy_(torch.from_numpy(tok))
    row_of.copy_(torch.from_numpy(row))
    if aq is not None:
        t = torch.from_numpy(tok.astype(np.int64))
        aq[:len(tok)].copy_(xq[t])
        as_[:len(tok)].copy_(xs[t])


def moe_ep_scatter(row_of, values, out, stream=None):
    r = row_of.numpy().astype(np.int64)
    ok = r >= 0
    out[torch.from_numpy(r[ok])] = values[torch.from_numpy(ok)]


def fp8_grouped_gemm_blockscaled(G, group_offsets, m_capacity, N, K, A, sA, B, sB, epilogue, C, sC=None,
                                 status=None, stream=None):
    offs = group_offsets.numpy().astype(np.int64)[:G + 1]
    used = int(offs[-1])
    gu = oracle.grouped_gemm_blockscaled(offs, A[:used].numpy(), sA[:used].numpy(), B[:G].numpy(), sB[:G].numpy())
    lo = int(offs[0])
    if epilogue == MOE_EPI_SWIGLU_REQUANT:
        q, s, _ = oracle.swiglu_requant(gu)
        C[lo:used].copy_(torch.from_numpy(q[lo:used]))
        sC[lo:used].copy_(torch.from_numpy(s[lo:used]))
    else:
        C[lo:used].copy_(torch.from_numpy(oracle.round_bf16(gu[lo:used])).to(C.dtype))


def moe_combine(d, yperm, row_of, topk_w, yshared, out, out_f32=None, stream=None):
    w = topk_w.reshape(d.T, d.K).numpy().copy()
    r = row_of.numpy().astype(np.int64).copy()
    skip = r < 0                                  # slots the library's combine skips
    w.reshape(-1)[skip] = 0.0
    r[skip] = 0
    ysh = None if yshared is None else yshared.float().numpy()
    o = oracle.combine(yperm.float().numpy(), r, w, ysh)
    out.copy_(torch.from_numpy(oracle.round_bf16(o)).to(out.dtype))


def moe_bias_update(E, T, K, gamma, expert_load, e_bias, stream=None):
    e_bias.copy_(torch.from_numpy(oracle.bias_update(e_bias.numpy(), expert_load.numpy(), T, K, gamma)))


def moe_ep_plan(topk_idx, topk_w, E, world, placement, dest_rank, meta_ids, meta_w, status=None, stream=None):
    idx = topk_idx.numpy().astype(np.int64)
    T, K = idx.shape
    El = E // world
    rank = idx // El if placement == MOE_EP_BLOCK else idx % world
    local = idx % El if placement == MOE_EP_BLOCK else idx // world
    dest = np.full(T * K, -1, dtype=np.int32)
    mid = np.full((T * K, K), -1, dtype=np.int32)
    mw = np.zeros((T * K, K), dtype=np.float32)
    w = topk_w.numpy()
    for t in range(T):
        for k in range(K):
            if rank[t, k] in rank[t, :k]:
                continue
            dest[t * K + k] = rank[t, k]
            on = rank[t] == rank[t, k]
            mid[t * K + k, on] = local[t, on]
            mw[t * K + k, on] = w[t, on]
    dest_rank.copy_(torch.from_numpy(dest))
    meta_ids.copy_(torch.from_numpy(mid))
    meta_w.copy_(torch.from_numpy(mw))


def moe_ep_scatter_rows(row_of, values, out, stream=None):
    r = row_of.numpy().astype(np.int64)
    ok = r >= 0
    out[torch.from_numpy(r[ok])] = values[torch.from_numpy(ok)]
