"""Expert-parallel DeepSeekMoE layer forward: the routed experts spread over the
ranks of a process group, each rank routing its own tokens.

Two dispatch forms:

* per slot (dedupe=False): every (token, slot) pair is sent to the rank of its
  expert as its own row, computed there and returned as its own row; the
  source combines them exactly as the single-GPU layer (same bits).
* node-limited (dedupe=True, the default): a token crosses to each rank it
  selected at most once (section 3.4 of the walkthrough: a token reaches at
  most M nodes; section 4.1: it crosses once and is forwarded there to its
  experts).  The row carries the local expert ids and gates of all of the
  token's slots on that rank; the receiving rank computes them and sums them
  (gated) into one partial row, which crosses back in bf16; the source adds the
  partial rows and the shared expert.  With placement "block" (expert e on rank
  e // (E/world)) and world == n_group, a rank is a routing group, so a token
  crosses to at most topk_group ranks.  The extra bf16 rounding of each
  partial makes this form equal to the oracle's combine_by_rank, not to the
  single-GPU layer's bits.

The "DeepSeek-V3 technical report" walkthrough (2kiu.com), section 4.1, runs
the routed experts with expert parallelism: every device holds a subset of the
experts, a token's rows are dispatched to the devices of its experts, processed
there and combined back (dispatch -> expert MLP -> combine), with the dispatch
payload in FP8.  Here routed expert e lives on rank e % world as local expert
e // world; the shared expert is replicated (every rank runs it on its own
tokens).  One forward on each rank:

  1  route and quantise the rank's T tokens (as the single-GPU layer)
  2  moe_ep_split: destination rank and local expert id of every (token, slot)
  3  moe_permute with the ranks as groups: the E4M3 rows and scales of the
     (token, slot) pairs in destination order (the send buffer), and
     moe_ep_scatter of the local expert ids into the same order
  4  all-to-all of the row counts, then of rows, scales and ids (torch.distributed:
     NCCL between GPUs, gloo on CPU)
  5  moe_permute of the received rows by local expert, the two grouped GEMMs of
     the local experts, and moe_combine with unit weights to put the results back
     in received order
  6  all-to-all of the result rows back to their sources
  7  the shared expert's two GEMMs on the rank's own tokens, and moe_combine of
     the returned rows (by the send permutation's row_of) with the gates

Every arithmetic step runs in the library's kernels (or, in the CPU tests, in
an injected stand-in of the binding); torch.distributed only moves buffers.

The bias update (section 3.3 of the walkthrough: b_e moves by gamma against the
imbalance of expert e's load over the batch) needs every expert's load over all
ranks' tokens.  Expert e's global load is exactly the number of rows rank
e % world received for it (the local permutation's load), so bias_update
all-gathers the local loads into the global vector and every rank applies the
same update to its copy of the bias: the copies stay identical without
exchanging the bias itself.
"""
from __future__ import annotations

from typing import Optional

import torch
import torch.distributed as dist

from . import _abi
from .layer import QuantWeights


class EPMoELayer:
    """One rank's part of an expert-parallel layer for T tokens per rank.

    weights holds this rank's routed experts in local order followed by the
    shared expert: with placement "cyclic" the global experts rank, rank +
    world, ...; with "block" the experts rank * E/world .. (rank + 1) * E/world - 1."""

    def __init__(self, T: int, H: int, E: int, K: int, n_group: int, topk_group: int, I: int, rho: float,
                 w_router: torch.Tensor, e_bias: torch.Tensor, weights: QuantWeights, group=None,
                 router_offset: Optional[torch.Tensor] = None, device="cuda", abi=None, dedupe: bool = True,
                 placement: str = "block"):
        self.abi = _abi if abi is None else abi
        if placement not in ("cyclic", "block"):
            raise ValueError("placement is 'cyclic' or 'block'")
        if not dedupe and placement != "cyclic":
            raise ValueError("the per-slot dispatch places experts cyclically")
        self.dedupe, self.placement = dedupe, placement
        self.group = group
        self.world = dist.get_world_size(group) if (group is not None or dist.is_initialized()) else 1
        self.rank = dist.get_rank(group) if self.world > 1 or dist.is_initialized() else 0
        if E % self.world != 0:
            raise ValueError("the expert count must divide evenly over the ranks")
        self.T, self.H, self.E, self.K, self.I = T, H, E, K, I
        self.E_local = E // self.world
        if weights.E != self.E_local:
            raise ValueError("weights must hold this rank's E/world routed experts plus the shared one")
        self.qw = weights
        self.d = self.abi.dims(T, H, E, K, n_group, topk_group, I, rho)
        self.w_router, self.e_bias, self.router_offset = w_router, e_bias, router_offset
        i32 = dict(dtype=torch.int32, device=device)
        f32 = dict(dtype=torch.float32, device=device)
        u8 = dict(dtype=torch.uint8, device=device)
        bf = dict(dtype=torch.bfloat16, device=device)
        TK, W, Rmax = T * K, self.world, self.world * T * K
        self.w_pieces = torch.empty(self.abi.moe_router_pieces_bytes(E, H) // 2, **bf)
        self.abi.moe_router_split(w_router, self.w_pieces)
        ws_bytes = max(self.abi.workspace_size(self.d),
                       self.abi.workspace_size(self.abi.dims(Rmax, H, self.E_local, 1, 1, 1, I, rho)),
                       self.abi.workspace_size(self.abi.dims(W * T, H, self.E_local, K, 1, 1, I, rho)), 256)
        self.ws = torch.empty((ws_bytes + 255) // 256 * 256, **u8)
        self.topk_idx = torch.empty(T, K, **i32)
        self.topk_w = torch.empty(T, K, **f32)
        self.scores = torch.empty(T, E, **f32)
        self.xq = torch.empty(T, H, **u8)
        self.xs = torch.empty(T, H // 128, **f32)
        self.dest = torch.empty(TK, **i32)
        self.local = torch.empty(TK, **i32)
        self.send_load = torch.empty(W, **i32)
        self.send_offs = torch.empty(W + 1, **i32)
        self.tok_of_s = torch.empty(TK, **i32)
        self.row_of_s = torch.empty(TK, **i32)
        self.send_q = torch.empty(TK, H, **u8)
        self.send_s = torch.empty(TK, H // 128, **f32)
        self.send_ids = torch.empty(TK, **i32)
        self.recv_counts = torch.empty(W, **i32)
        self.recv_q = torch.empty(Rmax, H, **u8)
        self.recv_s = torch.empty(Rmax, H // 128, **f32)
        self.recv_ids = torch.empty(Rmax, **i32)
        self.load_l = torch.zeros(self.E_local, **i32)
        self.load_all = torch.zeros(E, **i32)
        self.offs_l = torch.empty(self.E_local + 1, **i32)
        self.tok_of_l = torch.empty(Rmax, **i32)
        self.row_of_l = torch.empty(Rmax, **i32)
        self.aq_l = torch.empty(Rmax, H, **u8)
        self.as_l = torch.empty(Rmax, H // 128, **f32)
        self.actq_l = torch.empty(Rmax, I, **u8)
        self.acts_l = torch.empty(Rmax, I // 128, **f32)
        self.yperm_l = torch.empty(Rmax, H, **bf)
        self.y_recv = torch.empty(Rmax, H, **bf)
        self.ones = torch.ones(Rmax, **f32)
        if dedupe:
            # node-limited dispatch: at most one row per (token, rank) each way,
            # with the K slots' local ids and gates riding along
            self.meta_ids = torch.empty(TK, K, **i32)
            self.meta_w = torch.empty(TK, K, **f32)
            self.send_mids = torch.empty(TK, K, **i32)
            self.send_mw = torch.empty(TK, K, **f32)
            self.recv_mids = torch.empty(W * T, K, **i32)
            self.recv_mw = torch.empty(W * T, K, **f32)
            self.row_of_p = torch.empty(W * T * K, **i32)
            self.ones_tk = torch.ones(T, K, **f32)
        self.y_back = torch.empty(TK, H, **bf)
        self.offs_sh = torch.tensor([0, T], **i32)
        self.actq_s = torch.empty(T, I, **u8)
        self.acts_s = torch.empty(T, I // 128, **f32)
        self.ysh = torch.empty(T, H, **bf)
        self.out = torch.empty(T, H, **bf)
        self.status = torch.zeros(1, **i32)

    def _all_to_all(self, out, inp, out_splits, in_splits):
        if self.world == 1:
            n = int(in_splits[0])
            if n:
                out[:n].copy_(inp[:n])
            return
        dist.all_to_all_single(out, inp, out_splits, in_splits, group=self.group)

    def forward(self, x: torch.Tensor) -> torch.Tensor:
        if self.dedupe:
            return self._forward_node_limited(x)
        a, T, H, K, I, E_l = self.abi, self.T, self.H, self.K, self.I, self.E_local
        st, qw = self.status, self.qw
        a.moe_route_pieces(self.d, x, self.w_pieces, self.e_bias, self.router_offset, self.topk_idx, self.topk_w,
                           self.scores, self.ws, st)
        a.fp8_quant_1x128(x, self.xq, self.xs, st)
        # dispatch: rows grouped by destination rank, local expert ids in the same order
        a.moe_ep_split(self.topk_idx, self.E, self.world, self.dest, self.local, st)
        dd = a.dims(T, H, self.world, K, 1, 1, I, 1.0)
        a.moe_permute(dd, self.dest, self.xq, self.xs, self.send_load, self.send_offs, self.tok_of_s, self.row_of_s,
                      self.send_q, self.send_s, self.ws, st)
        a.moe_ep_scatter(self.row_of_s, self.local, self.send_ids)
        self._all_to_all(self.recv_counts, self.send_load, [1] * self.world, [1] * self.world)
        send_splits = [int(v) for v in self.send_load.tolist()]
        recv_splits = [int(v) for v in self.recv_counts.tolist()]
        R = sum(recv_splits)
        self._all_to_all(self.recv_q[:R], self.send_q, recv_splits, send_splits)
        self._all_to_all(self.recv_s[:R], self.send_s, recv_splits, send_splits)
        self._all_to_all(self.recv_ids[:R], self.send_ids, recv_splits, send_splits)
        # the local experts on the received rows, results back in received order
        if R == 0:
            self.load_l.zero_()
        if R > 0:
            dl = a.dims(R, H, E_l, 1, 1, 1, I, 1.0)
            a.moe_permute(dl, self.recv_ids[:R], self.recv_q[:R], self.recv_s[:R], self.load_l, self.offs_l,
                          self.tok_of_l[:R], self.row_of_l[:R], self.aq_l[:R], self.as_l[:R], self.ws, st)
            a.fp8_grouped_gemm_blockscaled(E_l, self.offs_l, R, 2 * I, H, self.aq_l, self.as_l, qw.w13, qw.s13,
                                           a.MOE_EPI_SWIGLU_REQUANT, self.actq_l, self.acts_l, st)
            a.fp8_grouped_gemm_blockscaled(E_l, self.offs_l, R, H, I, self.actq_l, self.acts_l, qw.w2, qw.s2,
                                           a.MOE_EPI_BF16, self.yperm_l, None, st)
            a.moe_combine(dl, self.yperm_l, self.row_of_l[:R], self.ones[:R], None, self.y_recv[:R])
        self._all_to_all(self.y_back, self.y_recv[:R], send_splits, recv_splits)
        # the shared expert on this rank's tokens, then the gated combine
        a.fp8_grouped_gemm_blockscaled(1, self.offs_sh, T, 2 * I, H, self.xq, self.xs, qw.w13[E_l:], qw.s13[E_l:],
                                       a.MOE_EPI_SWIGLU_REQUANT, self.actq_s, self.acts_s, st)
        a.fp8_grouped_gemm_blockscaled(1, self.offs_sh, T, H, I, self.actq_s, self.acts_s, qw.w2[E_l:], qw.s2[E_l:],
                                       a.MOE_EPI_BF16, self.ysh, None, st)
        a.moe_combine(dd, self.y_back, self.row_of_s, self.topk_w, self.ysh, self.out)
        return self.out

    def _forward_node_limited(self, x: torch.Tensor) -> torch.Tensor:
        a, T, H, K, I, E_l, W = self.abi, self.T, self.H, self.K, self.I, self.E_local, self.world
        st, qw = self.status, self.qw
        a.moe_route_pieces(self.d, x, self.w_pieces, self.e_bias, self.router_offset, self.topk_idx, self.topk_w,
                           self.scores, self.ws, st)
        a.fp8_quant_1x128(x, self.xq, self.xs, st)
        # dispatch plan: one row per (token, rank), the first slot of each rank
        # stands for it; rows grouped by destination rank
        a.moe_ep_plan(self.topk_idx, self.topk_w, self.E, W,
                      a.MOE_EP_BLOCK if self.placement == "block" else a.MOE_EP_CYCLIC,
                      self.dest, self.meta_ids, self.meta_w, st)
        dd = a.dims(T, H, W, K, 1, 1, I, 1.0)
        # status None: the -1 entries of dest are slots that are not sent
        a.moe_permute(dd, self.dest, self.xq, self.xs, self.send_load, self.send_offs, self.tok_of_s, self.row_of_s,
                      self.send_q, self.send_s, self.ws, None)
        a.moe_ep_scatter_rows(self.row_of_s, self.meta_ids, self.send_mids)
        a.moe_ep_scatter_rows(self.row_of_s, self.meta_w.view(torch.int32), self.send_mw.view(torch.int32))
        self._all_to_all(self.recv_counts, self.send_load, [1] * W, [1] * W)
        send_splits = [int(v) for v in self.send_load.tolist()]
        recv_splits = [int(v) for v in self.recv_counts.tolist()]
        R = sum(recv_splits)
        S = sum(send_splits)
        self._all_to_all(self.recv_q[:R], self.send_q[:S], recv_splits, send_splits)
        self._all_to_all(self.recv_s[:R], self.send_s[:S], recv_splits, send_splits)
        self._all_to_all(self.recv_mids[:R], self.send_mids[:S], recv_splits, send_splits)
        self._all_to_all(self.recv_mw[:R], self.send_mw[:S], recv_splits, send_splits)
        # the local experts of every received row, then each row's gated sum
        if R == 0:
            self.load_l.zero_()
        else:
            dl = a.dims(R, H, E_l, K, 1, 1, I, 1.0)
            a.moe_permute(dl, self.recv_mids[:R], self.recv_q[:R], self.recv_s[:R], self.load_l, self.offs_l,
                          self.tok_of_l[:R * K], self.row_of_p[:R * K], self.aq_l, self.as_l, self.ws, None)
            a.fp8_grouped_gemm_blockscaled(E_l, self.offs_l, R * K, 2 * I, H, self.aq_l, self.as_l, qw.w13, qw.s13,
                                           a.MOE_EPI_SWIGLU_REQUANT, self.actq_l, self.acts_l, st)
            a.fp8_grouped_gemm_blockscaled(E_l, self.offs_l, R * K, H, I, self.actq_l, self.acts_l, qw.w2, qw.s2,
                                           a.MOE_EPI_BF16, self.yperm_l, None, st)
            a.moe_combine(dl, self.yperm_l, self.row_of_p[:R * K], self.recv_mw[:R], None, self.y_recv[:R])
        self._all_to_all(self.y_back[:S], self.y_recv[:R], send_splits, recv_splits)
        # the shared expert on this rank's tokens, then the partial rows and the shared row
        a.fp8_grouped_gemm_blockscaled(1, self.offs_sh, T, 2 * I, H, self.xq, self.xs, qw.w13[E_l:], qw.s13[E_l:],
                                       a.MOE_EPI_SWIGLU_REQUANT, self.actq_s, self.acts_s, st)
        a.fp8_grouped_gemm_blockscaled(1, self.offs_sh, T, H, I, self.actq_s, self.acts_s, qw.w2[E_l:], qw.s2[E_l:],
                                       a.MOE_EPI_BF16, self.ysh, None, st)
        a.moe_combine(dd, self.y_back, self.row_of_s, self.ones_tk, self.ysh, self.out)
        return self.out

    def bias_update(self, gamma: float, bias: Optional[torch.Tensor] = None, stream=None):
        """b += gamma * sign(T_all*K/E - load) with every expert's load over all
        ranks' T tokens of the last forward (T_all = world * T), applied to the
        routing bias (default) or to `bias`.  Collective: every rank calls it."""
        W = self.world
        if W == 1:
            self.load_all.copy_(self.load_l)
        else:
            parts = [torch.empty_like(self.load_l) for _ in range(W)]
            dist.all_gather(parts, self.load_l, group=self.group)
            if self.placement == "block":
                # parts[r][j] is the load of global expert r * E/world + j
                self.load_all.copy_(torch.cat(parts))
            else:
                # parts[r][j] is the load of global expert j * world + r
                self.load_all.copy_(torch.stack(parts, dim=1).reshape(-1))
        self.abi.moe_bias_update(self.E, self.T * W, self.K, gamma, self.load_all,
                                 self.e_bias if bias is None else bias, stream)
