"""DeepSeekMoE layer forward on one B200, chaining the C-ABI calls.

PyTorch only allocates device memory and supplies the stream; every step of
the forward runs in the library's kernels:

  1  moe_route_pieces router GEMM (tensor cores, on the bf16 pieces of W_r split
                      once at construction) + sigmoid, group-limited top-K,
                      gates (2 kernels)
  2  fp8_quant_1x128  x -> e4m3 codes + 1x128 scales, written straight into the
                      last T rows of the expert-ordered A matrix
  3  moe_permute      stable counting sort by expert + row gather (4 kernels)
                      into the first T*K rows
  4  grouped GEMM     W13 of the E routed experts and, as group E, of the
                      shared expert over the T token rows; SwiGLU + 1x128
                      requant fused.  With gather=True the permute writes only
                      the maps (3 kernels) and the GEMM fetches each routed row
                      from the token's quantised row through tok_of with TMA
                      row gathers, so the permuted copy is never written; same
                      bits, but measured slower on B200 at the DeepSeek-V3
                      shape (32 four-row gathers per A tile instead of one
                      tiled load), hence not the default
  5  grouped GEMM     W2 of the same E + 1 groups -> bf16 rows
  6  moe_combine      gate-weighted sum of the K rows + the shared row -> bf16.
                      With fused_combine=True the W2 GEMM adds each gated row
                      into an fp32 accumulator of the output itself (no rows
                      stored; additions in no fixed order) and
                      moe_combine_finish rounds it to bf16
  (7 moe_bias_update  after the step, from the expert loads of step 3)

Treating the shared expert as one more group of the same two launches lets its
compute-bound tiles run in the tail of the weight-bound routed tiles.  Order and
arithmetic follow the "DeepSeek-V3 technical report" walkthrough (2kiu.com),
sections 3.2, 3.4 and 4.3.
"""
from __future__ import annotations

from dataclasses import dataclass
from typing import Callable, Optional

import torch

from . import _abi as abi

LAUNCHES_PER_FORWARD = 10   # 2 route + 1 quant + 4 permute + 2 GEMM + 1 combine (gather=True: 9)


@dataclass
class QuantWeights:
    """128x128 block-quantised expert weights resident in HBM, routed experts
    0..E-1 and the shared expert as expert E.

    w13 e4m3 [E+1, 2I, H] (gate rows 0..I-1, up rows I..2I-1), s13 fp32
    [E+1, 2I/128, H/128]; w2 e4m3 [E+1, H, I], s2 fp32 [E+1, H/128, I/128]."""
    w13: torch.Tensor
    s13: torch.Tensor
    w2: torch.Tensor
    s2: torch.Tensor

    @property
    def E(self) -> int:
        return self.w13.shape[0] - 1

    @property
    def nbytes(self) -> int:
        return sum(t.numel() * t.element_size() for t in (self.w13, self.s13, self.w2, self.s2))

    @staticmethod
    def from_master(master: Callable[[str, int], torch.Tensor], E: int, H: int, I: int,
                    device="cuda", status: Optional[torch.Tensor] = None) -> "QuantWeights":
        """Quantise master weights expert by expert with fp8_quant_128x128.

        master(kind, e) returns a bf16 tensor: kind "w13" -> [2I, H], "w2" ->
        [H, I]; e = -1 is the shared expert (stored as expert E)."""
        u8 = dict(dtype=torch.uint8, device=device)
        f32 = dict(dtype=torch.float32, device=device)
        w13 = torch.empty(E + 1, 2 * I, H, **u8)
        s13 = torch.empty(E + 1, 2 * I // 128, H // 128, **f32)
        w2 = torch.empty(E + 1, H, I, **u8)
        s2 = torch.empty(E + 1, H // 128, I // 128, **f32)
        for e in range(-1, E):
            slot = E if e < 0 else e
            a = master("w13", e).to(device).contiguous()
            abi.fp8_quant_128x128(a, w13[slot], s13[slot], status)
            del a
            b = master("w2", e).to(device).contiguous()
            abi.fp8_quant_128x128(b, w2[slot], s2[slot], status)
            del b
        return QuantWeights(w13, s13, w2, s2)


class MoELayer:
    """One layer for a fixed token count T, with all buffers preallocated."""

    def __init__(self, T: int, H: int, E: int, K: int, n_group: int, topk_group: int, I: int,
                 rho: float, w_router: torch.Tensor, e_bias: torch.Tensor, weights: QuantWeights,
                 router_offset: Optional[torch.Tensor] = None, device="cuda", gather: bool = False,
                 fused_combine: bool = False):
        self.T, self.H, self.E, self.K, self.I = T, H, E, K, I
        self.gather, self.fused_combine = gather, fused_combine
        # the fused combine adds a gate scatter and a finishing pass and drops the combine kernel
        self.launches_per_forward = LAUNCHES_PER_FORWARD - (1 if gather else 0) + (1 if fused_combine else 0)
        self.n_group, self.topk_group, self.rho = n_group, topk_group, rho
        self.d = abi.dims(T, H, E, K, n_group, topk_group, I, rho)
        self.w_router, self.e_bias, self.router_offset = w_router, e_bias, router_offset
        # the router weights' three exact bf16 pieces, split once (refresh_router
        # after changing w_router)
        self.w_pieces = torch.empty(abi.moe_router_pieces_bytes(E, H) // 2, dtype=torch.bfloat16, device=device)
        self.refresh_router()
        self.qw = weights
        assert weights.E == E, "weights hold E routed experts plus the shared one"
        dev = dict(device=device)
        i32 = dict(dtype=torch.int32, **dev)
        f32 = dict(dtype=torch.float32, **dev)
        u8 = dict(dtype=torch.uint8, **dev)
        bf = dict(dtype=torch.bfloat16, **dev)
        TK = T * K
        self.topk_idx = torch.empty(T, K, **i32)
        self.topk_w = torch.empty(T, K, **f32)
        self.scores = torch.empty(T, E, **f32)
        ws_bytes = max(abi.workspace_size(self.d), 256)
        self.ws = torch.empty((ws_bytes + 255) // 256 * 256, **u8)
        # rows of the first GEMM: rows 0..T*K-1 the routed (token, slot) pairs in
        # expert order, rows T*K..T*K+T-1 the tokens themselves (shared expert)
        # token of every row: tok_of (written by moe_permute), then 0..T-1
        self.rows_tok = torch.empty(TK + T, **i32)
        self.rows_tok[TK:] = torch.arange(T, **i32)
        self.tok_of = self.rows_tok[:TK]
        if gather:
            # read through rows_tok from the T quantised token rows
            self.aq = self.as_ = None
            self.xq = torch.empty(T, H, **u8)
            self.xs = torch.empty(T, H // 128, **f32)
            self.a_map = self.rows_tok
        else:
            # a materialised copy in that order; the last T rows are the quantiser's output
            self.aq = torch.empty(TK + T, H, **u8)
            self.as_ = torch.empty(TK + T, H // 128, **f32)
            self.xq = self.aq[TK:]
            self.xs = self.as_[TK:]
            self.a_map = None
        self.load = torch.empty(E, **i32)
        # group offsets of the E + 1 groups: moe_permute writes entries 0..E,
        # entry E + 1 closes the shared group
        self.offsets_all = torch.full((E + 2,), TK + T, **i32)
        self.offsets = self.offsets_all[:E + 1]
        self.row_of = torch.empty(TK, **i32)
        self.actq = torch.empty(TK + T, I, **u8)
        self.acts = torch.empty(TK + T, I // 128, **f32)
        if fused_combine:
            # gate of every row in row order (1 for the shared expert's rows) and the
            # fp32 accumulator of the output (zero between forwards)
            self.row_gate = torch.ones(TK + T, **f32)
            self.out_acc = torch.zeros(T, H, **f32)
            self.yperm = self.ysh = None
        else:
            self.yperm = torch.empty(TK + T, H, **bf)
            self.ysh = self.yperm[TK:]
        self.out = torch.empty(T, H, **bf)
        self.out_f32 = None
        self.status = torch.zeros(1, **i32)

    def forward(self, x: torch.Tensor, out_f32: bool = False, stream=None, gemm_events=None,
                out: Optional[torch.Tensor] = None) -> torch.Tensor:
        """x bf16 [T, H] on the device -> out bf16 [T, H] (self.out, or `out` if
        given: a caller-owned contiguous bf16 [T, H] device tensor, e.g. one of
        two buffers while the previous result is still being copied out).

        gemm_events, if given, is a triple of CUDA events recorded on the
        launching stream before the W13 grouped GEMM, between W13 and W2, and
        after W2."""
        T, H, E, K, I = self.T, self.H, self.E, self.K, self.I
        if out is None:
            out = self.out
        elif (out.dtype != torch.bfloat16 or tuple(out.shape) != (T, H) or not out.is_contiguous()
              or out.device != self.out.device):
            raise ValueError("out must be a contiguous bf16 [T, H] tensor on the layer's device")
        if T == 0:
            return out
        if out_f32 and self.out_f32 is None:
            self.out_f32 = torch.empty(T, H, dtype=torch.float32, device=self.out.device)
        st = self.status
        M = T * K + T
        abi.moe_route_pieces(self.d, x, self.w_pieces, self.e_bias, self.router_offset, self.topk_idx,
                             self.topk_w, self.scores, self.ws, st, stream)
        abi.fp8_quant_1x128(x, self.xq, self.xs, st, stream)
        if self.gather:
            abi.moe_permute(self.d, self.topk_idx, None, None, self.load, self.offsets, self.tok_of,
                            self.row_of, None, None, self.ws, st, stream)
        else:
            abi.moe_permute(self.d, self.topk_idx, self.xq, self.xs, self.load, self.offsets, self.tok_of,
                            self.row_of, self.aq, self.as_, self.ws, st, stream)
        qw = self.qw
        ev_stream = torch.cuda.current_stream() if stream is None else stream
        if gemm_events is not None:
            gemm_events[0].record(ev_stream)
        if self.gather:
            abi.fp8_grouped_gemm_blockscaled_gather(E + 1, self.offsets_all, M, 2 * I, H, self.xq, self.xs,
                                                    self.a_map, qw.w13, qw.s13, abi.MOE_EPI_SWIGLU_REQUANT,
                                                    self.actq, self.acts, st, stream)
        else:
            abi.fp8_grouped_gemm_blockscaled(E + 1, self.offsets_all, M, 2 * I, H, self.aq, self.as_, qw.w13,
                                             qw.s13, abi.MOE_EPI_SWIGLU_REQUANT, self.actq, self.acts, st, stream)
        if gemm_events is not None:
            gemm_events[1].record(ev_stream)
        if self.fused_combine:
            # the gates into row order (fp32 moved as its bit pattern), then W2 adds
            # every gated row into the output accumulator
            abi.moe_ep_scatter(self.row_of, self.topk_w.view(torch.int32), self.row_gate[:T * K].view(torch.int32),
                               stream)
            abi.fp8_grouped_gemm_blockscaled_combine(E + 1, self.offsets_all, M, H, I, self.actq, self.acts, qw.w2,
                                                     qw.s2, self.rows_tok, self.row_gate, self.out_acc, st, stream)
            if gemm_events is not None:
                gemm_events[2].record(ev_stream)
            abi.moe_combine_finish(self.out_acc, out, self.out_f32 if out_f32 else None, True, stream)
            return out
        abi.fp8_grouped_gemm_blockscaled(E + 1, self.offsets_all, M, H, I, self.actq, self.acts, qw.w2, qw.s2,
                                         abi.MOE_EPI_BF16, self.yperm, None, st, stream)
        if gemm_events is not None:
            gemm_events[2].record(ev_stream)
        abi.moe_combine(self.d, self.yperm, self.row_of, self.topk_w, self.ysh, out,
                        self.out_f32 if out_f32 else None, stream)
        return out

    def native(self, bias_out: Optional[torch.Tensor] = None, gamma: float = 0.0) -> "abi.MoeLayerC":
        """The header's moe_layer for this layer's buffers (the materialised
        path), for moe_layer_forward / moe_layer_run_host: the whole forward,
        and the bias update into bias_out if given, behind one C call."""
        if self.gather or self.fused_combine:
            raise ValueError("the one-call forward runs the materialised path (gather=False, fused_combine=False)")
        qw = self.qw
        bufs = dict(w13=qw.w13, s13=qw.s13, w2=qw.w2, s2=qw.s2, w_pieces=self.w_pieces, e_bias=self.e_bias,
                    router_offset=self.router_offset, topk_idx=self.topk_idx, topk_w=self.topk_w,
                    scores=self.scores, aq=self.aq, load=self.load, offsets=self.offsets_all,
                    tok_of=self.tok_of, row_of=self.row_of, actq=self.actq, acts=self.acts, yperm=self.yperm)
        bufs["as"] = self.as_
        return abi.moe_layer(self.d, bufs, self.ws, self.status, bias_out, gamma)

    def forward_native(self, x: torch.Tensor, out: Optional[torch.Tensor] = None, stream=None,
                       bias_out: Optional[torch.Tensor] = None, gamma: float = 0.0) -> torch.Tensor:
        """forward() as one C call (moe_layer_forward); same kernels, same bits."""
        out = self.out if out is None else out
        abi.moe_layer_forward(self.native(bias_out, gamma), x, out, stream)
        return out

    def run_host(self, x_host, out_host, x_dev, out_dev, stream=None, bias_out: Optional[torch.Tensor] = None,
                 gamma: float = 0.0):
        """Batches from pinned host memory through moe_layer_run_host: uploads and
        downloads of neighbouring batches overlap each forward (two device input
        and output buffers).  Returns once enqueued on `stream`."""
        abi.moe_layer_run_host(self.native(bias_out, gamma), x_host, out_host, x_dev, out_dev, stream)

    def capture_graph(self, x: torch.Tensor, gamma: Optional[float] = None,
                      bias: Optional[torch.Tensor] = None) -> "torch.cuda.CUDAGraph":
        """Capture one forward on the device tensor x (and, with gamma, the bias
        update into `bias` or the routing bias) as a CUDA graph.  Replaying it
        reruns the same kernels on whatever x then holds, writing self.out,
        without per-launch host work.  One eager forward on a side stream runs
        first, so that every kernel's one-time setup happens outside the
        capture."""
        side = torch.cuda.Stream(device=x.device)
        side.wait_stream(torch.cuda.current_stream(x.device))
        with torch.cuda.stream(side):
            self.forward(x)
        torch.cuda.current_stream(x.device).wait_stream(side)
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph):
            self.forward(x)
            if gamma is not None:
                self.bias_update(gamma, bias=bias)
        return graph

    def refresh_router(self, stream=None):
        """Split the router weights into the pieces the forward routes with."""
        abi.moe_router_split(self.w_router, self.w_pieces, stream)

    def bias_update(self, gamma: float, stream=None, bias: Optional[torch.Tensor] = None):
        """b += gamma * sign(T*K/E - load) from this step's expert loads, into
        the routing bias (default) or into `bias` (keeps the routing fixed)."""
        abi.moe_bias_update(self.E, self.T, self.K, gamma, self.load, self.e_bias if bias is None else bias, stream)

    def balance_stats(self, seq_len: int, alpha: float = 0.001, stream=None):
        """(per-sequence balance loss float64 [T/seq_len], load entropy float64 [1])
        of the last forward, computed on the device."""
        loss = torch.empty(self.T // seq_len, dtype=torch.float64, device=self.out.device)
        ent = torch.empty(1, dtype=torch.float64, device=self.out.device)
        abi.moe_balance_stats(self.d, self.scores, self.topk_idx, self.load, seq_len, alpha, loss, ent, stream)
        return loss, ent

    # ---- algorithmic work of one forward (for throughput and roofline figures)
    def flops(self) -> dict:
        T, H, K, I = self.T, self.H, self.K, self.I
        routed = 2 * T * K * (2 * I * H + H * I)
        shared = 2 * T * (2 * I * H + H * I)
        router = 2 * T * self.E * H
        return dict(routed=routed, shared=shared, router=router, total=routed + shared + router)
