"""ctypes binding of libmoe_b200.so: argument marshalling only.

Every function here has the name of its C entry point (include/moe_b200.h),
takes torch tensors (device memory owned by the caller) or None, passes their
data pointers and the current CUDA stream, and raises MoEError on a non-zero
return code.  No arithmetic of the layer happens in Python.
"""
from __future__ import annotations

import ctypes
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libmoe_b200.so")

MOE_OK, MOE_ERR_INVALID_ARG, MOE_ERR_UNSUPPORTED, MOE_ERR_WORKSPACE, MOE_ERR_CUDA, MOE_ERR_TOO_LARGE = range(6)
MOE_FLAG_NONFINITE, MOE_FLAG_BAD_INDEX, MOE_FLAG_TIMEOUT, MOE_FLAG_BAD_OFFSETS = 1, 2, 4, 8
MOE_EPI_BF16, MOE_EPI_F32, MOE_EPI_SWIGLU_REQUANT, MOE_EPI_COMBINE_F32 = 0, 1, 2, 3
MOE_GEMM_SINGLE_CTA, MOE_GEMM_PAIR_CTA = 0x100, 0x200
MOE_EP_CYCLIC, MOE_EP_BLOCK = 0, 1


class MoEError(RuntimeError):
    def __init__(self, fn: str, code: int):
        super().__init__(f"{fn} returned {code}: {status_string(code)}")
        self.code = code


class MoeDims(ctypes.Structure):
    _fields_ = [("T", ctypes.c_int32), ("H", ctypes.c_int32), ("E", ctypes.c_int32),
                ("K", ctypes.c_int32), ("n_group", ctypes.c_int32), ("topk_group", ctypes.c_int32),
                ("I", ctypes.c_int32), ("routed_scaling_factor", ctypes.c_float)]


_LAYER_PTRS = ("w13", "s13", "w2", "s2", "w_pieces", "e_bias", "router_offset", "topk_idx", "topk_w", "scores",
               "aq", "as", "load", "offsets", "tok_of", "row_of", "actq", "acts", "yperm", "ws")


class MoeLayerC(ctypes.Structure):
    """moe_layer of the header: the dims and every device buffer of one layer."""
    _fields_ = ([("dims", MoeDims)] + [(n, ctypes.c_void_p) for n in _LAYER_PTRS] +
                [("ws_bytes", ctypes.c_size_t), ("status", ctypes.c_void_p), ("bias_out", ctypes.c_void_p),
                 ("gamma", ctypes.c_float)])


def _load() -> ctypes.CDLL:
    if not os.path.exists(LIB_PATH):
        raise ImportError(
            f"{LIB_PATH} is missing: build it with `python sparse_moe_layer_group_b200/build.py` "
            "(there is no fallback path)")
    return ctypes.CDLL(LIB_PATH)


_lib = _load()

_P, _I32, _I64, _F, _SZ = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64, ctypes.c_float, ctypes.c_size_t
_DIMS = ctypes.POINTER(MoeDims)

_SIGS = {
    "moe_status_string": (ctypes.c_char_p, [ctypes.c_int]),
    "moe_abi_version": (ctypes.c_int, []),
    "moe_workspace_size": (_SZ, [_DIMS]),
    "fp8_quant_1x128": (ctypes.c_int, [_P, _I64, _I64, _P, _P, _P, _P]),
    "fp8_quant_128x128": (ctypes.c_int, [_P, _I64, _I64, _I64, _P, _P, _P, _P]),
    "moe_route": (ctypes.c_int, [_DIMS, _P, _P, _P, _P, _P, _P, _P, _P, _SZ, _P, _P]),
    "moe_route_select": (ctypes.c_int, [_DIMS, _P, _P, _P, _P, _P]),
    "moe_router_pieces_bytes": (_SZ, [_I32, _I32]),
    "moe_router_split": (ctypes.c_int, [_P, _I32, _I32, _P, _P]),
    "moe_route_pieces": (ctypes.c_int, [_DIMS, _P, _P, _P, _P, _P, _P, _P, _P, _SZ, _P, _P]),
    "moe_permute": (ctypes.c_int, [_DIMS, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _SZ, _P, _P]),
    "moe_permute_noalloc": (ctypes.c_int, [_DIMS, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P]),
    "moe_permute_noalloc_max_scratch": (_SZ, []),
    "fp8_grouped_gemm_blockscaled": (ctypes.c_int, [_I32, _P, _I64, _I64, _I64, _P, _P, _P, _P, _I32,
                                                    _P, _P, _P, _P]),
    "fp8_grouped_gemm_blockscaled_gather": (ctypes.c_int, [_I32, _P, _I64, _I64, _I64, _P, _P, _I64, _P, _P, _P,
                                                           _I32, _P, _P, _P, _P]),
    "fp8_grouped_gemm_blockscaled_combine": (ctypes.c_int, [_I32, _P, _I64, _I64, _I64, _P, _P, _P, _P, _P, _P,
                                                            _I64, _P, _P, _P]),
    "moe_combine_finish": (ctypes.c_int, [_P, _I64, _P, _P, _I32, _P]),
    "swiglu_requant": (ctypes.c_int, [_P, _I64, _I64, _P, _P, _P, _P]),
    "fp8_quant_128x1_grouped": (ctypes.c_int, [_P, _I64, _I64, _I32, _P, _P, _I64, _P, _I64, _P, _P]),
    "fp8_grouped_gemm_wgrad": (ctypes.c_int, [_I32, _P, _I64, _I64, _I64, _P, _P, _P, _P, _I64, _I64, _P, _P,
                                              _P]),
    "moe_combine": (ctypes.c_int, [_DIMS, _P, _P, _P, _P, _P, _P, _P]),
    "moe_bias_update": (ctypes.c_int, [_I32, _I64, _I32, _F, _P, _P, _P]),
    "moe_ep_split": (ctypes.c_int, [_P, _I64, _I32, _I32, _P, _P, _P, _P]),
    "moe_ep_scatter": (ctypes.c_int, [_P, _P, _I64, _P, _P]),
    "moe_ep_plan": (ctypes.c_int, [_P, _P, _I64, _I32, _I32, _I32, _I32, _P, _P, _P, _P, _P]),
    "moe_ep_scatter_rows": (ctypes.c_int, [_P, _P, _I64, _I32, _P, _P]),
    "moe_balance_stats": (ctypes.c_int, [_DIMS, _P, _P, _P, _I32, ctypes.c_double, _P, _P, _P]),
    "moe_layer_forward": (ctypes.c_int, [ctypes.POINTER(MoeLayerC), _P, _P, _P]),
    "moe_layer_run_host": (ctypes.c_int, [ctypes.POINTER(MoeLayerC), _P, _P, _I32, _P, _P, _P]),
}
for _name, (_res, _args) in _SIGS.items():
    _f = getattr(_lib, _name)
    _f.restype = _res
    _f.argtypes = _args

EXPORTED = tuple(_SIGS)


def status_string(code: int) -> str:
    return _lib.moe_status_string(int(code)).decode()


def abi_version() -> int:
    return int(_lib.moe_abi_version())


def dims(T, H, E, K, n_group, topk_group, I, rho) -> MoeDims:
    return MoeDims(int(T), int(H), int(E), int(K), int(n_group), int(topk_group), int(I), float(rho))


def workspace_size(d: MoeDims) -> int:
    return int(_lib.moe_workspace_size(ctypes.byref(d)))


def _ptr(t):
    if t is None:
        return None
    if isinstance(t, int):
        return t
    return t.data_ptr()


def _stream(stream):
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


def _check(fn: str, rc: int):
    if rc != MOE_OK:
        raise MoEError(fn, rc)


def fp8_quant_1x128(x, q, scales, status=None, stream=None):
    rows, cols = x.shape
    _check("fp8_quant_1x128", _lib.fp8_quant_1x128(_ptr(x), rows, cols, _ptr(q), _ptr(scales),
                                                   _ptr(status), _stream(stream)))


def fp8_quant_128x128(w, q, scales, status=None, stream=None):
    if w.dim() == 2:
        batch, (rows, cols) = 1, w.shape
    else:
        batch, rows, cols = w.shape
    _check("fp8_quant_128x128", _lib.fp8_quant_128x128(_ptr(w), batch, rows, cols, _ptr(q), _ptr(scales),
                                                       _ptr(status), _stream(stream)))


def moe_route(d, x, w_router, e_bias, router_offset, topk_idx, topk_w, scores=None, ws=None,
              status=None, stream=None):
    ws_bytes = 0 if ws is None else ws.numel() * ws.element_size()
    _check("moe_route", _lib.moe_route(ctypes.byref(d), _ptr(x), _ptr(w_router), _ptr(e_bias),
                                       _ptr(router_offset), _ptr(topk_idx), _ptr(topk_w), _ptr(scores),
                                       _ptr(ws), ws_bytes, _ptr(status), _stream(stream)))


def moe_router_pieces_bytes(E, H) -> int:
    return int(_lib.moe_router_pieces_bytes(int(E), int(H)))


def moe_router_split(w_router, w_pieces, stream=None):
    E, H = w_router.shape
    _check("moe_router_split", _lib.moe_router_split(_ptr(w_router), E, H, _ptr(w_pieces), _stream(stream)))


def moe_route_pieces(d, x, w_pieces, e_bias, router_offset, topk_idx, topk_w, scores=None, ws=None,
                     status=None, stream=None):
    ws_bytes = 0 if ws is None else ws.numel() * ws.element_size()
    _check("moe_route_pieces", _lib.moe_route_pieces(ctypes.byref(d), _ptr(x), _ptr(w_pieces), _ptr(e_bias),
                                                     _ptr(router_offset), _ptr(topk_idx), _ptr(topk_w),
                                                     _ptr(scores), _ptr(ws), ws_bytes, _ptr(status),
                                                     _stream(stream)))


def moe_route_select(d, scores, e_bias, topk_idx, topk_w, stream=None):
    _check("moe_route_select", _lib.moe_route_select(ctypes.byref(d), _ptr(scores), _ptr(e_bias),
                                                     _ptr(topk_idx), _ptr(topk_w), _stream(stream)))


def moe_permute(d, topk_idx, xq, xs, expert_load, expert_offsets, tok_of, row_of, aq, as_, ws,
                status=None, stream=None):
    ws_bytes = 0 if ws is None else ws.numel() * ws.element_size()
    _check("moe_permute", _lib.moe_permute(ctypes.byref(d), _ptr(topk_idx), _ptr(xq), _ptr(xs),
                                           _ptr(expert_load), _ptr(expert_offsets), _ptr(tok_of),
                                           _ptr(row_of), _ptr(aq), _ptr(as_), _ptr(ws), ws_bytes,
                                           _ptr(status), _stream(stream)))


def moe_permute_noalloc(d, topk_idx, xq, xs, expert_load, expert_offsets, tok_of, row_of, aq, as_,
                        status=None, stream=None):
    """moe_permute without a workspace (static device scratch; see the header)."""
    _check("moe_permute_noalloc", _lib.moe_permute_noalloc(
        ctypes.byref(d), _ptr(topk_idx), _ptr(xq), _ptr(xs), _ptr(expert_load), _ptr(expert_offsets),
        _ptr(tok_of), _ptr(row_of), _ptr(aq), _ptr(as_), _ptr(status), _stream(stream)))


def moe_permute_noalloc_max_scratch() -> int:
    return int(_lib.moe_permute_noalloc_max_scratch())


def fp8_grouped_gemm_blockscaled(G, group_offsets, m_capacity, N, K, A, sA, B, sB, epilogue, C, sC=None,
                                 status=None, stream=None):
    _check("fp8_grouped_gemm_blockscaled", _lib.fp8_grouped_gemm_blockscaled(
        int(G), _ptr(group_offsets), int(m_capacity), int(N), int(K), _ptr(A), _ptr(sA), _ptr(B), _ptr(sB),
        int(epilogue), _ptr(C), _ptr(sC), _ptr(status), _stream(stream)))


def fp8_grouped_gemm_blockscaled_gather(G, group_offsets, m_capacity, N, K, A, sA, a_map, B, sB, epilogue, C,
                                        sC=None, status=None, stream=None):
    """A: e4m3 [a_rows, K] source rows, a_map int32 [m_capacity] (GEMM row -> A row)."""
    _check("fp8_grouped_gemm_blockscaled_gather", _lib.fp8_grouped_gemm_blockscaled_gather(
        int(G), _ptr(group_offsets), int(m_capacity), int(N), int(K), _ptr(A), _ptr(sA), int(A.shape[0]),
        _ptr(a_map), _ptr(B), _ptr(sB), int(epilogue), _ptr(C), _ptr(sC), _ptr(status), _stream(stream)))


def fp8_grouped_gemm_blockscaled_combine(G, group_offsets, m_capacity, N, K, A, sA, B, sB, row_token, row_gate,
                                         out_f32, status=None, stream=None):
    """out_f32[row_token[m], :] += row_gate[m] * bf16(row m of the GEMM), fp32 [out_rows, N]."""
    _check("fp8_grouped_gemm_blockscaled_combine", _lib.fp8_grouped_gemm_blockscaled_combine(
        int(G), _ptr(group_offsets), int(m_capacity), int(N), int(K), _ptr(A), _ptr(sA), _ptr(B), _ptr(sB),
        _ptr(row_token), _ptr(row_gate), int(out_f32.shape[0]), _ptr(out_f32), _ptr(status), _stream(stream)))


def moe_combine_finish(acc, out_bf16, out_f32=None, zero: bool = True, stream=None):
    _check("moe_combine_finish", _lib.moe_combine_finish(_ptr(acc), acc.numel(), _ptr(out_bf16), _ptr(out_f32),
                                                         1 if zero else 0, _stream(stream)))


def wgrad_capacities(M: int, G: int) -> tuple:
    """(p_capacity, t_capacity) that fit any grouping of M rows into G groups."""
    t_cap = (M + 127) // 128 + G
    return 128 * t_cap, t_cap


def fp8_quant_128x1_grouped(x, group_offsets, q_t, scales, status=None, stream=None):
    M, C = x.shape
    G = group_offsets.numel() - 1
    _check("fp8_quant_128x1_grouped", _lib.fp8_quant_128x1_grouped(
        _ptr(x), M, C, G, _ptr(group_offsets), _ptr(q_t), q_t.shape[1], _ptr(scales), scales.shape[0],
        _ptr(status), _stream(stream)))


def fp8_grouped_gemm_wgrad(group_offsets, M, dy_t, sdy, x_t, sx, dW, status=None, stream=None):
    G = group_offsets.numel() - 1
    N, K = dy_t.shape[0], x_t.shape[0]
    _check("fp8_grouped_gemm_wgrad", _lib.fp8_grouped_gemm_wgrad(
        G, _ptr(group_offsets), int(M), N, K, _ptr(dy_t), _ptr(sdy), _ptr(x_t), _ptr(sx), dy_t.shape[1],
        sdy.shape[0], _ptr(dW), _ptr(status), _stream(stream)))


def swiglu_requant(gu, q, s, status=None, stream=None):
    M, two_i = gu.shape
    _check("swiglu_requant", _lib.swiglu_requant(_ptr(gu), M, two_i // 2, _ptr(q), _ptr(s), _ptr(status),
                                                 _stream(stream)))


def moe_combine(d, yperm, row_of, topk_w, yshared, out, out_f32=None, stream=None):
    _check("moe_combine", _lib.moe_combine(ctypes.byref(d), _ptr(yperm), _ptr(row_of), _ptr(topk_w),
                                           _ptr(yshared), _ptr(out), _ptr(out_f32), _stream(stream)))


def moe_ep_split(topk_idx, E, world, dest_rank, local_idx, status=None, stream=None):
    _check("moe_ep_split", _lib.moe_ep_split(_ptr(topk_idx), topk_idx.numel(), int(E), int(world), _ptr(dest_rank),
                                             _ptr(local_idx), _ptr(status), _stream(stream)))


def moe_ep_scatter(row_of, values, out, stream=None):
    _check("moe_ep_scatter", _lib.moe_ep_scatter(_ptr(row_of), _ptr(values), row_of.numel(), _ptr(out),
                                                 _stream(stream)))


def moe_bias_update(E, T, K, gamma, expert_load, e_bias, stream=None):
    _check("moe_bias_update", _lib.moe_bias_update(int(E), int(T), int(K), float(gamma), _ptr(expert_load),
                                                   _ptr(e_bias), _stream(stream)))


def moe_balance_stats(d, scores, topk_idx, expert_load, seq_len, alpha, seq_loss, entropy, stream=None):
    _check("moe_balance_stats", _lib.moe_balance_stats(ctypes.byref(d), _ptr(scores), _ptr(topk_idx),
                                                       _ptr(expert_load), int(seq_len), float(alpha),
                                                       _ptr(seq_loss), _ptr(entropy), _stream(stream)))


def moe_ep_plan(topk_idx, topk_w, E, world, placement, dest_rank, meta_ids, meta_w, status=None, stream=None):
    T, K = topk_idx.shape
    _check("moe_ep_plan", _lib.moe_ep_plan(_ptr(topk_idx), _ptr(topk_w), int(T), int(K), int(E), int(world),
                                           int(placement),
                                           _ptr(dest_rank), _ptr(meta_ids), _ptr(meta_w), _ptr(status),
                                           _stream(stream)))


def moe_ep_scatter_rows(row_of, values, out, stream=None):
    """out[row_of[i], :] = values[i, :] for int32 (or fp32, moved as bits) rows."""
    n, width = values.shape
    _check("moe_ep_scatter_rows", _lib.moe_ep_scatter_rows(_ptr(row_of), _ptr(values), int(n), int(width),
                                                           _ptr(out), _stream(stream)))


def moe_layer(d, buffers: dict, ws, status=None, bias_out=None, gamma: float = 0.0) -> MoeLayerC:
    """Fill a moe_layer from device tensors: buffers maps each pointer field of
    the header's struct (w13, s13, ..., yperm) to a tensor (router_offset may be None)."""
    L = MoeLayerC()
    L.dims = d
    for n in _LAYER_PTRS:
        setattr(L, n, _ptr(ws if n == "ws" else buffers.get(n)))
    L.ws_bytes = 0 if ws is None else ws.numel() * ws.element_size()
    L.status = _ptr(status)
    L.bias_out = _ptr(bias_out)
    L.gamma = float(gamma)
    return L


def moe_layer_forward(L: MoeLayerC, x, out, stream=None):
    _check("moe_layer_forward", _lib.moe_layer_forward(ctypes.byref(L), _ptr(x), _ptr(out), _stream(stream)))


def moe_layer_run_host(L: MoeLayerC, x_host, out_host, x_dev, out_dev, stream=None):
    """Batches x_host[i] -> out_host[i] (pinned host tensors) through the device
    double buffers x_dev[0..1], out_dev[0..1]; returns once enqueued."""
    n = len(x_host)
    if len(out_host) != n or len(x_dev) != 2 or len(out_dev) != 2:
        raise ValueError("n host inputs and outputs, two device inputs and outputs")
    xs = (ctypes.c_void_p * n)(*[_ptr(t) for t in x_host])
    os_ = (ctypes.c_void_p * n)(*[_ptr(t) for t in out_host])
    xd = (ctypes.c_void_p * 2)(*[_ptr(t) for t in x_dev])
    od = (ctypes.c_void_p * 2)(*[_ptr(t) for t in out_dev])
    _check("moe_layer_run_host", _lib.moe_layer_run_host(ctypes.byref(L), xs, os_, n, xd, od, _stream(stream)))
