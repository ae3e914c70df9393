"""B200-native (sm_100a) DeepSeekMoE layer forward: FP8 block-scaled grouped GEMMs
on tcgen05/TMEM tensor cores behind a small C ABI (include/moe_b200.h).

Importing this package loads libmoe_b200.so and fails loudly if it is missing;
there is no CPU or PyTorch fallback for any step of the layer.
"""
from . import _abi as abi
from ._abi import (MOE_EPI_BF16, MOE_EPI_F32, MOE_EPI_SWIGLU_REQUANT, MOE_FLAG_BAD_INDEX,
                   MOE_FLAG_BAD_OFFSETS, MOE_FLAG_NONFINITE, MOE_FLAG_TIMEOUT, MoEError, dims,
                   fp8_grouped_gemm_blockscaled, fp8_grouped_gemm_blockscaled_gather,
                   fp8_grouped_gemm_blockscaled_combine, moe_combine_finish, MOE_EPI_COMBINE_F32, fp8_quant_128x128, fp8_quant_1x128, moe_bias_update,
                   moe_balance_stats, moe_combine, moe_permute, moe_route, moe_route_pieces, moe_route_select,
                   moe_router_pieces_bytes, moe_router_split, swiglu_requant, fp8_quant_128x1_grouped,
                   fp8_grouped_gemm_wgrad, wgrad_capacities, moe_ep_split, moe_ep_scatter, moe_ep_plan,
                   moe_ep_scatter_rows, MOE_EP_CYCLIC, MOE_EP_BLOCK,
                   workspace_size)
from .ep import EPMoELayer
from .layer import LAUNCHES_PER_FORWARD, MoELayer, QuantWeights

__all__ = [
    "abi", "MoEError", "dims", "workspace_size", "fp8_quant_1x128", "fp8_quant_128x128", "moe_route",
    "moe_route_select", "moe_route_pieces", "moe_router_split", "moe_router_pieces_bytes", "moe_permute", "fp8_grouped_gemm_blockscaled",
    "fp8_grouped_gemm_blockscaled_gather", "fp8_grouped_gemm_blockscaled_combine", "moe_combine_finish",
    "MOE_EPI_COMBINE_F32", "swiglu_requant", "moe_combine",
    "moe_bias_update", "moe_balance_stats", "fp8_quant_128x1_grouped", "fp8_grouped_gemm_wgrad",
    "wgrad_capacities", "moe_ep_split", "moe_ep_scatter", "moe_ep_plan", "moe_ep_scatter_rows",
    "MOE_EP_CYCLIC", "MOE_EP_BLOCK", "EPMoELayer", "MoELayer", "QuantWeights", "LAUNCHES_PER_FORWARD",
    "MOE_EPI_BF16", "MOE_EPI_F32", "MOE_EPI_SWIGLU_REQUANT",
    "MOE_FLAG_NONFINITE", "MOE_FLAG_BAD_INDEX", "MOE_FLAG_TIMEOUT", "MOE_FLAG_BAD_OFFSETS",
]
