"""CPU oracle of the DeepSeekMoE layer forward -- TEST INFRASTRUCTURE ONLY.

A plain, slow, obviously correct restatement of what the layer computes, in
numpy float64, written from the pages and nothing else.  Only the test suite
(`tests/`), the graft entry's `smoke()` and the CPU-baseline leg of
`bench.py` may import it.  The product path (the CUDA library and its Python
binding) never touches this package, and this package never touches the
product path: the two share no code.  Their only common input is the seeded
generator module `synth`.

Sources (page titles as fetched; sections as numbered on each page):

* [report-walkthrough] "DeepSeek-V3 technical report" walkthrough (2kiu.com):
  section 3.2 "the bias only changes the ranking, not the value" (router,
  gate, bias-update pseudocode), section 3.4 "node-limited routing",
  section 4.3 "FP8: block scaling and high-precision accumulation".
* [repro-guide] "From technical report to a runnable config: DeepSeek-V3's
  MoE/MLA/FP8" (lpnh.cn), section 3 "copyable config" (num_experts 256,
  num_experts_per_tok 8, moe_intermediate_size 2048, norm_topk_prob,
  routed_scaling_factor 2.5, e4m3, 1x128 input tiles, 128x128 weight
  blocks, moe_gating kept in high precision).
* [infra-answer] Zhihu answer on DeepSeek-V3's infrastructure (question
  7837132971): E4M3 throughout, per-tile 1x128 and per-group 128x128
  scaling, products promoted as partial sums because the hardware has no
  micro-scaling support.
* [arch-overview] "DeepSeek-V3 MoE architecture and FP8 training" (0539edu.com):
  1 shared + 256 routed experts, expert intermediate 2048, hidden 7168.
* The OCP 8-bit floating point specification (OFP8), E4M3 format, for the
  encoder and decoder.

Pins: every function here is checked in `tests/test_oracle_*.py` against
something other than itself (hand-derived codes, brute force over all
subsets, closed forms, library routines, integer-exact products).  No
function is "parity unpinned".
"""
from .fp8 import (E4M3_MAX, e4m3_encode, e4m3_decode, e4m3_encode_scalar, e4m3_decode_scalar,
                  round_bf16, quant_1x128, quant_128x128, dequant_1x128, dequant_128x128)
from .routing import (router_scores, select_experts, select_experts_bruteforce,
                      expert_load, bias_update, seq_balance_loss, load_entropy)
from .dispatch import permute, unpermute_rows, combine, combine_by_rank
from .expert import (gemm_blockscaled, grouped_gemm_blockscaled, silu, swiglu,
                     swiglu_requant, expert_ffn)
from .layer import LayerWeights, quantize_layer_weights, moe_forward, moe_forward_tokens

__all__ = [
    "E4M3_MAX", "e4m3_encode", "e4m3_decode", "e4m3_encode_scalar", "e4m3_decode_scalar",
    "round_bf16", "quant_1x128", "quant_128x128", "dequant_1x128", "dequant_128x128",
    "router_scores", "select_experts", "select_experts_bruteforce", "expert_load", "bias_update",
    "seq_balance_loss", "load_entropy",
    "permute", "unpermute_rows", "combine", "combine_by_rank",
    "gemm_blockscaled", "grouped_gemm_blockscaled", "silu", "swiglu", "swiglu_requant", "expert_ffn",
    "LayerWeights", "quantize_layer_weights", "moe_forward", "moe_forward_tokens",
]
from .backward import quant_128x1, dgrad_blockscaled, wgrad_blockscaled
