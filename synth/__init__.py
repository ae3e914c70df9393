"""Seeded synthetic inputs for the DeepSeekMoE layer forward.

This module is the only code shared by the CPU oracle and the CUDA path.  It
draws random numbers and shapes them into the workloads described below; it
holds none of the layer's arithmetic (no routing, no quantisation, no GEMM).

Every generator takes an explicit integer seed and a torch device and returns
torch tensors.  The same seed on the same device always yields the same bits
(torch's CPU generator on "cpu", its Philox generator on "cuda").  A CPU draw
and a CUDA draw of the same seed are NOT the same numbers; a test draws once
and hands the same tensor to both sides.

Workload recipes (the pages' layer: hidden 7168, 256 routed + 1 shared
expert, top-8, expert intermediate 2048 -- "DeepSeek-V3 technical-report
walkthrough" (2kiu.com), sections 1 and 3; "Reproduction guide: from the
technical report to a runnable config" (lpnh.cn), section 3):

* activations x: bf16 N(0, 1); optionally a seeded 0.1 % of the hidden
  channels (the same channels for every token) scaled by 50 as outliers;
* router weights W_r: fp32 N(0, std) with std 0.02 (tiny) or 0.006 (DSV3);
* expert weights: bf16 N(0, std), drawn per expert from its own seed so any
  one expert can be regenerated alone;
* expert bias b: fp32 U(lo, hi) (tiny) or zeros (DSV3);
* skewed routing: a per-expert additive router-logit offset from a Zipf(1.1)
  ranking, o_e = -kappa * 1.1 * ln(rank_e), rank a seeded permutation of 1..E;
* GEMM sweep: A bf16 N(0, 1) with 1 % of the entries times 100, B N(0, 0.02);
  group sizes a uniform random composition (255 sorted uniform cut points).
"""
from __future__ import annotations

import math
from dataclasses import dataclass

import torch

__all__ = [
    "MoEShape", "TINY", "DSV3", "PREFILL", "DECODE", "MID",
    "gen", "activations", "router_weights", "expert_bias", "expert_weight",
    "zipf_offset", "scores", "topk_indices", "heavy_tailed", "normal",
    "group_sizes", "seed_of",
]


@dataclass(frozen=True)
class MoEShape:
    """One layer shape: T tokens, H hidden, E routed experts, K top-k,
    n_group groups with topk_group kept, I expert intermediate, rho the
    routed scaling factor, plus the synthetic-input recipe."""
    name: str
    T: int
    H: int
    E: int
    K: int
    n_group: int
    topk_group: int
    I: int
    rho: float = 2.5
    x_outlier_frac: float = 0.0
    x_outlier_scale: float = 50.0
    wr_std: float = 0.02
    w_std: float = 0.02
    bias_range: float = 0.0   # b ~ U(-bias_range, bias_range); 0 means b = 0
    seed_base: int = 0


# Named workloads (sizes as the pages give them).
TINY = MoEShape("tiny", T=64, H=256, E=16, K=4, n_group=4, topk_group=2, I=128,
                wr_std=0.02, w_std=0.02, bias_range=0.01, seed_base=0)
DSV3 = MoEShape("dsv3", T=4096, H=7168, E=256, K=8, n_group=8, topk_group=4, I=2048,
                x_outlier_frac=0.001, wr_std=0.006, w_std=0.006, seed_base=2000)
PREFILL = MoEShape("prefill_skew", T=32768, H=7168, E=256, K=8, n_group=8, topk_group=4,
                   I=2048, x_outlier_frac=0.001, wr_std=0.006, w_std=0.006, seed_base=3000)
DECODE = MoEShape("decode", T=128, H=7168, E=256, K=8, n_group=8, topk_group=4, I=2048,
                  wr_std=0.006, w_std=0.006, seed_base=4000)
# A mid-size shape for parity: several M, N and K tiles and ragged tails.
MID = MoEShape("mid", T=300, H=512, E=32, K=4, n_group=4, topk_group=2, I=256,
               x_outlier_frac=0.01, wr_std=0.02, w_std=0.02, bias_range=0.01, seed_base=500)


def seed_of(shape_or_base, tensor_id: int, sub: int = 0) -> int:
    """Seed of one tensor of a workload: seed_base*1000 + tensor_id, plus
    sub*100003 for per-expert tensors (sub = expert number)."""
    base = shape_or_base.seed_base if isinstance(shape_or_base, MoEShape) else int(shape_or_base)
    return base * 1000 + tensor_id + sub * 100_003


# tensor ids used with seed_of
X, WR, BIAS, W13, W2, SH13, SH2, ZIPF = 1, 2, 3, 4, 5, 6, 7, 8


def gen(seed: int, device) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(int(seed) & 0x7FFF_FFFF_FFFF_FFFF)
    return g


def normal(shape, std: float, seed: int, device="cpu", dtype=torch.float32) -> torch.Tensor:
    """N(0, std^2) drawn in fp32, then rounded (RNE) to dtype."""
    g = gen(seed, device)
    t = torch.randn(*shape, generator=g, device=device, dtype=torch.float32)
    if std != 1.0:
        t.mul_(std)
    return t.to(dtype)


def activations(T: int, H: int, seed: int, outlier_frac: float = 0.0,
                outlier_scale: float = 50.0, device="cpu") -> torch.Tensor:
    """x bf16 [T, H] ~ N(0,1); round(outlier_frac*H) seeded channels x outlier_scale."""
    g = gen(seed, device)
    x = torch.randn(T, H, generator=g, device=device, dtype=torch.float32)
    n_out = int(round(outlier_frac * H))
    if n_out > 0:
        gc = gen(seed + 777, "cpu")
        ch = torch.randperm(H, generator=gc)[:n_out].to(device)
        x[:, ch] *= outlier_scale
    return x.to(torch.bfloat16)


def router_weights(E: int, H: int, std: float, seed: int, device="cpu") -> torch.Tensor:
    """W_r fp32 [E, H] ~ N(0, std^2)."""
    return normal((E, H), std, seed, device, torch.float32)


def expert_bias(E: int, half_range: float, seed: int, device="cpu") -> torch.Tensor:
    """b fp32 [E] ~ U(-half_range, half_range); zeros when half_range == 0."""
    if half_range == 0.0:
        return torch.zeros(E, dtype=torch.float32, device=device)
    g = gen(seed, device)
    u = torch.rand(E, generator=g, device=device, dtype=torch.float32)
    return (u * 2.0 - 1.0) * half_range


def expert_weight(rows: int, cols: int, std: float, seed: int, device="cpu") -> torch.Tensor:
    """One expert's master weight, bf16 [rows, cols] ~ N(0, std^2)."""
    return normal((rows, cols), std, seed, device, torch.bfloat16)


def zipf_offset(E: int, kappa: float, seed: int, s: float = 1.1, device="cpu") -> torch.Tensor:
    """Per-expert router-logit offset o_e = -kappa * s * ln(rank_e), fp32 [E].

    rank is a seeded permutation of 1..E, so the most favoured expert (rank 1)
    gets offset 0 and the others fall off like a Zipf(s) law."""
    g = gen(seed, "cpu")
    rank = torch.randperm(E, generator=g).to(torch.float64) + 1.0
    o = -kappa * s * torch.log(rank)
    return o.to(torch.float32).to(device)


def scores(T: int, E: int, seed: int, tie_frac: float = 0.0, device="cpu") -> torch.Tensor:
    """Synthetic affinities, fp32 [T, E] ~ U(0.02, 0.98).

    With tie_frac > 0, that fraction of each row is overwritten by copies of
    other entries of the same row, so exact ties occur."""
    g = gen(seed, device)
    s = torch.rand(T, E, generator=g, device=device, dtype=torch.float32) * 0.96 + 0.02
    if tie_frac > 0.0:
        n = max(1, int(round(tie_frac * E)))
        src = torch.randint(0, E, (T, n), generator=g, device=device)
        dst = torch.randint(0, E, (T, n), generator=g, device=device)
        s.scatter_(1, dst, torch.gather(s, 1, src))
    return s


def topk_indices(T: int, E: int, K: int, seed: int, skew: float = 0.0, device="cpu") -> torch.Tensor:
    """Random routing table int32 [T, K]: K distinct experts per token.

    skew > 0 biases the draw towards low expert numbers (weights exp(-skew*e/E))."""
    g = gen(seed, "cpu")
    w = torch.exp(-skew * torch.arange(E, dtype=torch.float64) / max(E, 1))
    w = w.expand(T, E) if T > 0 else w.reshape(1, E)[:0]
    idx = torch.multinomial(w, K, replacement=False, generator=g) if T > 0 else torch.zeros(0, K, dtype=torch.int64)
    return idx.to(torch.int32).to(device)


def heavy_tailed(M: int, K: int, seed: int, frac: float = 0.01, scale: float = 100.0,
                 device="cpu") -> torch.Tensor:
    """A bf16 [M, K]: N(0,1) with a seeded `frac` of the entries times `scale`."""
    g = gen(seed, device)
    a = torch.randn(M, K, generator=g, device=device, dtype=torch.float32)
    mask = torch.rand(M, K, generator=g, device=device) < frac
    a = torch.where(mask, a * scale, a)
    return a.to(torch.bfloat16)


def group_sizes(total: int, G: int, seed: int) -> list[int]:
    """A uniform random composition of `total` into G parts (empty parts
    allowed): G-1 sorted uniform cut points in [0, total]."""
    g = gen(seed, "cpu")
    cuts = torch.randint(0, total + 1, (G - 1,), generator=g).sort().values.tolist()
    edges = [0] + cuts + [total]
    return [edges[i + 1] - edges[i] for i in range(G)]


def zipf_kappa_default() -> float:
    """The Zipf offset strength of the skewed-prefill workload: 0.46 gives an
    initial max/mean expert load of about 20 (measured with the oracle's router
    on a 4096-token slice of that workload at b = 0)."""
    return 0.46


def _check():  # pragma: no cover - tiny self-check for manual runs
    assert sum(group_sizes(1000, 16, 1)) == 1000
    assert math.isclose(float(zipf_offset(8, 1.0, 0).max()), 0.0)
