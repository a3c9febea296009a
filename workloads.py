"""Seeded synthetic inputs for the MoE token round trip.

This module is shared by the CPU oracle's tests, the GPU parity tests, the smoke check and the
benchmark.  It only draws random inputs (hidden states, routing, expert outputs, shared-expert
bias) with the shapes and distributions of the workloads below; it holds none of the layout,
dispatch or combine arithmetic.  Every tensor comes from its own CPU ``torch.Generator`` seeded
with ``seed * 1000 + stream_id``, so the same bytes come out on every machine.

Workload shapes follow the pages' benchmark settings:
  * "DeepEP expert-parallel communication" (blog.hotdry.top), "Performance benchmark":
    4096 tokens per batch, hidden 7168, top-4 groups then top-8 experts (DeepSeek-V3/R1),
    FP8 dispatch and BF16 combine; low-latency decode with 128 tokens, top-8, batch < 256.
  * "Why MoE gets stuck on communication" (locsic.com), section 3: 16384 tokens capacity,
    hidden 7168, 256 experts, top-6, alignment 128, no bias; the 10/10/10/30 ms load model.
"""
from __future__ import annotations

import dataclasses
from dataclasses import dataclass

import torch

# generator stream ids (seed * 1000 + id)
_S_X, _S_ROUTE, _S_WEIGHT, _S_Y, _S_BIAS, _S_MASK = 1, 2, 3, 4, 5, 6


@dataclass(frozen=True)
class Workload:
    name: str
    tokens_per_rank: int
    ranks: int                 # logical expert-parallel ranks R
    hidden: int                # H
    experts: int               # E
    topk: int                  # k
    alignment: int             # expert_alignment A
    fp8: bool                  # FP8 E4M3 dispatch with 1x128 block scales (else BF16)
    zero_padding: bool
    cpu_sync: bool
    bias: bool                 # shared-expert output added in combine
    routing: str               # "uniform", "group_limited" or "zipf"
    n_groups: int = 0
    topk_groups: int = 0
    zipf_s: float = 0.0
    num_sms: int = 0           # 0 = every SM
    max_tokens_per_rank: int = 0   # > 0: receive capacity from the worst-case bound
    weighted_combine: bool = False
    seed: int = 0

    @property
    def tokens(self) -> int:
        return self.tokens_per_rank * self.ranks

    @property
    def experts_per_rank(self) -> int:
        return self.experts // self.ranks

    def with_(self, **kw) -> "Workload":
        return dataclasses.replace(self, **kw)


WORKLOADS = {
    # 64 tokens in total (32 per rank), H=256, E=8 over 2 ranks, top-2, A=16, BF16 both ways.
    "tiny": Workload("tiny", 32, 2, 256, 8, 2, 16, fp8=False, zero_padding=True,
                     cpu_sync=True, bias=False, routing="uniform"),
    # DeepSeek-V3 prefill: 4096 tokens/rank x 8 ranks, H=7168, 256 experts in 8 groups,
    # top-4 groups then top-8 experts, FP8 dispatch, BF16 combine, A=128.
    "deepseek": Workload("deepseek", 4096, 8, 7168, 256, 8, 128, fp8=True, zero_padding=True,
                         cpu_sync=True, bias=False, routing="group_limited", n_groups=8,
                         topk_groups=4),
    # Decode: 128 tokens/rank x 8, top-8 uniform, no host sync, outputs sized for 256
    # tokens/rank, FP8 dispatch, BF16 combine with the shared-expert bias.
    "decode": Workload("decode", 128, 8, 7168, 256, 8, 128, fp8=True, zero_padding=False,
                       cpu_sync=False, bias=True, routing="uniform", max_tokens_per_rank=256),
    # Large capacity: 16384 tokens over 32 ranks, top-6, A=128, zero padding, no bias.
    "large": Workload("large", 512, 32, 7168, 256, 6, 128, fp8=True, zero_padding=True,
                      cpu_sync=True, bias=False, routing="uniform"),
    # Skewed: 8192 tokens over 16 ranks, H=4096, 128 experts, Zipf(1.2) popularity, BF16,
    # dispatch and combine capped at 24 SMs.
    "skewed": Workload("skewed", 512, 16, 4096, 128, 8, 128, fp8=False, zero_padding=True,
                       cpu_sync=True, bias=False, routing="zipf", zipf_s=1.2, num_sms=24),
}


def _gen(wl: Workload, stream: int) -> torch.Generator:
    g = torch.Generator(device="cpu")
    g.manual_seed(wl.seed * 1000 + stream)
    return g


def gen_x(wl: Workload) -> torch.Tensor:
    """Hidden states x [T, H], bf16 rounding of N(0, 1)."""
    return torch.randn(wl.tokens, wl.hidden, generator=_gen(wl, _S_X)).to(torch.bfloat16)


def _softmax_weights(wl: Workload) -> torch.Tensor:
    logits = torch.randn(wl.tokens, wl.topk, generator=_gen(wl, _S_WEIGHT))
    return torch.softmax(logits, dim=1).to(torch.float32)


def gen_routing(wl: Workload) -> tuple[torch.Tensor, torch.Tensor]:
    """Top-k routing: (topk_idx int64 [T, k], topk_weights fp32 [T, k]).

    uniform        k distinct experts, uniform over subsets (top-k of uniform keys);
                   weights = softmax of k fresh N(0, 1) logits.
    group_limited  N(0, 1) logits, sigmoid scores; a group's score is the sum of its two best
                   scores; keep the best ``topk_groups`` groups, then the best k experts among
                   them; weights = the chosen scores over their sum.
    zipf           popularity p(e) ~ (e + 1)^-s; k distinct experts drawn without replacement
                   by Gumbel-top-k on log p; softmax weights.
    """
    T, E, k = wl.tokens, wl.experts, wl.topk
    g = _gen(wl, _S_ROUTE)
    if wl.routing == "uniform":
        keys = torch.rand(T, E, generator=g)
        idx = keys.topk(k, dim=1).indices
        w = _softmax_weights(wl)
    elif wl.routing == "group_limited":
        logits = torch.randn(T, E, generator=g)
        scores = torch.sigmoid(logits)
        G = wl.n_groups
        grouped = scores.view(T, G, E // G)
        group_score = grouped.topk(2, dim=2).values.sum(dim=2)
        keep = group_score.topk(wl.topk_groups, dim=1).indices
        mask = torch.zeros(T, G, dtype=torch.bool)
        mask.scatter_(1, keep, True)
        masked = scores.masked_fill(~mask.repeat_interleave(E // G, dim=1), -1.0)
        top = masked.topk(k, dim=1)
        idx = top.indices
        w = (top.values / top.values.sum(dim=1, keepdim=True)).to(torch.float32)
    elif wl.routing == "zipf":
        logp = -wl.zipf_s * torch.log(torch.arange(1, E + 1, dtype=torch.float64))
        u = torch.rand(T, E, generator=g, dtype=torch.float64).clamp_min(1e-300)
        gumbel = -torch.log(-torch.log(u))
        idx = (logp.unsqueeze(0) + gumbel).topk(k, dim=1).indices
        w = _softmax_weights(wl)
    else:
        raise ValueError(f"unknown routing {wl.routing!r}")
    return idx.to(torch.int64).contiguous(), w.contiguous()


def mask_entries(wl: Workload, idx: torch.Tensor, frac: float) -> torch.Tensor:
    """Replace a seeded fraction of routing entries with -1 (masked)."""
    m = torch.rand(idx.shape, generator=_gen(wl, _S_MASK)) < frac
    return idx.masked_fill(m, -1)


def gen_y(wl: Workload, cap: int) -> torch.Tensor:
    """Expert outputs y [R, cap, H], bf16 rounding of N(0, 1)."""
    return torch.randn(wl.ranks, cap, wl.hidden, generator=_gen(wl, _S_Y)).to(torch.bfloat16)


def gen_bias(wl: Workload) -> torch.Tensor:
    """Shared-expert output [T, H], bf16 rounding of N(0, 1)."""
    return torch.randn(wl.tokens, wl.hidden, generator=_gen(wl, _S_BIAS)).to(torch.bfloat16)


def worst_case_rows_per_rank(wl: Workload, max_tokens_per_rank: int) -> int:
    """Receive rows one rank may need when every rank sends it max_tokens_per_rank tokens:
    each token reaches at most min(k, E_loc) of its experts, and each of its E_loc experts
    may add up to A - 1 padding rows."""
    e_loc = wl.experts_per_rank
    return wl.ranks * max_tokens_per_rank * min(wl.topk, e_loc) + e_loc * (wl.alignment - 1)


def gen_y_device(wl: Workload, cap: int, device="cuda") -> torch.Tensor:
    """Expert outputs y [R, cap, H] drawn on the GPU (for full-size runs where a CPU draw of
    several GB would dominate): bf16 rounding of N(0, 1) from a seeded CUDA generator."""
    g = torch.Generator(device=device)
    g.manual_seed(wl.seed * 1000 + _S_Y)
    return torch.randn(wl.ranks, cap, wl.hidden, generator=g, device=device).to(torch.bfloat16)
