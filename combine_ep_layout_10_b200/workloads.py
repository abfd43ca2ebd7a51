"""Seeded synthetic workloads for the MoE layout / dispatch / combine path.

This module is the one piece both the CUDA path's tests/benchmark and the CPU
oracle consume.  It holds none of the method's arithmetic: it only draws the
inputs a gate would hand to dispatch (hidden states, top-k expert ids and
top-k weights) and the expert outputs combine reads.  It imports torch only
(CPU tensors; no CUDA, no library code).

The five workloads follow the shapes of the pages' test setting (8K tokens
per batch, hidden 7168, top-8 experts, FP8 dispatch, BF16 combine: "DeepSeek
publica DeepEP ..." (news.hada.io), "Resultados de medición de rendimiento")
plus a tiny case, a prefill case, a decoding case with a cached handle
("DeepEP (DeepEveryParallel) Documentation", item 3) and a large skewed case.
The group-limited gate is the one of the DeepSeek-V3 paper that the downcodes
article on the DeepEP launch says the library matches.

Recipe (all draws from one torch.Generator seeded with the workload seed):
  1. x = randn(T, H) in fp32, rounded to bf16;
  2. logits = randn(T, E) in fp32;
  3. routing scores: "normal" -> logits; "group_limited" -> logits + ln p_e
     with Zipf p_e ~ (e+1)^-s, then only the top `topk_groups` groups of
     `group_size` experts by group max stay eligible; "zipf" -> logits + ln p_e;
  4. topk_idx = top-k of the scores (sorted, distinct experts), int32;
  5. topk_w = softmax over the k selected *unbiased* logits, fp32.
Expert outputs for combine: randn(n_rows, H) rounded to bf16, drawn in seeded blocks
(make_expert_out).
"""
from __future__ import annotations

import math
import os
from dataclasses import dataclass, field, replace

import torch


@dataclass(frozen=True)
class Workload:
    name: str
    T: int                  # tokens
    H: int                  # hidden size
    E: int                  # experts
    k: int                  # top-k
    R: int                  # virtual ranks
    fp8: bool               # FP8 e4m3 dispatch (else BF16)
    capacity: int = 0       # rows per expert (padded layout), 0 = packed
    align: int = 1          # expert_alignment of packed segments
    routing: str = "normal"  # "normal" | "group_limited" | "zipf"
    zipf_s: float = 0.0
    groups: int = 1
    topk_groups: int = 1
    steps: int = 1          # decode: steps reusing one handle
    seed: int = 0
    notes: str = field(default="", compare=False)

    def scaled(self, **kw) -> "Workload":
        """A copy with some fields replaced (e.g. fewer tokens for oracle-sized tests)."""
        return replace(self, **kw)


WORKLOADS = {
    "tiny": Workload("tiny", T=128, H=256, E=16, k=4, R=4, fp8=False, routing="normal",
                     notes="top-4 of N(0,1) logits, BF16 dispatch + combine"),
    "prefill": Workload("prefill", T=4096, H=7168, E=256, k=8, R=8, fp8=True, routing="normal",
                        notes="training prefill: top-8 of N(0,1), FP8 dispatch"),
    "group_limited": Workload("group_limited", T=8192, H=7168, E=256, k=8, R=64, fp8=True,
                              routing="group_limited", zipf_s=1.0, groups=8, topk_groups=4,
                              notes="8 groups x 32, top-4 groups by group max, top-8 inside; "
                                    "Zipf(1.0) logit bias; FP8 dispatch, BF16 combine"),
    "decode": Workload("decode", T=128, H=7168, E=256, k=8, R=8, fp8=True, capacity=128,
                       routing="normal", steps=100,
                       notes="cached handle, 128 rows per expert, new x every step"),
    "large_skewed": Workload("large_skewed", T=32768, H=4096, E=128, k=8, R=16, fp8=False,
                             routing="zipf", zipf_s=1.2,
                             notes="Zipf(1.2) logit bias, BF16 dispatch + combine"),
}

#: The workload the headline metric is quoted on (8192 tokens, H=7168, top-8).
METRIC_WORKLOAD = "group_limited"


def zipf_log_bias(E: int, s: float) -> torch.Tensor:
    """ln p_e for Zipf popularity p_e ~ (e+1)^-s, expert 0 the hottest (fp32)."""
    e = torch.arange(E, dtype=torch.float64)
    logp = -s * torch.log(e + 1.0)
    logp = logp - torch.logsumexp(logp, dim=0)
    return logp.to(torch.float32)


def make_routing(w: Workload, seed: int | None = None):
    """Draw (x bf16 [T,H], topk_idx int32 [T,k], topk_w fp32 [T,k]) on the CPU."""
    seed = w.seed if seed is None else seed
    g = torch.Generator().manual_seed(seed)
    x = torch.randn(w.T, w.H, generator=g, dtype=torch.float32).to(torch.bfloat16)
    logits = torch.randn(w.T, w.E, generator=g, dtype=torch.float32)
    scores = logits
    if w.routing in ("group_limited", "zipf"):
        scores = logits + zipf_log_bias(w.E, w.zipf_s)[None, :]
    if w.routing == "group_limited":
        assert w.E % w.groups == 0
        gs = w.E // w.groups
        group_score = scores.view(w.T, w.groups, gs).amax(dim=2)
        keep = torch.topk(group_score, w.topk_groups, dim=1, sorted=True).indices
        mask = torch.zeros(w.T, w.groups, dtype=torch.bool)
        mask.scatter_(1, keep, True)
        scores = scores.masked_fill(~mask.repeat_interleave(gs, dim=1), float("-inf"))
    elif w.routing not in ("normal", "zipf"):
        raise ValueError("unknown routing %r" % w.routing)
    idx = torch.topk(scores, w.k, dim=1, sorted=True).indices
    sel = torch.gather(logits, 1, idx)
    topk_w = torch.softmax(sel, dim=1).to(torch.float32).contiguous()
    return x.contiguous(), idx.to(torch.int32).contiguous(), topk_w


def make_x(w: Workload, seed: int) -> torch.Tensor:
    """A fresh bf16 [T,H] batch of hidden states (decode steps: seed 1000 + step)."""
    g = torch.Generator().manual_seed(seed)
    return torch.randn(w.T, w.H, generator=g, dtype=torch.float32).to(torch.bfloat16).contiguous()


def make_expert_out(n_rows: int, H: int, seed: int) -> torch.Tensor:
    """Synthetic expert outputs y bf16 [n_rows, H] ~ N(0,1) for combine.

    Drawn in blocks of about 2^24 values, block i from its own generator
    seeded with seed * 1000003 + i, so the result does not depend on how many
    host threads fill the blocks (several do, for the multi-GB full-size
    cases)."""
    out = torch.empty(n_rows, H, dtype=torch.bfloat16)
    rows = max(1, (1 << 24) // max(H, 1))
    starts = list(range(0, n_rows, rows))

    def fill(i):
        r0 = starts[i]
        r1 = min(n_rows, r0 + rows)
        g = torch.Generator().manual_seed(seed * 1000003 + i)
        out[r0:r1] = torch.randn(r1 - r0, H, generator=g, dtype=torch.float32).to(torch.bfloat16)

    if len(starts) <= 1:
        for i in range(len(starts)):
            fill(i)
    else:
        from concurrent.futures import ThreadPoolExecutor
        with ThreadPoolExecutor(max_workers=min(8, os.cpu_count() or 1, len(starts))) as pool:
            list(pool.map(fill, range(len(starts))))
    return out


def load_stats(topk_idx: torch.Tensor, E: int) -> dict:
    """Hottest-expert load over the mean load (a property of the drawn routing)."""
    valid = topk_idx[topk_idx >= 0].to(torch.int64)
    cnt = torch.bincount(valid, minlength=E).to(torch.float64)
    mean = cnt.sum().item() / E
    return {"hottest": int(cnt.max().item()), "mean": mean,
            "hot_over_mean": (cnt.max().item() / mean) if mean > 0 else math.nan}
