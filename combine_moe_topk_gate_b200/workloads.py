"""Seeded synthetic workloads for the MoE routing path.

This module only draws inputs; it holds none of the routing arithmetic, so the
CUDA path and the CPU oracle can both be fed from it without sharing any of the
method's code.  Shapes follow the workloads the pages measure on:

* ``tiny``     - a 64-token toy case (8 experts, top-2, plain softmax weights).
* ``decode``   - the low-latency batch of 128 tokens, hidden 7168, 256 experts
  ("DeepSeek, DeepEP 오픈소스 공개", section 저지연 커널 / low-latency kernels).
* ``prefill``  - 4096 tokens, hidden 7168, top-4 groups / top-8 experts, FP8
  dispatch and BF16 combine (same page, section 일반 커널 / normal kernels).
* ``skewed``   - 8192 tokens, hidden 7168, top-8, FP8 dispatch / BF16 combine
  (DeepEP V2 summary, section "performance measurement results"), with a
  Zipf(1.1) bias on the router logits of the hot experts.
* ``mixtral``  - Mixtral-8x7B-shaped routing (8 experts, top-2, renormalised
  softmax) over 16384 tokens of hidden 4096, with +2.0 on expert 0's logit
  ("Efficient and portable mixture-of-experts communication", Introduction,
  names Mixtral 8x7B).

Draw order for one seed (``torch.Generator('cpu').manual_seed(seed)``):
logits ``randn(N, E)`` fp32 -> (skewed only) ``randperm(E)`` -> x ``randn(N, H)``
rounded to bf16 -> (random expert outputs only) y ``randn(N*k, H)`` rounded to
bf16.  Expert outputs are the identity (``y = recv_x``) for the BF16 configs.
"""
from __future__ import annotations

from dataclasses import dataclass, field

import torch

GATE_KINDS = {"softmax": 0, "softmax_renorm": 1, "sigmoid_group": 2}
DTYPES = {"bf16": 0, "fp8": 1, "fp8_token": 2, "mxfp8": 3, "fp8_ue8m0": 6}


@dataclass(frozen=True)
class Workload:
    name: str
    N: int                 # tokens
    H: int                 # hidden size
    E: int                 # experts
    k: int                 # experts per token
    R: int                 # logical EP ranks (partitions of the receive buffer)
    gate: str              # "softmax" | "softmax_renorm" | "sigmoid_group"
    dtype: str             # dispatch payload: "bf16" | "fp8" | "fp8_token" | "mxfp8"
    expert_out: str        # "identity" (y = recv_x) | "random" (seeded bf16 y)
    n_groups: int = 1
    topk_groups: int = 1
    group_topn: int = 1
    bias: str = "none"     # "none" | "zipf1.1" | "expert0+2"
    extra: dict = field(default_factory=dict)

    @property
    def S(self) -> int:
        return self.N * self.k

    @property
    def gate_kind(self) -> int:
        return GATE_KINDS[self.gate]

    @property
    def dtype_code(self) -> int:
        return DTYPES[self.dtype]

    def scaled(self, N: int) -> "Workload":
        """Same routing shape with another token count (ragged/edge cases)."""
        return Workload(**{**self.__dict__, "N": N, "name": f"{self.name}@N={N}"})


WORKLOADS = {
    "tiny": Workload("tiny", 64, 256, 8, 2, 2, "softmax", "bf16", "identity"),
    "decode": Workload("decode", 128, 7168, 256, 8, 8, "sigmoid_group", "fp8", "random",
                       n_groups=8, topk_groups=4, group_topn=2),
    "prefill": Workload("prefill", 4096, 7168, 256, 8, 32, "sigmoid_group", "fp8", "random",
                        n_groups=8, topk_groups=4, group_topn=2),
    "skewed": Workload("skewed", 8192, 7168, 256, 8, 64, "sigmoid_group", "fp8", "random",
                       n_groups=8, topk_groups=4, group_topn=2, bias="zipf1.1"),
    "mixtral": Workload("mixtral", 16384, 4096, 8, 2, 8, "softmax_renorm", "bf16", "identity",
                        bias="expert0+2"),
}


def zipf_bias(E: int, perm: torch.Tensor, s: float = 1.1) -> torch.Tensor:
    """Per-expert logit bias for the skewed workload.

    Expert ``e`` gets popularity rank ``perm[e] + 1``; with Zipf weights
    ``p_r = r^-s / sum_q q^-s`` the bias is ``max(0, ln(E * p_r))``, so only
    the experts more popular than uniform (about 36 of 256 at s = 1.1) are
    pushed up, by at most ``ln(E * p_1)`` (about +3.97).
    """
    ranks = torch.arange(1, E + 1, dtype=torch.float64)
    p = ranks.pow(-s)
    p = p / p.sum()
    b_rank = torch.clamp(torch.log(E * p), min=0.0)
    return b_rank[perm].to(torch.float32)


@dataclass
class Inputs:
    logits: torch.Tensor            # fp32 [N, E]
    x: torch.Tensor                 # bf16 [N, H]
    y: torch.Tensor | None          # bf16 [N*k, H] (random expert outputs) or None


def make_inputs(w: Workload, seed: int = 0, *, with_y: bool = True) -> Inputs:
    g = torch.Generator(device="cpu")
    g.manual_seed(seed)
    logits = torch.randn(w.N, w.E, generator=g, dtype=torch.float32)
    if w.bias == "zipf1.1":
        perm = torch.randperm(w.E, generator=g)
        logits += zipf_bias(w.E, perm)
    elif w.bias == "expert0+2":
        logits[:, 0] += 2.0
    x = torch.randn(w.N, w.H, generator=g, dtype=torch.float32).to(torch.bfloat16)
    y = None
    if with_y and w.expert_out == "random":
        y = torch.randn(w.S, w.H, generator=g, dtype=torch.float32).to(torch.bfloat16)
    return Inputs(logits, x, y)


def algorithmic_bytes(w: Workload) -> dict:
    """Bytes each step must move at least once (each token row read once,
    written k times; int32 metadata of the step included)."""
    N, H, E, k = w.N, w.H, w.E, w.k
    row = {"bf16": 2 * H, "nvfp4": H // 2, "e5m6": H // 2 * 3}.get(w.dtype, H)   # payload bytes of a receive row
    scales = {"fp8": 4 * N * k * (H // 128), "fp8_token": 4 * N * k,
              "mxfp8": N * k * (H // 32), "nvfp4": N * k * (H // 16) + 4 * N * k,
              "fp8_ue8m0": N * k * (H // 128)}.get(w.dtype, 0)
    return {
        "gate": 4 * N * E + 8 * N * k,
        "layout": 4 * N * k + 8 * N * k + 4 * (4 * E + 3 * w.R),
        "dispatch": 2 * N * H + N * k * row + scales + 4 * N * k,
        "combine": 2 * N * k * H + 2 * N * H + 8 * N * k,
        # backward: gradient rows in, token gradient out (dispatch); token
        # gradient + expert rows in, scaled rows + weight gradients out (combine)
        "dispatch_backward": 2 * N * k * H + 2 * N * H + 4 * N * k,
        "combine_backward": 2 * N * H + 4 * N * k * H + 12 * N * k,
    }


def mean_expert_load(counts) -> tuple[float, float]:
    c = [int(v) for v in counts]
    return max(c), sum(c) / max(1, len(c))


__all__ = ["Workload", "WORKLOADS", "Inputs", "make_inputs", "algorithmic_bytes",
           "zipf_bias", "GATE_KINDS", "DTYPES"]
