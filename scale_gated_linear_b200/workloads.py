"""Seeded synthetic workloads for the MS-GLA layer forward pass.

This module only draws random inputs and weights; it holds none of the layer's
arithmetic. Both the CUDA path (through the binding) and the CPU oracle are fed
from here, so that they see bit-identical values.

Shapes follow the 340M-parameter setting of "MS-GLA: Multi-Scale Gated Linear
Attention" (reading notes, Sec. 4: 24-layer decoder, hidden size 1024, 4 heads,
training length 2048) and the variant table of Sec. 4 ({1,2,4} with heads
[2,1,1], {1} = plain GLA, {1,2,4,8}, the {2,4} ablation). The pages' datasets
(FineWeb-Edu and the evaluation suites) are not used: these synthetic inputs
stand in for them.

Recipe (all draws from one ``torch.Generator`` seeded per workload):
  * X ~ N(0, 1) per element; for the bf16 workloads each row is then divided by
    its RMS (the layer input is the output of a pre-norm).
  * projection weights ~ N(0, std) with std = 1/sqrt(fan_in) for the tiny fp32
    workload and std = 0.02 otherwise; W_g2 (the second low-rank gate factor)
    and all biases are fp32, everything else is rounded to bf16.
  * the long-sequence workload skews the forget gates toward long memory:
    b_g = +3, W_g1 ~ N(0, 1/d), W_g2 ~ N(0, 1/r), so that the gate
    pre-activation is about N(3, 1) for RMS-normalised rows.
  * valid-token masks (``make_mask``, uint8 [B, L], 1 = valid): left or right
    padding of a per-sequence length drawn uniformly from [0, L/2] (a batch of
    unequal-length prompts), independent Bernoulli(0.8) tokens, or all padding.
"""
from __future__ import annotations

import dataclasses
import math
from typing import Dict, List, Optional

import torch


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    B: int
    L: int
    d: int
    scales: tuple
    heads: tuple
    d_k: int
    d_v: int
    chunk: int
    gate_rank: int = 16
    gate_normalizer: float = 16.0
    dtype: str = "bf16"            # storage type of X and of the bf16 weights
    weight_std: Optional[float] = 0.02   # None -> 1/sqrt(fan_in)
    rms_norm_x: bool = True
    gate_bias: float = 0.0
    gate_fan_in_init: bool = False  # W_g1 ~ N(0,1/d), W_g2 ~ N(0,1/r)
    head_norm: bool = False         # per-head RMS norm of the GLA output (norm_w ~ N(1, 0.1^2))
    norm_eps: float = 1e-5
    seed: int = 0

    @property
    def H(self) -> int:
        return sum(self.heads)

    def replace(self, **kw) -> "Workload":
        return dataclasses.replace(self, **kw)


WORKLOADS: Dict[str, Workload] = {
    # tiny case the oracle finishes in milliseconds
    "tiny": Workload("tiny", B=1, L=64, d=64, scales=(1, 2, 4), heads=(2, 1, 1),
                     d_k=16, d_v=16, chunk=16, dtype="fp32", weight_std=None,
                     rms_norm_x=False, seed=1000),
    # 340M-shaped layer, the measured configuration
    "msgla_340m": Workload("msgla_340m", B=8, L=2048, d=1024, scales=(1, 2, 4), heads=(2, 1, 1),
                           d_k=256, d_v=512, chunk=64, seed=1001),
    # plain GLA layer of the same width (single scale)
    "gla_340m": Workload("gla_340m", B=8, L=2048, d=1024, scales=(1,), heads=(4,),
                         d_k=256, d_v=512, chunk=64, seed=1002),
    # one long sequence with long-memory gates
    "long_32k": Workload("long_32k", B=1, L=32768, d=1024, scales=(1, 2, 4), heads=(2, 1, 1),
                         d_k=256, d_v=512, chunk=64, gate_bias=3.0, gate_fan_in_init=True,
                         seed=1003),
    # wider scale set and its no-fine-branch ablation (same inputs: same seed)
    "wide_8k": Workload("wide_8k", B=4, L=8192, d=2048, scales=(1, 2, 4, 8), heads=(4, 2, 1, 1),
                        d_k=256, d_v=512, chunk=128, seed=1004),
    "wide_8k_no_fine": Workload("wide_8k_no_fine", B=4, L=8192, d=2048, scales=(2, 4), heads=(2, 2),
                                d_k=256, d_v=512, chunk=128, seed=1004),
}


def _normal(g: torch.Generator, shape, std: float) -> torch.Tensor:
    return torch.randn(*shape, generator=g, dtype=torch.float32) * std


def make_inputs(w: Workload, B: Optional[int] = None, L: Optional[int] = None,
                seed: Optional[int] = None, round_to_bf16: Optional[bool] = None) -> dict:
    """Draw X and all weights for workload ``w`` (CPU tensors).

    Returns a dict with ``X`` [B, L, d] and ``branches`` (one dict per scale
    with Wq [h*d_k, d], Wk [h*d_k, d], Wv [h*d_v, d], Wg1 [r, d], Wg2 [h*d_k, r],
    bg [h*d_k], Wo [d, h*d_v], and norm_w [h*d_v] fp32 for ``head_norm``
    workloads) plus ``Wfuse`` [n_scales, d] and ``bfuse``
    [n_scales]. Tensors meant for bf16 storage are returned as bfloat16 when
    ``round_to_bf16`` (default: the workload's dtype is bf16); fp32 otherwise.
    Weights are drawn before X so that a different B or L keeps the weights.
    """
    B = w.B if B is None else B
    L = w.L if L is None else L
    g = torch.Generator().manual_seed(w.seed if seed is None else seed)
    if round_to_bf16 is None:
        round_to_bf16 = (w.dtype == "bf16")
    d, r = w.d, w.gate_rank

    def std_for(fan_in):
        return (1.0 / math.sqrt(fan_in)) if w.weight_std is None else w.weight_std

    lo = (lambda t: t.to(torch.bfloat16)) if round_to_bf16 else (lambda t: t)
    branches: List[dict] = []
    for s, h in zip(w.scales, w.heads):
        br = {
            "Wq": lo(_normal(g, (h * w.d_k, d), std_for(d))),
            "Wk": lo(_normal(g, (h * w.d_k, d), std_for(d))),
            "Wv": lo(_normal(g, (h * w.d_v, d), std_for(d))),
        }
        if w.gate_fan_in_init:
            br["Wg1"] = lo(_normal(g, (r, d), 1.0 / math.sqrt(d)))
            br["Wg2"] = _normal(g, (h * w.d_k, r), 1.0 / math.sqrt(r))
        else:
            br["Wg1"] = lo(_normal(g, (r, d), std_for(d)))
            br["Wg2"] = _normal(g, (h * w.d_k, r), std_for(r))
        br["bg"] = torch.full((h * w.d_k,), float(w.gate_bias), dtype=torch.float32)
        br["Wo"] = lo(_normal(g, (d, h * w.d_v), std_for(h * w.d_v)))
        if w.head_norm:
            br["norm_w"] = 1.0 + _normal(g, (h * w.d_v,), 0.1)
        branches.append(br)
    Wfuse = lo(_normal(g, (len(w.scales), d), std_for(d)))
    bfuse = torch.zeros(len(w.scales), dtype=torch.float32)
    X = torch.randn(B, L, d, generator=g, dtype=torch.float32)
    if w.rms_norm_x:
        X = X / X.pow(2).mean(-1, keepdim=True).sqrt()
    return {"X": lo(X), "branches": branches, "Wfuse": Wfuse, "bfuse": bfuse}


MASK_KINDS = ("left", "right", "random", "none", "all_padding")


def make_mask(B: int, L: int, kind: str, seed: int = 0) -> torch.Tensor:
    """Valid-token mask uint8 [B, L] (1 = valid, 0 = padding) of the given kind."""
    g = torch.Generator().manual_seed(seed)
    if kind == "none":
        return torch.ones(B, L, dtype=torch.uint8)
    if kind == "all_padding":
        return torch.zeros(B, L, dtype=torch.uint8)
    if kind == "random":
        return (torch.rand(B, L, generator=g) < 0.8).to(torch.uint8)
    if kind not in ("left", "right"):
        raise ValueError(f"unknown mask kind {kind!r}")
    pad = torch.randint(0, L // 2 + 1, (B,), generator=g)
    pos = torch.arange(L)[None, :]
    valid = pos >= pad[:, None] if kind == "left" else pos < (L - pad)[:, None]
    return valid.to(torch.uint8)


def to_float64(inp: dict) -> dict:
    """Widen every tensor of ``make_inputs`` output to float64 numpy arrays."""
    f = lambda t: t.to(torch.float64).numpy()
    return {
        "X": f(inp["X"]),
        "branches": [{k: f(v) for k, v in br.items()} for br in inp["branches"]],
        "Wfuse": f(inp["Wfuse"]),
        "bfuse": f(inp["bfuse"]),
    }


def round_inputs_to_bf16(inp: dict) -> dict:
    """Round the tensors that the CUDA path stores as bf16 (X, Wq/Wk/Wv/Wg1/Wo,
    Wfuse); W_g2 and the biases stay fp32."""
    b = lambda t: t.to(torch.bfloat16)
    return {
        "X": b(inp["X"]),
        "branches": [{k: (b(v) if k in ("Wq", "Wk", "Wv", "Wg1", "Wo") else v.float())
                      for k, v in br.items()} for br in inp["branches"]],
        "Wfuse": b(inp["Wfuse"]),
        "bfuse": inp["bfuse"].float(),
    }
