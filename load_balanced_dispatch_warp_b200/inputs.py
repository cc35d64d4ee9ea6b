"""Seeded synthetic inputs for one MoE layer: router logits, token rows and expert weights.

This module only draws random numbers and applies a per-expert logit bias whose shape
is fixed by the workload recipe.  It holds none of the layer's arithmetic (no top-k, no
histogram, no plan, no FFN): both the CUDA path and the CPU oracle receive the tensors
it returns, and neither is imported here.

Workload shapes follow the model cards on "DeepEP-on-EFA Guidance §1 -- What is MoE"
(Qwen3-30B-A3B: 128 experts top-8; Mixtral-like: 8 experts top-2; DeepSeek-like: 256
routed experts top-8) and the hotspot of "Your MoE router sends 90% of tokens to 10% of
the experts" (90% of assignments to 26 of 256 experts).  Hidden and FFN sizes, rank and
slot counts are listed in ``WORKLOADS`` below; slot counts follow the MoonEP article's
slot policy (slots = experts per rank for training, 3-4 for inference).

Bias recipes (added to N(0,1) logits; expert e has Zipf rank e+1):
  zipf  : bias[e] = -alpha * ln(e + 1)
  gauss : bias[e] = sigma * z[e], z ~ N(0,1) drawn from the seed
  hot   : bias[e] = beta for 26 experts drawn from the seed, 0 elsewhere
The scalar of each recipe (alpha, sigma, beta) was bisected once by
``oracle/calibrate_workloads.py`` against the oracle's own maxvio / hot share and
stored in ``workload_bias.json`` beside this file.
"""
from __future__ import annotations

import json
import math
import os
from dataclasses import dataclass, field

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
BIAS_FILE = os.path.join(_HERE, "workload_bias.json")


@dataclass(frozen=True)
class Workload:
    name: str
    T: int   # tokens
    E: int   # experts
    k: int   # top-k
    R: int   # simulated expert-parallel ranks
    S: int   # prefetch slots per rank
    d: int   # hidden size
    F: int   # FFN (intermediate) size of one SwiGLU expert
    bias_kind: str            # "zipf" | "gauss" | "hot"
    target: float             # maxvio target ("zipf"/"gauss") or hot share ("hot")
    fixed_param: float | None = None  # recipe scalar fixed by the workload itself
    n_hot: int = 26
    seed: int = 0
    note: str = field(default="", compare=False)

    @property
    def B(self) -> int:
        return self.E // self.R

    @property
    def A(self) -> int:
        return self.T * self.k

    @property
    def C(self) -> int:
        return self.A // self.R


WORKLOADS: dict[str, Workload] = {w.name: w for w in [
    Workload("tiny", 16, 8, 2, 4, 2, 128, 256, "zipf", float("nan"), fixed_param=1.5,
             note="16 tokens, bias 1.5*(-ln zipf rank)"),
    Workload("near_balanced", 4096, 64, 6, 8, 8, 2048, 1408, "gauss", 0.2,
             note="fine-grained, 8 experts/rank, S = experts/rank (training)"),
    Workload("qwen_mv0.2", 8192, 128, 8, 16, 8, 2048, 768, "zipf", 0.2),
    Workload("qwen_mv1", 8192, 128, 8, 16, 8, 2048, 768, "zipf", 1.0),
    Workload("qwen_mv5", 8192, 128, 8, 16, 8, 2048, 768, "zipf", 5.0),
    # maxvio 20 cannot be reached at R=16 (the maximum is R-1 = 15): the top sweep point
    # is the extreme case where every token picks experts 0..7, maxvio exactly 15.
    Workload("qwen_mv15", 8192, 128, 8, 16, 8, 2048, 768, "zipf", 15.0, fixed_param=200.0,
             note="stand-in for maxvio 20: all tokens pick experts 0-7"),
    Workload("mixtral", 8192, 8, 2, 8, 3, 4096, 14336, "zipf", 1.0,
             note="coarse experts, 1 expert/rank, S=3 (inference)"),
    Workload("deepseek", 16384, 256, 8, 32, 4, 7168, 2048, "hot", 0.90,
             note="26 hot experts take 90% of assignments, S=4 (inference)"),
    # the DeepSeek-shaped expert (d = 7168, F = 2048, top-8) with tokens and experts cut so
    # that the whole layer holds under 3 GB on the device: the case for detailed counter
    # captures of the grouped FFN, which must stay small
    Workload("deepseek_small", 2048, 16, 8, 2, 4, 7168, 2048, "zipf", float("nan"),
             fixed_param=0.5, note="DeepSeek-shaped expert, 2048 tokens, 16 experts"),
]}

# Sweep order of the Qwen-shaped skew sweep.
QWEN_SWEEP = ["qwen_mv0.2", "qwen_mv1", "qwen_mv5", "qwen_mv15"]


def _gen(seed: int, stream: int, device="cpu") -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(seed * 1_000_003 + stream)
    return g


# stream ids: one independent generator per tensor, fixed order
_S_LOGITS, _S_BIAS, _S_X, _S_W1, _S_W3, _S_W2 = 1, 2, 3, 4, 5, 6


def load_bias_params() -> dict:
    if not os.path.exists(BIAS_FILE):
        return {}
    with open(BIAS_FILE) as f:
        return json.load(f)


def bias_param(w: Workload) -> float:
    if w.fixed_param is not None:
        return float(w.fixed_param)
    params = load_bias_params()
    if w.name not in params:
        raise KeyError(f"no calibrated bias for workload {w.name!r}; run oracle/calibrate_workloads.py")
    return float(params[w.name]["param"])


def expert_bias(w: Workload, param: float | None = None) -> torch.Tensor:
    """Per-expert logit bias [E] fp32 for the workload's recipe and scalar."""
    p = bias_param(w) if param is None else float(param)
    e = torch.arange(w.E, dtype=torch.float64)
    if w.bias_kind == "zipf":
        b = -p * torch.log(e + 1.0)
    elif w.bias_kind == "gauss":
        z = torch.randn(w.E, generator=_gen(w.seed, _S_BIAS), dtype=torch.float64)
        b = p * z
    elif w.bias_kind == "hot":
        hot = hot_experts(w)
        b = torch.zeros(w.E, dtype=torch.float64)
        b[hot] = p
    else:
        raise ValueError(w.bias_kind)
    return b.to(torch.float32)


def hot_experts(w: Workload) -> torch.Tensor:
    """The seeded set of hot experts of the "hot" recipe (sorted ids)."""
    perm = torch.randperm(w.E, generator=_gen(w.seed, _S_BIAS))
    return torch.sort(perm[: w.n_hot]).values


def base_logits(w: Workload) -> torch.Tensor:
    """N(0,1) fp32 router logits [T,E] before the bias (always drawn on the CPU)."""
    return torch.randn(w.T, w.E, generator=_gen(w.seed, _S_LOGITS), dtype=torch.float32)


def make_logits(w: Workload, param: float | None = None) -> torch.Tensor:
    """Router logits [T,E] fp32 (CPU): N(0,1) + the workload's per-expert bias."""
    return base_logits(w) + expert_bias(w, param)[None, :]


def make_x(w: Workload) -> torch.Tensor:
    """Token rows x [T,d] bf16 (CPU), N(0,1)."""
    return torch.randn(w.T, w.d, generator=_gen(w.seed, _S_X), dtype=torch.float32).to(torch.bfloat16)


def make_weights(w: Workload, device="cpu"):
    """Expert weights W1,W3 [E,F,d] and W2 [E,d,F], N(0, 1/d) rounded to bf16, drawn on
    ``device``.  W1 and W3 are stored as bf16; W2 holds the same bf16-rounded values in an
    fp16 tensor (the down projection's storage type), so every input value is identical for
    the CUDA path and the oracle.  Each projection is one contiguous tensor.
    """
    std = 1.0 / math.sqrt(w.d)
    out = []
    for stream, shape, dt in ((_S_W1, (w.E, w.F, w.d), torch.bfloat16),
                              (_S_W3, (w.E, w.F, w.d), torch.bfloat16),
                              (_S_W2, (w.E, w.d, w.F), torch.float16)):
        t = torch.empty(shape, dtype=dt, device=device)
        g = _gen(w.seed, stream, device)
        # draw in slabs of one expert to bound the fp32 temporary
        for e in range(w.E):
            v = torch.randn(shape[1:], generator=g, dtype=torch.float32, device=device) * std
            t[e] = v.to(torch.bfloat16).to(dt)
        out.append(t)
    return tuple(out)


def small_workload(name: str, T: int, E: int, k: int, R: int, S: int, d: int, F: int,
                   alpha: float = 1.0, seed: int = 0) -> Workload:
    """A Zipf-biased workload of arbitrary small shape (parity cases, edge cases)."""
    return Workload(name, T, E, k, R, S, d, F, "zipf", float("nan"), fixed_param=alpha, seed=seed)
