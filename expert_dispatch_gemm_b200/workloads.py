"""Seeded synthetic workloads for the MoE routing-and-dispatch layer.

This module is shared by the CUDA path's tests and benchmark and by the CPU
oracle's tests. It holds shapes, modes and random-number recipes only: none
of the layer's arithmetic (no scores, no top-k, no quotas or capacities; the
expert-choice quota and the capacity are derived from ``c`` / ``capacity_factor``
by each side on its own).

Workload shapes follow the model families the pages name (Mixtral top-2 of 8,
OLMoE top-8 of 64, DeepSeek-V3 sigmoid, group-limited, 1 shared + 256
routed, and the expert-choice worked example of 4,096 tokens, 64 experts,
c = 2). Inputs are random-initialised with fixed seeds; there are no trained
weights and no datasets.

Recipe (every tensor from its own seeded stream, seed*1000 + stream id):
    X      ~ N(0, 1)            [n, d]       (fp32 or bf16)
    W_g    ~ N(0, 1/d)          [d, E]       fp32
    W1, W3 ~ N(0, 2/d)          [E, h, d]    (fan_in = d)
    W2     ~ N(0, 2/h)          [E, d, h]    (fan_in = h)
    shared expert weights likewise, [n_shared, ...]
    logit skew b_g[e] ~ N(0, variance) when ``logit_skew_var`` > 0
    selection bias starts at 0.
bf16 tensors are drawn in fp32 and rounded to bf16 by torch.
"""
from __future__ import annotations

import dataclasses
from dataclasses import dataclass, field

import torch


@dataclass(frozen=True)
class Workload:
    name: str
    n: int
    d: int
    E: int
    h: int
    mode: str                 # "ec" (expert choice) or "tc" (token choice)
    score: str = "softmax"    # "softmax", "sigmoid" or "sqrtsoftplus"
    c: float = 0.0            # EC capacity factor (k = n c / E)
    K: int = 0                # TC experts per token
    capacity_factor: float = 0.0   # TC: > 0 enables a per-expert buffer
    n_groups: int = 1
    topk_groups: int = 1
    group_topn: int = 1
    weights: str = "raw"      # "raw" or "normalized" (over the selected)
    act: str = "relu"         # "relu", "gelu" or "swiglu"
    dtype: str = "bf16"       # "f32" or "bf16"
    n_shared: int = 0
    logit_skew_var: float = 0.0
    lb_coef: float = 0.01
    z_coef: float = 0.001
    bias_steps: int = 0       # simulated steps of the selection-bias update
    bias_rate: float = 0.001
    seed: int = 0

    def replace(self, **kw) -> "Workload":
        return dataclasses.replace(self, **kw)

    @property
    def torch_dtype(self):
        return torch.float32 if self.dtype == "f32" else torch.bfloat16


# The five named workloads (full size).
EC_FP32 = Workload("ec-fp32-n512-d128-e8-c2-relu512", n=512, d=128, E=8, h=512,
                   mode="ec", c=2.0, act="relu", dtype="f32")
EC_BF16 = Workload("ec-bf16-n4096-d1024-e64-c2-gelu4096", n=4096, d=1024, E=64, h=4096,
                   mode="ec", c=2.0, act="gelu")
TC_TOP2_CAP = Workload("tc-softmax-top2of8-cap1.25-n8192-d4096-swiglu14336", n=8192,
                       d=4096, E=8, h=14336, mode="tc", K=2, capacity_factor=1.25,
                       weights="normalized", act="swiglu", logit_skew_var=1.5)
TC_DROPLESS = Workload("tc-softmax-top8of64-dropless-n16384-d2048-swiglu1024", n=16384,
                       d=2048, E=64, h=1024, mode="tc", K=8, weights="raw", act="swiglu")
TC_SIGMOID_GROUPED = Workload(
    "tc-sigmoid-grouped8keep4-top8of256-shared1-n8192-d7168-swiglu2048", n=8192, d=7168,
    E=256, h=2048, mode="tc", score="sigmoid", K=8, n_groups=8, topk_groups=4,
    group_topn=2, weights="normalized", act="swiglu", n_shared=1, bias_steps=10)

FULL = [EC_FP32, EC_BF16, TC_TOP2_CAP, TC_DROPLESS, TC_SIGMOID_GROUPED]
# the decoding regime of the DeepSeek-V3-shaped layer: 64 tokens, so most of
# the 256 experts see no token or one; the step streams the active experts'
# weights (a bench workload, not one of the five configurations)
DECODE = TC_SIGMOID_GROUPED.replace(
    name="tc-sigmoid-grouped8keep4-top8of256-shared1-decode-n64-d7168-swiglu2048", n=64,
    bias_steps=0)

# Reduced sizes of the same five routings: the oracle finishes these in
# seconds; they still span several GEMM tiles and leave ragged tails.
SMALL = [
    EC_FP32,
    EC_BF16.replace(name="ec-bf16-n640-d256-e16-c2-gelu384", n=640, d=256, E=16, h=384),
    TC_TOP2_CAP.replace(name="tc-top2of8-cap1.25-n1000-d256-swiglu320", n=1000, d=256,
                        h=320),
    TC_DROPLESS.replace(name="tc-top8of64-dropless-n777-d192-swiglu256", n=777, d=192,
                        h=256),
    TC_SIGMOID_GROUPED.replace(name="tc-sigmoid-grouped8keep4-top8of64-shared1-n300-d256-"
                               "swiglu128", n=300, d=256, E=64, h=128, bias_steps=3),
]

# Reduced versions of two token-choice layers (same d and h; a quarter of the
# batch, or an eighth of the batch and of the experts) for ncu captures that
# replay every launch: a few GB on the device at most
PROFILE = [
    TC_DROPLESS.replace(name="tc-softmax-top8of64-dropless-n4096-d2048-swiglu1024", n=4096),
    TC_SIGMOID_GROUPED.replace(
        name="tc-sigmoid-grouped8keep4-top8of32-shared1-n1024-d7168-swiglu2048", n=1024, E=32,
        bias_steps=0),
]

BY_NAME = {w.name: w for w in FULL + SMALL + [DECODE] + PROFILE}


def _gen(device, seed: int, stream: int) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(seed * 1000 + stream)
    return g


def _normal(shape, std, dtype, device, gen, chunk_dim0=False):
    """N(0, std^2) drawn in fp32 and cast; optionally one leading slice at a
    time so a large bf16 tensor never needs a full fp32 copy."""
    if not chunk_dim0 or len(shape) < 2:
        return (torch.randn(shape, generator=gen, device=device, dtype=torch.float32) * std
                ).to(dtype)
    out = torch.empty(shape, dtype=dtype, device=device)
    for i in range(shape[0]):
        out[i] = (torch.randn(shape[1:], generator=gen, device=device,
                              dtype=torch.float32) * std).to(dtype)
    return out


def make_inputs(w: Workload, device="cpu", experts: bool = True) -> dict:
    """All inputs of one layer call, seeded; tensors live on `device`."""
    dt = w.torch_dtype
    out = {}
    out["X"] = _normal((w.n, w.d), 1.0, dt, device, _gen(device, w.seed, 0))
    out["Wg"] = _normal((w.d, w.E), (1.0 / w.d) ** 0.5, torch.float32, device,
                        _gen(device, w.seed, 1))
    if w.logit_skew_var > 0:
        out["logit_bias"] = _normal((w.E,), w.logit_skew_var ** 0.5, torch.float32, device,
                                    _gen(device, w.seed, 8))
    else:
        out["logit_bias"] = None
    out["sel_bias"] = (torch.zeros(w.E, dtype=torch.float32, device=device)
                       if w.score in ("sigmoid", "sqrtsoftplus") else None)
    if experts:
        big = w.E * w.h * w.d > (1 << 26)
        out["W1"] = _normal((w.E, w.h, w.d), (2.0 / w.d) ** 0.5, dt, device,
                            _gen(device, w.seed, 2), big)
        out["W3"] = (_normal((w.E, w.h, w.d), (2.0 / w.d) ** 0.5, dt, device,
                             _gen(device, w.seed, 3), big) if w.act == "swiglu" else None)
        out["W2"] = _normal((w.E, w.d, w.h), (2.0 / w.h) ** 0.5, dt, device,
                            _gen(device, w.seed, 4), big)
        if w.n_shared:
            out["sW1"] = _normal((w.n_shared, w.h, w.d), (2.0 / w.d) ** 0.5, dt, device,
                                 _gen(device, w.seed, 5), big)
            out["sW3"] = (_normal((w.n_shared, w.h, w.d), (2.0 / w.d) ** 0.5, dt, device,
                                  _gen(device, w.seed, 6), big) if w.act == "swiglu"
                          else None)
            out["sW2"] = _normal((w.n_shared, w.d, w.h), (2.0 / w.h) ** 0.5, dt, device,
                                 _gen(device, w.seed, 7), big)
    return out


def tie_heavy_scores(n: int, E: int, levels: int, seed: int, device="cpu") -> torch.Tensor:
    """A score matrix whose entries take only `levels` distinct values, so
    that top-k boundaries are full of exact ties (including +0 and -0)."""
    g = _gen(device, seed, 20)
    q = torch.randint(0, levels, (n, E), generator=g, device=device)
    S = q.to(torch.float32) / max(levels - 1, 1)
    # sprinkle negative zeros where the value is zero
    flip = torch.randint(0, 2, (n, E), generator=g, device=device).bool()
    S = torch.where((S == 0) & flip, torch.full_like(S, -0.0), S)
    return S


def random_scores(n: int, E: int, seed: int, device="cpu") -> torch.Tensor:
    """A softmax-like positive score matrix with continuous values."""
    g = _gen(device, seed, 21)
    return torch.rand((n, E), generator=g, device=device, dtype=torch.float32)
