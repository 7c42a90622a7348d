"""Seeded synthetic inputs for the K2-style MoE FFN layer.

This module only draws random numbers and lays them out. It holds none of the
layer's arithmetic (no router, no top-k, no SwiGLU, no combine), so that both
the CPU oracle and the CUDA path can be fed from it without sharing any of the
method's code.

Workloads follow the layer shapes of the Kimi-K2 / DeepSeek-V3 MoE FFN
("Kimi K2.5 deep dive", CH4.1-4.3: 384 routed experts, top-8, 1 shared expert,
moe_intermediate_size 2048, hidden 7168; routed_scaling_factor 2.827 for K2 and
2.5 for DeepSeek-V3 per the K2 team member's answer, "Architecture / different").

Distributions (one reading per quantity):
  x            ~ N(0, 1)                    drawn fp32, rounded to bf16
  W (all)      ~ N(0, std = 1/sqrt(fan_in)) drawn fp32, rounded to bf16
               fan_in = d for router / gate / up, fan_in = inter for down
  bias         ~ U(-0.01, 0.01) fp32, or for the skewed workload
               b_e = 0.5 * ln(1 / (e + 1))  (Zipf-like expert loads)

Draw order on one torch.Generator seeded once: x, router weight, bias, then for
each routed expert e = 0..E-1: gate_e [I,d], up_e [I,d], down_e [d,I]; then the
shared expert's gate, up, down.  Each expert is drawn separately so the peak
temporary memory stays at one expert's fp32 weights.

Stacked layout handed to the library and the oracle:
  w_gate_up [E, 2I, d]  rows [0, I) = gate_proj, rows [I, 2I) = up_proj
  w_down    [E, d, I]
  ws_gate_up [2I, d], ws_down [d, I]   (the shared expert)
"""
from __future__ import annotations

import math
from dataclasses import dataclass, asdict

import torch


@dataclass(frozen=True)
class MoEConfig:
    name: str
    T: int
    d: int
    E: int
    k: int
    inter: int
    scale: float
    bias: str = "uniform"   # "uniform" | "zipf" | "zero"

    def as_dict(self):
        return asdict(self)


# The five workloads.  The first is small enough for the oracle to finish in
# seconds; the rest are full K2 / DeepSeek-V3 layer shapes.
CONFIGS = {
    "tiny": MoEConfig("tiny", T=64, d=512, E=32, k=4, inter=128, scale=2.827),
    "k2_decode": MoEConfig("k2_decode", T=64, d=7168, E=384, k=8, inter=2048, scale=2.827),
    "k2_prefill": MoEConfig("k2_prefill", T=8192, d=7168, E=384, k=8, inter=2048, scale=2.827),
    "k2_skew": MoEConfig("k2_skew", T=4096, d=7168, E=384, k=8, inter=2048, scale=2.827,
                         bias="zipf"),
    "v3": MoEConfig("v3", T=2048, d=7168, E=256, k=8, inter=2048, scale=2.5),
}


def _normal_bf16(shape, std, gen, device, out=None):
    t = torch.randn(shape, generator=gen, device=device, dtype=torch.float32)
    if std != 1.0:
        t.mul_(std)
    if out is None:
        return t.to(torch.bfloat16)
    out.copy_(t)
    return out


def make_bias(cfg: MoEConfig, gen, device):
    if cfg.bias == "uniform":
        b = torch.rand((cfg.E,), generator=gen, device=device, dtype=torch.float32)
        return b.mul_(0.02).sub_(0.01)
    if cfg.bias == "zipf":
        e = torch.arange(cfg.E, dtype=torch.float64)
        return (0.5 * torch.log(1.0 / (e + 1.0))).to(torch.float32).to(device)
    if cfg.bias == "zero":
        return torch.zeros((cfg.E,), dtype=torch.float32, device=device)
    raise ValueError(f"unknown bias kind {cfg.bias!r}")


def make_inputs(cfg: MoEConfig, seed: int = 0, device="cpu"):
    """All layer inputs for `cfg`, drawn in the documented order on `device`."""
    dev = torch.device(device)
    gen = torch.Generator(device=dev)
    gen.manual_seed(seed)
    T, d, E, I = cfg.T, cfg.d, cfg.E, cfg.inter
    x = _normal_bf16((T, d), 1.0, gen, dev)
    w_router = _normal_bf16((E, d), 1.0 / math.sqrt(d), gen, dev)
    bias = make_bias(cfg, gen, dev)
    if cfg.bias != "uniform":
        # keep the stream position identical to the uniform case
        torch.rand((E,), generator=gen, device=dev)
    w_gate_up = torch.empty((E, 2 * I, d), dtype=torch.bfloat16, device=dev)
    w_down = torch.empty((E, d, I), dtype=torch.bfloat16, device=dev)
    for e in range(E):
        _normal_bf16((I, d), 1.0 / math.sqrt(d), gen, dev, out=w_gate_up[e, :I])
        _normal_bf16((I, d), 1.0 / math.sqrt(d), gen, dev, out=w_gate_up[e, I:])
        _normal_bf16((d, I), 1.0 / math.sqrt(I), gen, dev, out=w_down[e])
    ws_gate_up = torch.empty((2 * I, d), dtype=torch.bfloat16, device=dev)
    _normal_bf16((I, d), 1.0 / math.sqrt(d), gen, dev, out=ws_gate_up[:I])
    _normal_bf16((I, d), 1.0 / math.sqrt(d), gen, dev, out=ws_gate_up[I:])
    ws_down = _normal_bf16((d, I), 1.0 / math.sqrt(I), gen, dev)
    return dict(x=x, w_router=w_router, bias=bias, w_gate_up=w_gate_up, w_down=w_down,
                ws_gate_up=ws_gate_up, ws_down=ws_down)


def make_topk_idx(T: int, E: int, k: int, seed: int = 0, device="cpu", skew: float = 0.0):
    """Random routing decisions: k distinct experts per token (int32 [T, k]).

    With skew > 0 the expert draw favours low indices (keys perturbed by
    -skew*log(e+1)), which gives ragged, uneven per-expert loads.
    """
    gen = torch.Generator(device=device)
    gen.manual_seed(seed)
    keys = torch.rand((T, E), generator=gen, device=device, dtype=torch.float64)
    if skew:
        keys = keys + skew * torch.log(torch.arange(E, dtype=torch.float64, device=device) + 1.0)
    return keys.argsort(dim=1)[:, :k].to(torch.int32).contiguous()


def make_combine_inputs(T: int, d: int, k: int, seed: int = 0, device="cpu"):
    """Random expert outputs, weights and a slot->row bijection for the combine stage."""
    gen = torch.Generator(device=device)
    gen.manual_seed(seed)
    y = torch.randn((T * k, d), generator=gen, device=device).to(torch.bfloat16)
    y_shared = torch.randn((T, d), generator=gen, device=device).to(torch.bfloat16)
    topk_w = torch.rand((T, k), generator=gen, device=device, dtype=torch.float32)
    slot_row = torch.randperm(T * k, generator=gen, device=device).to(torch.int32)
    return dict(y=y, y_shared=y_shared, topk_w=topk_w, slot_row=slot_row)
