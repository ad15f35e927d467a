"""Seeded synthetic inputs for the routed-expert MoE layer.

This module only draws random numbers with the shapes and distributions of the
workloads; it holds none of the method's arithmetic (no quantisation, routing
or FFN).  Tests hand the same arrays to the CUDA library and to the oracle.

Distributions (the workload statement of the layer):
  expert weights  W ~ N(0, 0.02) fp32, one seed per (config, layer, expert, matrix)
  router gate     G [E, H] ~ N(0, 0.02) fp32
  router bias     U(-a, a), or Zipf(s=1.1) over a seeded random expert ranking,
                  bias_e = 0.5 * rank_e^-1.1 (the magnitude 0.5 is a chosen value; none is given)
  activations     x ~ N(0, 1) rounded to bf16, one seed per call
"""
from dataclasses import dataclass, field, replace
import hashlib

import torch


@dataclass(frozen=True)
class LayerConfig:
    name: str
    H: int
    I: int
    E: int
    k: int
    n_group: int
    topk_group: int
    rsf: float = 2.5
    bias_kind: str = "uniform"      # "uniform" or "zipf"
    bias_amp: float = 0.05
    shared: bool = True
    bits: int = 4
    T: int = 1
    topp: float = 0.0
    layers: int = 1
    eps: float = 1e-6

    def with_(self, **kw):
        return replace(self, **kw)


# The five workloads (tiny parity case, GLM-scale decode, small batches with a
# skewed router, 4096-token prefill, 16-layer stack).
TINY = LayerConfig("tiny H256 I128 E8 top2", H=256, I=128, E=8, k=2, n_group=1, topk_group=1,
                   bias_amp=0.1, T=4)
DECODE = LayerConfig("glm-scale decode H6144 I2048 E256+1 top8", H=6144, I=2048, E=256, k=8,
                     n_group=8, topk_group=4, T=1)
SMALL_BATCH = DECODE.with_(name="glm-scale small batch, zipf bias", bias_kind="zipf", T=8)
PREFILL = DECODE.with_(name="glm-scale prefill T4096", T=4096)
STACK = DECODE.with_(name="16-layer int4 stack", layers=16, T=1)
STACK_INT8 = DECODE.with_(name="8-layer int8 stack", layers=8, bits=8, T=1)
STACK_INT2 = DECODE.with_(name="16-layer int2 stack", layers=16, bits=2, T=1)


def seed_of(*parts) -> int:
    """A 63-bit seed from any tuple of labels (stable across processes)."""
    h = hashlib.sha256(repr(parts).encode()).digest()
    return int.from_bytes(h[:8], "little") & ((1 << 63) - 1)


def _gen(seed: int, device) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    return g


def normal(shape, std: float, seed: int, device="cpu") -> torch.Tensor:
    g = _gen(seed, device)
    return torch.randn(shape, generator=g, device=device, dtype=torch.float32) * std


def expert_weight(cfg: LayerConfig, layer: int, expert: int, matrix: str, device="cpu"):
    """fp32 weight of one expert matrix; expert == cfg.E is the shared expert.
    gate/up are [I, H], down is [H, I]."""
    shape = (cfg.I, cfg.H) if matrix in ("gate", "up") else (cfg.H, cfg.I)
    return normal(shape, 0.02, seed_of(cfg.H, cfg.I, cfg.E, layer, expert, matrix), device)


def router_gate(cfg: LayerConfig, layer: int = 0, device="cpu"):
    return normal((cfg.E, cfg.H), 0.02, seed_of(cfg.H, cfg.E, layer, "router-gate"), device)


def router_bias(cfg: LayerConfig, layer: int = 0, device="cpu"):
    g = _gen(seed_of(cfg.E, layer, cfg.bias_kind, cfg.bias_amp, "router-bias"), "cpu")
    if cfg.bias_kind == "zipf":
        rank = torch.randperm(cfg.E, generator=g).to(torch.float64) + 1.0
        b = (0.5 * rank.pow(-1.1)).to(torch.float32)
    else:
        b = (torch.rand(cfg.E, generator=g, dtype=torch.float32) * 2.0 - 1.0) * cfg.bias_amp
    return b.to(device)


def activations(T: int, H: int, seed: int, device="cpu"):
    """x ~ N(0,1) rounded to bf16."""
    return normal((T, H), 1.0, seed_of("x", T, H, seed), device).to(torch.bfloat16)


def bf16_bits(t: torch.Tensor):
    """uint16 bit pattern (numpy) of a bf16 tensor."""
    return t.detach().cpu().contiguous().view(torch.int16).numpy().view("uint16")
