"""Seeded synthetic inputs for the MoE layer (shared by the CUDA path's tests,
the benchmark and the oracle's tests; holds none of the layer's arithmetic).

Recipe, per workload (sizes in ``configs.py``):
  x        [T, d]    N(0, 1) drawn in fp32, cast to bf16 (round to nearest even)
  w_router [d, E]    N(0, 1/d) in fp32  (std = 1/sqrt(fan_in), fan_in = d)
  bias     [E]       None, or -s*ln(e+1) for the skewed workload: the log of a
                     Zipf(s) rank weight with rank e+1 (the normalising constant
                     is dropped; it cancels in the renormalised softmax and
                     does not move the top-k)
  w_gate   [E, d, f] N(0, 1/d) -> bf16
  w_up     [E, d, f] N(0, 1/d) -> bf16
  w_down   [E, f, d] N(0, 1/f) -> bf16
Every tensor has its own stream derived from (seed, tensor id), so the same
seed gives the same values whether a tensor is drawn on the CPU or, for the
large workloads, on the GPU (torch's Philox generator on that device; the two
devices give different but individually reproducible values).
"""
import math
from typing import Dict, Optional

import torch

from .configs import MoEConfig

_STREAM = {"x": 1, "w_router": 2, "w_gate": 3, "w_up": 4, "w_down": 5}


def _gen(device, seed: int, name: str) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(seed * 1000003 + _STREAM[name])
    return g


def _normal(shape, std, device, seed, name) -> torch.Tensor:
    """N(0, std^2) in fp32."""
    g = _gen(device, seed, name)
    return torch.randn(shape, generator=g, device=device, dtype=torch.float32).mul_(std)


def _normal_bf16(shape, std, device, seed, name) -> torch.Tensor:
    """N(0, std^2) cast to bf16, drawn one leading-index slice at a time so that
    the fp32 staging buffer stays one slice big."""
    g = _gen(device, seed, name)
    out = torch.empty(shape, dtype=torch.bfloat16, device=device)
    for i in range(shape[0]):
        out[i].copy_(torch.randn(shape[1:], generator=g, device=device,
                                 dtype=torch.float32).mul_(std))
    return out


def router_bias(cfg: MoEConfig, device="cpu") -> Optional[torch.Tensor]:
    if cfg.zipf_s is None:
        return None
    e = torch.arange(cfg.E, dtype=torch.float64)
    return (-cfg.zipf_s * torch.log(e + 1.0)).to(torch.float32).to(device)


def make_tokens(cfg: MoEConfig, device="cpu", seed: Optional[int] = None) -> torch.Tensor:
    s = cfg.seed if seed is None else seed
    return _normal((cfg.T, cfg.d), 1.0, device, s, "x").to(torch.bfloat16)


def make_weights(cfg: MoEConfig, device="cpu") -> Dict[str, torch.Tensor]:
    s = cfg.seed
    return {
        "w_router": _normal((cfg.d, cfg.E), 1.0 / math.sqrt(cfg.d), device, s, "w_router"),
        "bias": router_bias(cfg, device),
        "w_gate": _normal_bf16((cfg.E, cfg.d, cfg.f), 1.0 / math.sqrt(cfg.d), device, s, "w_gate"),
        "w_up": _normal_bf16((cfg.E, cfg.d, cfg.f), 1.0 / math.sqrt(cfg.d), device, s, "w_up"),
        "w_down": _normal_bf16((cfg.E, cfg.f, cfg.d), 1.0 / math.sqrt(cfg.f), device, s, "w_down"),
    }


def make_inputs(cfg: MoEConfig, device="cpu") -> Dict[str, torch.Tensor]:
    out = make_weights(cfg, device)
    out["x"] = make_tokens(cfg, device)
    return out
