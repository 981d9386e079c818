"""Seeded synthetic inputs for the MoE feed-forward layer.

This module is shared by the CUDA path's tests and benchmark and by the oracle's
tests. It holds none of the layer's arithmetic: only random draws, the scaling
of each weight by 1/sqrt(fan_in), the per-expert logit bias recipes and the bf16
rounding of stored tensors (round-to-nearest-even, done by torch's cast).

Recipe (the same on every device; the device's generator is part of it):

* one ``torch.Generator`` per tensor, seeded ``seed*1000 + i`` with i = 0..8 in
  the order x, W_g, bias, W1, W3, W2, W1s, W3s, W2s;
* fp32 standard normals, times 1/sqrt(fan_in), cast to bf16. x is N(0, 1);
  W_g, W1, W3, W1s, W3s have fan_in = d; W2 has fan_in = f; W2s has N_s*f;
* stacked routed weights are drawn one expert at a time from their generator,
  so peak temporary memory is one expert's fp32 matrix;
* bias "normal_var0.5": fp32 N(0, 0.5) per routed expert; bias "zipf1.1": a
  seeded permutation ranks the experts 1..N_r and expert e gets
  -1.1*ln(rank_e), a Zipf(s = 1.1) popularity in log space;
* the layouts are the library's: x (T, d); W_g (N_r, d); W1, W3 (N_r, f, d);
  W2 (N_r, d, f); W1s, W3s (N_s*f, d); W2s (d, N_s*f); bias (N_r,) fp32.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, replace
from typing import Dict, Optional

import torch

__all__ = ["LayerShape", "WORKLOADS", "make_layer_inputs"]


@dataclass(frozen=True)
class LayerShape:
    """Sizes of one MoE layer invocation: T tokens of width d, N_r routed experts
    of inner width f with top-k routing, N_s shared experts fused to inner N_s*f."""

    name: str
    T: int
    d: int
    f: int
    n_routed: int
    top_k: int
    n_shared: int
    renorm: bool
    bias: str = "none"          # "none" | "normal_var0.5" | "zipf1.1"

    def with_tokens(self, T: int) -> "LayerShape":
        return replace(self, T=T)

    def with_experts(self, n_routed: int) -> "LayerShape":
        """The same layer with fewer (or more) routed experts, top_k kept."""
        return replace(self, n_routed=max(n_routed, self.top_k))


# The layer shapes the pages describe, named by what they are.
WORKLOADS: Dict[str, LayerShape] = {
    # 31 fine-grained routed experts top-7 + 1 shared, the page's equal-budget toy
    "tiny_t256_d128_f64_e31k7_s1": LayerShape(
        "tiny_t256_d128_f64_e31k7_s1", 256, 128, 64, 31, 7, 1, True),
    # Mixtral-like coarse layer: 8 experts top-2, no shared expert
    "coarse_t4096_d4096_f14336_e8k2_s0": LayerShape(
        "coarse_t4096_d4096_f14336_e8k2_s0", 4096, 4096, 14336, 8, 2, 0, True),
    # DeepSeekMoE-small: 64 routed top-6 + 2 shared fused (inner 2816), raw gates
    "dsmoe_small_t8192_d2048_f1408_e64k6_s2": LayerShape(
        "dsmoe_small_t8192_d2048_f1408_e64k6_s2", 8192, 2048, 1408, 64, 6, 2, False),
    # DeepSeek-V3-shaped prefill: 256 routed top-8 + 1 shared, skewed by a bias
    "dsv3_prefill_t4096_d7168_f2048_e256k8_s1": LayerShape(
        "dsv3_prefill_t4096_d7168_f2048_e256k8_s1", 4096, 7168, 2048, 256, 8, 1, True,
        "normal_var0.5"),
    # 512-expert decode step: 128 tokens, top-10 + 1 shared, hot-expert skew
    "decode_t128_d2048_f512_e512k10_s1": LayerShape(
        "decode_t128_d2048_f512_e512k10_s1", 128, 2048, 512, 512, 10, 1, True,
        "zipf1.1"),
}


def _gen(seed: int, i: int, device) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(seed * 1000 + i)
    return g


def _normal_bf16(shape, gen, device, scale: float) -> torch.Tensor:
    v = torch.randn(shape, generator=gen, device=device, dtype=torch.float32)
    return (v * scale).to(torch.bfloat16)


def _stacked_bf16(n: int, rows: int, cols: int, gen, device, scale: float):
    out = torch.empty((n, rows, cols), dtype=torch.bfloat16, device=device)
    for e in range(n):
        out[e].copy_(_normal_bf16((rows, cols), gen, device, scale))
    return out


def make_layer_inputs(shape: LayerShape, seed: int = 0, device="cpu",
                      T: Optional[int] = None) -> Dict[str, Optional[torch.Tensor]]:
    """Draw every input of one layer invocation following the module's recipe.

    Returns a dict with keys x, W_g, bias, W1, W3, W2, W1s, W3s, W2s (the shared
    ones None when N_s = 0, bias None for the "none" recipe)."""
    T = shape.T if T is None else T
    d, f, n, ns = shape.d, shape.f, shape.n_routed, shape.n_shared
    dev = torch.device(device)
    out: Dict[str, Optional[torch.Tensor]] = {}
    out["x"] = _normal_bf16((T, d), _gen(seed, 0, dev), dev, 1.0)
    out["W_g"] = _normal_bf16((n, d), _gen(seed, 1, dev), dev, 1.0 / math.sqrt(d))
    gb = _gen(seed, 2, dev)
    if shape.bias == "none":
        out["bias"] = None
    elif shape.bias == "normal_var0.5":
        out["bias"] = torch.randn((n,), generator=gb, device=dev,
                                  dtype=torch.float32) * math.sqrt(0.5)
    elif shape.bias == "zipf1.1":
        rank = torch.randperm(n, generator=gb, device=dev).to(torch.float32) + 1.0
        out["bias"] = -1.1 * torch.log(rank)
    else:
        raise ValueError(f"unknown bias recipe {shape.bias!r}")
    out["W1"] = _stacked_bf16(n, f, d, _gen(seed, 3, dev), dev, 1.0 / math.sqrt(d))
    out["W3"] = _stacked_bf16(n, f, d, _gen(seed, 4, dev), dev, 1.0 / math.sqrt(d))
    out["W2"] = _stacked_bf16(n, d, f, _gen(seed, 5, dev), dev, 1.0 / math.sqrt(f))
    if ns > 0:
        fs = ns * f
        out["W1s"] = _normal_bf16((fs, d), _gen(seed, 6, dev), dev, 1.0 / math.sqrt(d))
        out["W3s"] = _normal_bf16((fs, d), _gen(seed, 7, dev), dev, 1.0 / math.sqrt(d))
        out["W2s"] = _normal_bf16((d, fs), _gen(seed, 8, dev), dev, 1.0 / math.sqrt(fs))
    else:
        out["W1s"] = out["W3s"] = out["W2s"] = None
    return out
