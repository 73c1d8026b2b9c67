"""Seeded synthetic inputs for one MoE layer.

Distributions (one reading of the layer description; the pages give no data):

* x  ~ N(0, 1)              [T, d]
* Wg ~ N(0, 0.02^2)         [d, E]      (gate, std 0.02)
* W1, W3 ~ N(0, 1/d)        [E, d, h]   (variance 1/d)
* W2 ~ N(0, 1/h)            [E, h, d]   (variance 1/h)
* dY ~ N(0, 1)              [T, d]      (upstream gradient)
* optional Zipf bias        [E] float32: bias_e = -c * s * ln(perm(e) + 1), perm a seeded permutation

Draws are made in float32 with a ``torch.Generator`` seeded with ``seed`` on the
target device, in the fixed order x, Wg, W1, W3, W2, dY, perm, then rounded to
the storage type (BF16 or FP32).  The same seed gives different numbers on CPU
and GPU (different generator streams); every comparison feeds the *same* tensors
to both sides, so this does not matter.  Large weight tensors are drawn one
expert at a time so the float32 staging buffer stays small.
"""
from __future__ import annotations

import math
from dataclasses import dataclass
from typing import Optional

import torch

from .configs import LayerConfig


def storage_dtype(cfg: LayerConfig) -> torch.dtype:
    return torch.bfloat16 if cfg.dtype == "bf16" else torch.float32


@dataclass
class LayerInputs:
    cfg: LayerConfig
    x: torch.Tensor
    wg: torch.Tensor
    bias: Optional[torch.Tensor]
    w1: torch.Tensor
    w3: torch.Tensor
    w2: torch.Tensor
    dy: torch.Tensor

    def to(self, device) -> "LayerInputs":
        mv = lambda t: None if t is None else t.to(device)
        return LayerInputs(self.cfg, mv(self.x), mv(self.wg), mv(self.bias), mv(self.w1),
                           mv(self.w3), mv(self.w2), mv(self.dy))


def _normal(shape, std, gen, device, dtype):
    t = torch.randn(*shape, generator=gen, device=device, dtype=torch.float32)
    if std != 1.0:
        t.mul_(std)
    return t.to(dtype)


def _expert_stack(E, rows, cols, std, gen, device, dtype):
    out = torch.empty(E, rows, cols, device=device, dtype=dtype)
    for e in range(E):
        out[e].copy_(_normal((rows, cols), std, gen, device, dtype))
    return out


def make_inputs(cfg: LayerConfig, seed: int = 0, device="cpu") -> LayerInputs:
    dt = storage_dtype(cfg)
    gen = torch.Generator(device=device)
    gen.manual_seed(seed)
    x = _normal((cfg.T, cfg.d), 1.0, gen, device, dt)
    wg = _normal((cfg.d, cfg.E), 0.02, gen, device, dt)
    w1 = _expert_stack(cfg.E, cfg.d, cfg.h, 1.0 / math.sqrt(cfg.d), gen, device, dt)
    w3 = _expert_stack(cfg.E, cfg.d, cfg.h, 1.0 / math.sqrt(cfg.d), gen, device, dt)
    w2 = _expert_stack(cfg.E, cfg.h, cfg.d, 1.0 / math.sqrt(cfg.h), gen, device, dt)
    dy = _normal((cfg.T, cfg.d), 1.0, gen, device, dt)
    bias = None
    if cfg.zipf_c > 0:
        perm = torch.randperm(cfg.E, generator=gen, device=device)
        bias = (-cfg.zipf_c * cfg.zipf_s * torch.log(perm.to(torch.float64) + 1.0)).to(torch.float32)
    return LayerInputs(cfg, x, wg, bias, w1, w3, w2, dy)


def make_topk_ids(T: int, E: int, k: int, seed: int = 0, device="cpu") -> torch.Tensor:
    """Uniformly random distinct expert choices per token, [T, k] int32 (for index-only stress shapes)."""
    gen = torch.Generator(device=device)
    gen.manual_seed(seed)
    scores = torch.rand(T, E, generator=gen, device=device)
    return torch.argsort(scores, dim=1)[:, :k].to(torch.int32).contiguous()
