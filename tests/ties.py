"""Layer inputs whose gate logits tie exactly.

x takes values in {-1, 0, 1} and the gate Wg values in {-2, ..., 2} / 8 (both exact
in BF16), and the bias is a multiple of 1/8.  Every product x_i Wg_ie is then a
multiple of 1/8 and every partial sum of at most a few thousand of them is an
exactly representable float32, so the logits come out the same, bit for bit,
whatever order the terms are summed in: on the GPU (tensor-core or CUDA-core GEMM,
split along K or not) and in the float64 oracle alike.  Only about 2d + 1 values
are possible, so equal logits are common, and duplicated gate columns make some
experts tie on every token.  The selection rule under test: rank by logit
descending, equal logits to the lower expert index (X-MoE article §1, large top-k
routing; the tie rule is this library's reading of the layer description).
"""
from __future__ import annotations

import torch

from workloads import make_inputs
from workloads.generate import storage_dtype


def tie_inputs(cfg, seed: int, device, dup_pairs: int = 0, zero_gate: bool = False, bias_levels=None):
    """make_inputs(cfg) with x, Wg (and optionally the bias) replaced by tie-prone values.

    dup_pairs: columns e = 2i + 1 copy column 2i for i < dup_pairs (those expert pairs tie on
    every token).  zero_gate: Wg = 0, so the logits are the bias alone (every token identical).
    bias_levels: the bias cycles through these values (multiples of 1/8)."""
    inp = make_inputs(cfg, seed=seed, device=device)
    dt = storage_dtype(cfg)
    g = torch.Generator(device="cpu").manual_seed(10_000 + seed)
    x = torch.randint(-1, 2, (cfg.T, cfg.d), generator=g).to(torch.float32)
    wg = torch.randint(-2, 3, (cfg.d, cfg.E), generator=g).to(torch.float32) / 8.0
    for i in range(dup_pairs):
        wg[:, 2 * i + 1] = wg[:, 2 * i]
    if zero_gate:
        wg.zero_()
    bias = None
    if bias_levels is not None:
        lv = torch.tensor(bias_levels, dtype=torch.float32)
        bias = lv[torch.arange(cfg.E) % len(lv)].contiguous().to(device)
    inp.x = x.to(dt).to(device)
    inp.wg = wg.to(dt).to(device)
    inp.bias = bias
    return inp
