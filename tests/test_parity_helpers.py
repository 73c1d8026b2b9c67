"""The full-size parity helper (tests/parity.py: sampled_layer with LazyExperts)
equals the oracle's whole-layer forward and backward on a small layer (CPU only)."""
import numpy as np
import torch

import oracle as O
from workloads import get_config, make_inputs

from tests.parity import LazyExperts, f64, sampled_layer


def test_sampled_layer_equals_full_layer():
    cfg = get_config("small_ragged_bf16")
    inp = make_inputs(cfg, seed=3, device="cpu")
    x, wg, bias, w1, w3, w2, dy = map(f64, (inp.x, inp.wg, inp.bias, inp.w1, inp.w3, inp.w2, inp.dy))
    z = O.gate_logits(x, wg, bias).astype(np.float32)
    fwd = O.layer_forward(x, wg, None, w1, w3, w2, cfg.k, logits=z)
    bwd = O.layer_backward(fwd, dy, x, wg, w1, w3, w2)
    rng = np.random.default_rng(0)
    S = np.sort(rng.choice(cfg.T, size=40, replace=False))
    ref = sampled_layer(O, S, z, x, wg, LazyExperts(inp.w1), LazyExperts(inp.w3), LazyExperts(inp.w2), dy, cfg.k)
    assert np.allclose(ref["y"], fwd["y"][S], rtol=1e-12, atol=1e-12)
    assert np.allclose(ref["dx"], bwd["dx"][S], rtol=1e-12, atol=1e-12)
    assert np.allclose(ref["dlogits"], bwd["dlogits"][S], rtol=1e-12, atol=1e-12)
    # dWg columns whose routed tokens all lie in S are complete
    e = int(fwd["ids"][S[0], 0])
    S2 = np.where((fwd["ids"] == e).any(axis=1))[0]
    ref2 = sampled_layer(O, S2, z, x, wg, LazyExperts(inp.w1), LazyExperts(inp.w3), LazyExperts(inp.w2), dy, cfg.k)
    assert np.allclose(ref2["dWg"][:, e], bwd["dWg"][:, e], rtol=1e-12, atol=1e-12)
