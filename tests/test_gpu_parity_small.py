"""CUDA path vs the CPU oracle, element by element, on layers the oracle runs in
full: several tiles per expert, ragged segment tails, d and h that are not
multiples of the GEMM tiles, empty experts, k = E, k > 16, a single token, rows
wider than 16 column chunks, FP32."""
import numpy as np
import pytest
import torch

import oracle as O
from workloads import get_config, make_inputs

from tests.parity import LOGIT_TOL, TOL, check_index_parity, f64, i64, make_layer, rel_err, run_step

SMALL = ["small_bf16", "small_ragged_bf16", "small_skew_bf16", "small_kE_bf16", "small_f32", "one_token_bf16",
         "tiny_fp32", "small_pairs_bf16", "wide_d_bf16", "wide_d_f32", "big_k_bf16"]


@pytest.mark.gpu
@pytest.mark.parametrize("name", SMALL)
def test_layer_parity(name):
    cfg = get_config(name)
    tol = TOL[cfg.dtype]
    inp = make_inputs(cfg, seed=1, device="cuda")
    layer = make_layer(cfg)
    assert run_step(layer, inp) == 0, "device error word set"

    x, wg, bias, w1, w3, w2, dy = map(f64, (inp.x, inp.wg, inp.bias, inp.w1, inp.w3, inp.w2, inp.dy))
    z_gpu = layer.logits.cpu().numpy()
    assert rel_err(z_gpu, O.gate_logits(x, wg, bias)) <= LOGIT_TOL

    ids, w = check_index_parity(layer, cfg, O)

    # Values, with the oracle routed by the same logits (selection is compared above).
    fwd = O.layer_forward(x, wg, bias, w1, w3, w2, cfg.k, logits=z_gpu)
    N = cfg.N
    assert np.array_equal(f64(layer.x_pft[:N]), fwd["x_pft"])          # a copy: exact
    for nm, t in (("H1", layer.h1), ("H3", layer.h3), ("A", layer.a), ("O", layer.out)):
        e = rel_err(f64(t[:N]), fwd[nm])
        assert e <= tol, (nm, e)
    assert rel_err(f64(layer.y), fwd["y"]) <= tol

    bwd = O.layer_backward(fwd, dy, x, wg, w1, w3, w2)
    for nm, t in (("dx", layer.dx), ("dWg", layer.dwg), ("dW1", layer.dw1), ("dW3", layer.dw3),
                  ("dW2", layer.dw2), ("dlogits", layer.dlogits)):
        e = rel_err(f64(t), bwd[nm])
        assert e <= tol, (nm, e)
    # experts without rows get exact zeros
    empty = np.where(i64(layer.tokens_per_expert) == 0)[0]
    for e_ in empty:
        assert not layer.dw1[e_].any() and not layer.dw3[e_].any() and not layer.dw2[e_].any()


@pytest.mark.gpu
def test_oracle_routing_agrees_away_from_ties():
    # Selecting on the oracle's float64 logits must agree with the GPU wherever the
    # k-th / (k+1)-th gap is clear of float32 rounding.
    cfg = get_config("small_skew_bf16")
    inp = make_inputs(cfg, seed=2, device="cuda")
    layer = make_layer(cfg)
    run_step(layer, inp)
    z_ref = O.gate_logits(f64(inp.x), f64(inp.wg), f64(inp.bias))
    ids_ref, _ = O.route(z_ref, cfg.k)
    s = -np.sort(-z_ref, axis=1)
    clear = (s[:, cfg.k - 1] - s[:, cfg.k]) > 1e-4 * np.abs(z_ref).max()
    assert clear.mean() > 0.9
    assert np.array_equal(i64(layer.topk_ids)[clear], ids_ref[clear])


@pytest.mark.gpu
def test_deterministic_bytes():
    cfg = get_config("small_bf16")
    inp = make_inputs(cfg, seed=3, device="cuda")
    a, b = make_layer(cfg), make_layer(cfg)
    run_step(a, inp)
    run_step(b, inp)
    for nm in ("logits", "topk_ids", "pos", "x_pft", "h1", "out", "y", "dx", "dwg", "dw1", "dw3", "dw2",
               "dlogits", "replica_expert"):
        ta, tb = getattr(a, nm), getattr(b, nm)
        assert torch.equal(ta.view(torch.uint8) if ta.dtype.is_floating_point else ta,
                           tb.view(torch.uint8) if tb.dtype.is_floating_point else tb), nm
