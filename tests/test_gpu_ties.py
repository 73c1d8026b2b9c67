"""Exact logit ties and non-finite logits on the GPU.

The tie layers use the quantised inputs of tests/ties.py: their float32 logits are
exact, so the GPU must reproduce the oracle's float64 logits bit for bit and its
selection must equal the oracle's own (not merely the oracle routed on the GPU's
logits).  Every index output (top-k ids, PFT, RBD) is compared bit for bit and the
values element-wise within the usual tolerance.  The CPU test
tests/test_ties_cpu.py shows that these inputs decide selections by the tie rule,
so a kernel that broke ties the other way would fail here.

The non-finite cases check the device error word: a NaN logit ranks below every
number and sets PFMOE_DEV_NONFINITE; so does a token whose largest logit is
+inf (its weights are undefined).
"""
import numpy as np
import pytest
import torch

import oracle as O
from padding_free_moe_b200 import _lib as L
from workloads import get_config

from tests.parity import TOL, f64, i64, make_layer, rel_err, run_step
from tests.ties import tie_inputs

CASES = {
    # name: (base config, overrides, tie_inputs keyword arguments)
    "dup_cols_bf16": ("small_bf16", dict(d=64, h=64, k=4), dict(dup_pairs=6)),
    "many_ties_e512_k16": ("small_bf16", dict(T=256, d=64, E=512, h=64, k=16, rbd_epd=16, rbd_dpn=8),
                           dict(dup_pairs=64)),
    "bias_only_bf16": ("small_bf16", dict(T=200, d=64, E=32, h=64, k=5, rbd_epd=4, rbd_dpn=2),
                       dict(zero_gate=True, bias_levels=[1.0, 0.5, 0.5, 0.0])),
    "ties_plus_bias_bf16": ("small_ragged_bf16", dict(d=64), dict(dup_pairs=3, bias_levels=[0.25, 0.0, 0.25])),
    "dup_cols_f32": ("small_f32", dict(d=64, E=12, k=3, rbd_epd=3, rbd_dpn=2), dict(dup_pairs=4)),
}


def case_inputs(name, device):
    base, over, kw = CASES[name]
    cfg = get_config(base).with_(name=name, **over)
    return cfg, tie_inputs(cfg, seed=4, device=device, **kw)


@pytest.mark.gpu
@pytest.mark.parametrize("name", sorted(CASES))
def test_exact_ties_match_oracle(name):
    cfg, inp = case_inputs(name, "cuda")
    layer = make_layer(cfg)
    assert run_step(layer, inp) == 0, "device error word set"
    x, wg, bias, w1, w3, w2, dy = map(f64, (inp.x, inp.wg, inp.bias, inp.w1, inp.w3, inp.w2, inp.dy))
    z_ref = O.gate_logits(x, wg, bias)
    z_gpu = layer.logits.cpu().numpy().astype(np.float64)
    assert np.array_equal(z_gpu, z_ref), "quantised logits must be exact on both sides"
    # the oracle routes on its own logits: selection, PFT and RBD must agree bit for bit
    fwd = O.layer_forward(x, wg, bias, w1, w3, w2, cfg.k)
    assert np.array_equal(i64(layer.topk_ids), fwd["ids"])
    assert np.abs(layer.topk_w.cpu().numpy() - fwd["w"]).max() <= 2e-6
    p = fwd["pft"]
    for nm, t in (("tokens_per_expert", layer.tokens_per_expert), ("expert_offsets", layer.expert_offsets),
                  ("tile_offsets", layer.tile_offsets), ("pos", layer.pos)):
        assert np.array_equal(i64(t), p[nm]), nm
    N = cfg.N
    assert np.array_equal(i64(layer.token_ids[:N]), p["token_ids"])
    assert np.array_equal(i64(layer.expert_ids[:N]), p["expert_ids"])
    if layer.has_rbd:
        r = O.rbd_plan(fwd["ids"], cfg.E, cfg.rbd_epd, cfg.rbd_dpn)
        P = r["num_pilots"]
        assert int(layer.rbd_counts[0]) == P and int(layer.rbd_counts[1]) == r["num_token_device_pairs"]
        assert np.array_equal(i64(layer.pilot_token[:P]), r["pilot_token"])
        assert np.array_equal(i64(layer.pilot_node[:P]), r["pilot_node"])
        assert np.array_equal(i64(layer.pilot_device[:P]), r["pilot_device"])
        assert np.array_equal(i64(layer.replica_offsets[:P + 1]), r["replica_offsets"])
        assert np.array_equal(i64(layer.replica_expert[:N]), r["replica_expert"])
        assert np.array_equal(i64(layer.assign_pilot), r["assign_pilot"])
    # values
    tol = TOL[cfg.dtype]
    assert rel_err(f64(layer.y), fwd["y"]) <= tol
    bwd = O.layer_backward(fwd, dy, x, wg, w1, w3, w2)
    for nm, t in (("dx", layer.dx), ("dWg", layer.dwg), ("dW1", layer.dw1), ("dW3", layer.dw3),
                  ("dW2", layer.dw2), ("dlogits", layer.dlogits)):
        e = rel_err(f64(t), bwd[nm])
        assert e <= tol, (nm, e)


def _route(cfg, x, wg, bias):
    T, d, E, k = cfg.T, cfg.d, cfg.E, cfg.k
    code = L.PFMOE_BF16 if cfg.dtype == "bf16" else L.PFMOE_F32
    logits = torch.empty(T, E, device="cuda")
    ids = torch.empty(T, k, device="cuda", dtype=torch.int32)
    w = torch.empty(T, k, device="cuda")
    ws_b = L.moe_route_workspace_size(T, d, E, k, code)
    ws = torch.empty(max(ws_b, 256), device="cuda", dtype=torch.uint8)
    err = torch.zeros(1, device="cuda", dtype=torch.int32)
    L.moe_route(x, wg, bias, T, d, E, k, code, logits, ids, w, ws, ws_b, err)
    torch.cuda.synchronize()
    return logits.cpu().numpy(), i64(ids), w.cpu().numpy(), int(err)


@pytest.mark.gpu
@pytest.mark.parametrize("base", ["small_bf16", "small_f32"])
def test_nan_logit_ranks_last_and_is_flagged(base):
    cfg = get_config(base)
    cfg = cfg.with_(k=min(cfg.k, cfg.E - 2))
    inp = tie_inputs(cfg, seed=5, device="cuda")
    bias = torch.zeros(cfg.E, device="cuda")
    bias[3] = float("nan")                        # expert 3's logit is NaN on every token
    z, ids, w, err = _route(cfg, inp.x, inp.wg, bias)
    assert err & L.DEV_NONFINITE
    assert np.isnan(z[:, 3]).all()
    ids_ref, w_ref = O.route(z, cfg.k)            # numpy ranks NaN after every number too
    assert np.array_equal(ids, ids_ref)
    assert not (ids == 3).any()
    assert np.isfinite(w).all() and np.abs(w - w_ref).max() <= 2e-6


@pytest.mark.gpu
def test_nan_token_row_is_flagged_and_others_unaffected():
    cfg = get_config("small_bf16")
    inp = tie_inputs(cfg, seed=6, device="cuda")
    x = inp.x.clone()
    x[17, 5] = float("nan")                       # every logit of token 17 is NaN
    z, ids, w, err = _route(cfg, x, inp.wg, None)
    assert err & L.DEV_NONFINITE
    assert np.isnan(z[17]).all()
    ok = np.ones(cfg.T, dtype=bool)
    ok[17] = False
    ids_ref, w_ref = O.route(z[ok], cfg.k)
    assert np.array_equal(ids[ok], ids_ref)
    assert np.abs(w[ok] - w_ref).max() <= 2e-6
    # all of token 17's logits rank equal (NaN): the k lowest expert ids, in order
    assert np.array_equal(ids[17], np.arange(cfg.k))


@pytest.mark.gpu
def test_infinite_max_logit_is_flagged():
    cfg = get_config("small_bf16")
    inp = tie_inputs(cfg, seed=7, device="cuda")
    bias = torch.zeros(cfg.E, device="cuda")
    bias[2] = float("inf")
    z, ids, w, err = _route(cfg, inp.x, inp.wg, bias)
    assert err & L.DEV_NONFINITE
    assert (ids[:, 0] == 2).all()
    # finite logits raise no flag
    _, _, w2, err2 = _route(cfg, inp.x, inp.wg, None)
    assert err2 == 0 and np.isfinite(w2).all()
