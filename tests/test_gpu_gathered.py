"""The gathered expert FFN (moe_expert_ffn_gathered): the dispatch gather fused into the
first expert GEMM (PFTMoELayer(fused_gather=True)).

It must write no [N, d] copy of x, and its outputs must equal those of the
materialised path (moe_dispatch -> moe_expert_ffn) bit for bit: both feed the same
BF16 rows to the same MMAs in the same order, only the copy into shared memory
differs.  The oracle comparisons below cover d that is not a multiple of the
128-column K step (zero-filled columns), one-token and 256-token-plus tiles, wide
rows and k > 16; the step tests compare the whole fused step (forward, RBD plan,
backward) with the materialised one, at full size too.
"""
import numpy as np
import pytest
import torch

import oracle as O
from workloads import get_config, make_inputs

from tests.parity import TOL, f64, make_layer, rel_err, run_step

SHAPES = ["small_bf16", "small_ragged_bf16", "small_skew_bf16", "small_kE_bf16", "one_token_bf16",
          "small_pairs_bf16", "wide_d_bf16", "big_k_bf16"]
SENTINEL = -12345   # int16 view of the bytes the forward must leave in x_pft


def _forward_both(cfg, seed):
    inp = make_inputs(cfg, seed=seed, device="cuda")
    layer = make_layer(cfg)
    layer.fused_gather = True
    layer.x_pft.view(torch.int16).fill_(SENTINEL)
    layer.err.zero_()
    layer.forward(inp.x, inp.wg, inp.bias, inp.w1, inp.w3, inp.w2)
    torch.cuda.synchronize()
    assert layer.device_error() == 0
    untouched = bool((layer.x_pft.view(torch.int16) == SENTINEL).all())
    fused = {nm: getattr(layer, nm).clone() for nm in ("h1", "h3", "a", "out", "y")}
    # the materialised path on the same layer and inputs
    layer.fused_gather = False
    layer.forward(inp.x, inp.wg, inp.bias, inp.w1, inp.w3, inp.w2)
    torch.cuda.synchronize()
    assert layer.device_error() == 0
    ref = {nm: getattr(layer, nm) for nm in fused}
    return inp, layer, untouched, fused, ref


@pytest.mark.gpu
@pytest.mark.parametrize("name", SHAPES)
def test_gathered_forward_writes_no_pft_copy_and_matches_bitwise(name):
    cfg = get_config(name)
    inp, layer, untouched, fused, ref = _forward_both(cfg, seed=11)
    assert untouched, "the gathered forward wrote x_pft"
    N = cfg.N
    for nm in ("h1", "h3", "a", "out"):
        assert torch.equal(fused[nm][:N].view(torch.int16), ref[nm][:N].view(torch.int16)), nm
    assert torch.equal(fused["y"].view(torch.int16), ref["y"].view(torch.int16))
    # and against the oracle, routed on the GPU's logits
    x, wg, bias, w1, w3, w2 = map(f64, (inp.x, inp.wg, inp.bias, inp.w1, inp.w3, inp.w2))
    fwd = O.layer_forward(x, wg, bias, w1, w3, w2, cfg.k, logits=layer.logits.cpu().numpy())
    for nm, key in (("h1", "H1"), ("h3", "H3"), ("a", "A"), ("out", "O")):
        assert rel_err(f64(fused[nm][:N]), fwd[key]) <= TOL[cfg.dtype], nm
    assert rel_err(f64(fused["y"]), fwd["y"]) <= TOL[cfg.dtype]


@pytest.mark.gpu
def test_gathered_forward_full_size_matches_materialised_path():
    cfg = get_config("dsv3_bf16")
    _, _, untouched, fused, ref = _forward_both(cfg, seed=12)
    assert untouched
    for nm in ("h1", "h3", "a", "out", "y"):
        assert torch.equal(fused[nm].view(torch.int16), ref[nm].view(torch.int16)), nm


@pytest.mark.gpu
@pytest.mark.parametrize("name", ["small_ragged_bf16", "small_pairs_bf16", "small_skew_bf16", "dsv3_bf16",
                                  "dsv3_zipf_bf16"])
def test_gathered_step_equals_materialised_step(name):
    # forward, RBD plan and backward: every output bit for bit
    cfg = get_config(name)
    inp = make_inputs(cfg, seed=13, device="cuda")
    outs = []
    for fused in (True, False):
        layer = make_layer(cfg)
        layer.fused_gather = fused
        assert run_step(layer, inp) == 0
        outs.append({nm: getattr(layer, nm).clone() for nm in
                     ("y", "dx", "dwg", "dw1", "dw3", "dw2", "dlogits", "x_pft", "h1", "out")})
        del layer
    for nm in outs[0]:
        a, b = outs[0][nm], outs[1][nm]
        assert torch.equal(a.view(torch.uint8), b.view(torch.uint8)), nm


@pytest.mark.gpu
def test_gathered_entry_rejects_f32():
    from padding_free_moe_b200 import _lib as L
    cfg = get_config("small_f32")
    z = torch.zeros(16, device="cuda")
    with pytest.raises(L.PFMoEError):
        L.moe_expert_ffn_gathered(z, z, z, z, cfg.N, cfg.E, cfg.d, cfg.h, L.PFMOE_F32, z, z, z, z, z, z, z)
