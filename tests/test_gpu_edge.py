"""Edge cases of the CUDA path: no tokens, out-of-range indices reported through
the device error word (nothing traps), a bounded wait that runs out, and argument
errors from a live context."""
import numpy as np
import pytest
import torch

import oracle as O
from padding_free_moe_b200 import _lib as L
from workloads import get_config, make_inputs

from tests.parity import i64, make_layer, run_step


@pytest.mark.gpu
def test_zero_tokens():
    cfg = get_config("small_bf16").with_(T=0)
    layer = make_layer(cfg)
    inp = make_inputs(cfg, seed=0, device="cuda")
    for t in (layer.expert_offsets, layer.tile_offsets, layer.tokens_per_expert, layer.node_offsets,
              layer.pilots_per_node, layer.rbd_counts, layer.replica_offsets):
        t.fill_(-7)
    layer.dw1.fill_(3.0); layer.dw3.fill_(3.0); layer.dw2.fill_(3.0); layer.dwg.fill_(3.0)
    assert run_step(layer, inp) == 0
    for t in (layer.expert_offsets, layer.tile_offsets, layer.tokens_per_expert, layer.node_offsets,
              layer.pilots_per_node, layer.rbd_counts):
        assert not t.any()
    assert int(layer.replica_offsets[0]) == 0
    for t in (layer.dw1, layer.dw3, layer.dw2, layer.dwg):
        assert not t.any()


@pytest.mark.gpu
def test_bad_expert_ids_set_error_bit():
    T, E, k = 50, 16, 2
    ids = torch.randint(0, E, (T, k), device="cuda", dtype=torch.int32)
    ids[7, 1] = E          # out of range
    ids[9, 0] = -3
    w = torch.full((T, k), 0.5, device="cuda")
    out = {n: torch.zeros(sz, device="cuda", dtype=torch.int32) for n, sz in
           (("tpe", E), ("off", E + 1), ("tok", T * k), ("eid", T * k), ("pos", T * k), ("tiles", E + 1))}
    cw = torch.zeros(T * k, device="cuda")
    ws_b = L.pft_build_workspace_size(T, E, k)
    ws = torch.empty(ws_b, device="cuda", dtype=torch.uint8)
    err = torch.zeros(1, device="cuda", dtype=torch.int32)
    L.pft_build(ids, w, T, E, k, out["tpe"], out["off"], out["tok"], out["eid"], cw, out["pos"], out["tiles"], ws,
                ws_b, err)
    torch.cuda.synchronize()
    assert int(err) & L.DEV_BAD_EXPERT_ID
    # the valid assignments are all counted
    assert int(out["tpe"].sum()) == T * k - 2


@pytest.mark.gpu
def test_bad_pos_sets_error_bit():
    T, k, d = 10, 2, 64
    o = torch.randn(T * k, d, device="cuda").to(torch.bfloat16)
    pos = torch.arange(T * k, device="cuda", dtype=torch.int32).view(T, k).contiguous()
    pos[3, 1] = T * k + 5
    w = torch.full((T, k), 0.5, device="cuda")
    y = torch.zeros(T, d, device="cuda", dtype=torch.bfloat16)
    err = torch.zeros(1, device="cuda", dtype=torch.int32)
    L.moe_combine(o, pos, w, T, k, d, L.PFMOE_BF16, y, err)
    torch.cuda.synchronize()
    assert int(err) & L.DEV_BAD_POS
    assert not y[3].any()          # the bad token was skipped


@pytest.mark.gpu
def test_argument_error_message():
    x = torch.zeros(4, 64, device="cuda", dtype=torch.bfloat16)
    with pytest.raises(L.PFMoEError, match="k <= E"):
        L.moe_route(x, x, None, 4, 64, 8, 9, L.PFMOE_BF16, x, x, x)


@pytest.mark.gpu
def test_rbd_stress_shape_matches_oracle():
    # A large index-only shape (no expert maths): 2^17 tokens, 256 experts, k = 8, 8 nodes.
    from workloads.generate import make_topk_ids
    T, E, k, epd, dpn = 1 << 17, 256, 8, 8, 4
    ids = make_topk_ids(T, E, k, seed=5, device="cuda")
    n_nodes = E // (epd * dpn)
    pmax = T * min(k, n_nodes)
    i32 = dict(device="cuda", dtype=torch.int32)
    o = dict(ppn=torch.empty(n_nodes, **i32), noff=torch.empty(n_nodes + 1, **i32), ptok=torch.empty(pmax, **i32),
             pnode=torch.empty(pmax, **i32), pdev=torch.empty(pmax, **i32), roff=torch.empty(pmax + 1, **i32),
             rexp=torch.empty(T * k, **i32), ap=torch.empty(T, k, **i32), cnt=torch.empty(2, **i32))
    ws_b = L.rbd_plan_workspace_size(T, k, E, epd, dpn)
    ws = torch.empty(ws_b, device="cuda", dtype=torch.uint8)
    err = torch.zeros(1, **i32)
    L.rbd_plan(ids, T, k, E, epd, dpn, o["ppn"], o["noff"], o["ptok"], o["pnode"], o["pdev"], o["roff"], o["rexp"],
               o["ap"], o["cnt"], ws, ws_b, err)
    torch.cuda.synchronize()
    assert int(err) == 0
    r = O.rbd_plan(i64(ids), E, epd, dpn)
    P = r["num_pilots"]
    assert int(o["cnt"][0]) == P
    assert np.array_equal(i64(o["ptok"][:P]), r["pilot_token"])
    assert np.array_equal(i64(o["pnode"][:P]), r["pilot_node"])
    assert np.array_equal(i64(o["roff"][:P + 1]), r["replica_offsets"])
    assert np.array_equal(i64(o["rexp"]), r["replica_expert"])
    assert np.array_equal(i64(o["ap"]), r["assign_pilot"])
    assert np.array_equal(i64(o["pdev"][:P]), r["pilot_device"])


@pytest.mark.gpu
def test_bounded_wait_gives_up_and_context_survives():
    # One warp waits, with the GEMMs' bounded mbarrier wait, on a barrier nothing arrives at:
    # after the 50 ms limit it reports PFMOE_DEV_TIMEOUT through the error word and returns.
    err = torch.zeros(1, device="cuda", dtype=torch.int32)
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    ev0.record()
    L.moe_selftest_wait_timeout(err, 50_000_000)
    ev1.record()
    torch.cuda.synchronize()
    assert int(err) == L.DEV_TIMEOUT
    assert 40.0 <= ev0.elapsed_time(ev1) < 2000.0       # it waited about the limit, then returned
    # the context is still usable: a full layer step runs clean afterwards
    cfg = get_config("small_bf16")
    layer = make_layer(cfg)
    inp = make_inputs(cfg, seed=3, device="cuda")
    assert run_step(layer, inp) == 0



def _pft_and_rbd_match_oracle(ids, w, E, k, epd, dpn):
    T = ids.shape[0]
    N = T * k
    i32 = dict(device="cuda", dtype=torch.int32)
    tpe, off, tiles = torch.empty(E, **i32), torch.empty(E + 1, **i32), torch.empty(E + 1, **i32)
    tok, eid, pos = torch.empty(N, **i32), torch.empty(N, **i32), torch.empty(T, k, **i32)
    cw = torch.empty(N, device="cuda")
    err = torch.zeros(1, **i32)
    ws_b = L.pft_build_workspace_size(T, E, k)
    ws = torch.empty(ws_b, device="cuda", dtype=torch.uint8)
    L.pft_build(ids, w, T, E, k, tpe, off, tok, eid, cw, pos, tiles, ws, ws_b, err)
    n_nodes = E // (epd * dpn)
    pmax = T * min(k, n_nodes)
    o = dict(ppn=torch.empty(n_nodes, **i32), noff=torch.empty(n_nodes + 1, **i32), ptok=torch.empty(pmax, **i32),
             pnode=torch.empty(pmax, **i32), pdev=torch.empty(pmax, **i32), roff=torch.empty(pmax + 1, **i32),
             rexp=torch.empty(N, **i32), ap=torch.empty(T, k, **i32), cnt=torch.empty(2, **i32))
    rws_b = L.rbd_plan_workspace_size(T, k, E, epd, dpn)
    rws = torch.empty(rws_b, device="cuda", dtype=torch.uint8)
    L.rbd_plan(ids, T, k, E, epd, dpn, o["ppn"], o["noff"], o["ptok"], o["pnode"], o["pdev"], o["roff"], o["rexp"],
               o["ap"], o["cnt"], rws, rws_b, err)
    torch.cuda.synchronize()
    assert int(err) == 0
    ids_h = i64(ids)
    p = O.pft_build(ids_h, w.cpu().numpy(), E)
    assert np.array_equal(i64(tpe), p["tokens_per_expert"])
    assert np.array_equal(i64(off), p["expert_offsets"])
    assert np.array_equal(i64(tiles), p["tile_offsets"])
    assert np.array_equal(i64(tok), p["token_ids"])
    assert np.array_equal(i64(eid), p["expert_ids"])
    assert np.array_equal(cw.cpu().numpy().astype(np.float64), p["combine_weights"])
    assert np.array_equal(i64(pos), p["pos"])
    r = O.rbd_plan(ids_h, E, epd, dpn)
    P = r["num_pilots"]
    assert int(o["cnt"][0]) == P and int(o["cnt"][1]) == r["num_token_device_pairs"]
    assert np.array_equal(i64(o["ppn"]), r["pilots_per_node"])
    assert np.array_equal(i64(o["noff"]), r["node_offsets"])
    assert np.array_equal(i64(o["ptok"][:P]), r["pilot_token"])
    assert np.array_equal(i64(o["pnode"][:P]), r["pilot_node"])
    assert np.array_equal(i64(o["pdev"][:P]), r["pilot_device"])
    assert np.array_equal(i64(o["roff"][:P + 1]), r["replica_offsets"])
    assert np.array_equal(i64(o["rexp"]), r["replica_expert"])
    assert np.array_equal(i64(o["ap"]), r["assign_pilot"])


@pytest.mark.gpu
@pytest.mark.parametrize("E,k,epd,dpn", [(256, 8, 8, 4), (1024, 4, 16, 8), (1024, 16, 2, 64)])
def test_pft_and_rbd_four_million_assignments_match_oracle(E, k, epd, dpn):
    # About 4.2 M assignments (2000+ sort chunks; RBD tiles past the scan's first pass).  The last map
    # has 8 nodes of 64 devices each: the per-token plan with more than 64 devices.
    from workloads.generate import make_topk_ids
    T = (1 << 22) // k + 123
    ids = make_topk_ids(T, E, k, seed=9, device="cuda")
    w = torch.rand(T, k, device="cuda")
    _pft_and_rbd_match_oracle(ids, w, E, k, epd, dpn)


@pytest.mark.gpu
@pytest.mark.parametrize("E,k,epd,dpn", [(64, 8, 2, 4), (64, 8, 1, 16), (64, 8, 1, 1), (512, 32, 1, 64)])
def test_pft_and_rbd_with_repeated_ids_match_oracle(E, k, epd, dpn):
    # Ids drawn with repetition, so a token can name one expert in several slots: the PFT keeps the
    # slots in order, and the RBD plan lists the repeats as separate replicas of one pilot, after
    # equal ids in slot order (the oracle's stable sort).  Maps: 8 nodes (per-token plan, up to 64
    # devices), 4 nodes of 16 devices, 64 nodes (the sort-based plan), 8 nodes of 64 devices.
    T = 20000 + 7
    g = torch.Generator(device="cuda").manual_seed(17)
    ids = torch.randint(0, E, (T, k), generator=g, device="cuda", dtype=torch.int32)
    ids[:, 1] = ids[:, 0]   # at least one repeat in every token
    w = torch.rand(T, k, device="cuda", generator=g)
    _pft_and_rbd_match_oracle(ids, w, E, k, epd, dpn)


@pytest.mark.gpu
@pytest.mark.parametrize("E,k,epd,dpn", [(2048, 8, 32, 8), (4096, 6, 16, 16), (4096, 8, 4, 2)])
def test_pft_and_rbd_wide_expert_ids_match_oracle(E, k, epd, dpn):
    # More than 1024 experts: the PFT scatter finds equal keys with __match_any_sync (not ballots) and
    # runs fewer warps per chunk; hundreds of chunks, so the chunk counts take the many-chunk scan.
    # Maps: 8 nodes of 8 devices (per-token plan), 16 nodes and 512 nodes (sort-based plan).
    T = 40000 + 3
    g = torch.Generator(device="cuda").manual_seed(19)
    ids = torch.randint(0, E, (T, k), generator=g, device="cuda", dtype=torch.int32)
    w = torch.rand(T, k, device="cuda", generator=g)
    _pft_and_rbd_match_oracle(ids, w, E, k, epd, dpn)


@pytest.mark.gpu
def test_rbd_many_nodes_general_path():
    # 64 nodes: more than the per-token fast plan handles, so the sort-based plan runs.
    from workloads.generate import make_topk_ids
    T, E, k, epd, dpn = 5000, 256, 8, 2, 2
    ids = make_topk_ids(T, E, k, seed=13, device="cuda")
    n_nodes = E // (epd * dpn)
    pmax = T * min(k, n_nodes)
    i32 = dict(device="cuda", dtype=torch.int32)
    o = dict(ppn=torch.empty(n_nodes, **i32), noff=torch.empty(n_nodes + 1, **i32), ptok=torch.empty(pmax, **i32),
             pnode=torch.empty(pmax, **i32), pdev=torch.empty(pmax, **i32), roff=torch.empty(pmax + 1, **i32),
             rexp=torch.empty(T * k, **i32), ap=torch.empty(T, k, **i32), cnt=torch.empty(2, **i32))
    ws_b = L.rbd_plan_workspace_size(T, k, E, epd, dpn)
    ws = torch.empty(ws_b, device="cuda", dtype=torch.uint8)
    err = torch.zeros(1, **i32)
    L.rbd_plan(ids, T, k, E, epd, dpn, o["ppn"], o["noff"], o["ptok"], o["pnode"], o["pdev"], o["roff"], o["rexp"],
               o["ap"], o["cnt"], ws, ws_b, err)
    torch.cuda.synchronize()
    assert int(err) == 0
    r = O.rbd_plan(i64(ids), E, epd, dpn)
    P = r["num_pilots"]
    assert int(o["cnt"][0]) == P and int(o["cnt"][1]) == r["num_token_device_pairs"]
    assert np.array_equal(i64(o["ppn"]), r["pilots_per_node"])
    assert np.array_equal(i64(o["noff"]), r["node_offsets"])
    assert np.array_equal(i64(o["ptok"][:P]), r["pilot_token"])
    assert np.array_equal(i64(o["pnode"][:P]), r["pilot_node"])
    assert np.array_equal(i64(o["pdev"][:P]), r["pilot_device"])
    assert np.array_equal(i64(o["roff"][:P + 1]), r["replica_offsets"])
    assert np.array_equal(i64(o["rexp"]), r["replica_expert"])
    assert np.array_equal(i64(o["ap"]), r["assign_pilot"])


@pytest.mark.gpu
@pytest.mark.parametrize("fused", [False, True])
def test_largest_routing_shape_matches_oracle(fused):
    # The routing limits: E = 1024 experts, k = 32 (RBD map of 8 nodes: the per-token plan at its
    # widest lane group), the whole layer forward and backward against the oracle.
    from tests.parity import TOL, check_index_parity, f64, rel_err
    cfg = get_config("small_bf16").with_(name="largest_routing", T=160, d=64, E=1024, h=64, k=32, rbd_epd=32,
                                         rbd_dpn=4)
    inp = make_inputs(cfg, seed=21, device="cuda")
    layer = make_layer(cfg)
    layer.fused_gather = fused
    assert run_step(layer, inp) == 0
    check_index_parity(layer, cfg, O)
    x, wg, bias, w1, w3, w2, dy = map(f64, (inp.x, inp.wg, inp.bias, inp.w1, inp.w3, inp.w2, inp.dy))
    fwd = O.layer_forward(x, wg, bias, w1, w3, w2, cfg.k, logits=layer.logits.cpu().numpy())
    assert rel_err(f64(layer.y), fwd["y"]) <= TOL[cfg.dtype]
    bwd = O.layer_backward(fwd, dy, x, wg, w1, w3, w2)
    for nm, t in (("dx", layer.dx), ("dWg", layer.dwg), ("dW1", layer.dw1), ("dW3", layer.dw3),
                  ("dW2", layer.dw2), ("dlogits", layer.dlogits)):
        assert rel_err(f64(t), bwd[nm]) <= TOL[cfg.dtype], nm
