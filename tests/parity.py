"""Helpers shared by the GPU parity tests: run the CUDA path on one layer and
compare with the CPU oracle."""
from __future__ import annotations

import numpy as np
import torch

from padding_free_moe_b200.layer import PFTMoELayer, Shape
from workloads.generate import storage_dtype

# Per-tensor bound on max|gpu - ref| / max|ref| (spec tolerance).
TOL = {"bf16": 2e-2, "f32": 1e-4}
# The logits are float32 accumulations of exactly representable products in both dtypes.
LOGIT_TOL = 1e-4


def rel_err(got, ref) -> float:
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    assert got.shape == ref.shape, (got.shape, ref.shape)
    if got.size == 0:
        return 0.0
    den = np.abs(ref).max()
    return float(np.abs(got - ref).max() / (den if den > 0 else 1.0))


def f64(t):
    if t is None:
        return None
    return t.detach().to("cpu").to(torch.float64).numpy()


def i64(t):
    return t.detach().to("cpu").to(torch.int64).numpy()


def make_layer(cfg, device="cuda") -> PFTMoELayer:
    return PFTMoELayer(Shape(cfg.T, cfg.d, cfg.E, cfg.h, cfg.k, storage_dtype(cfg), cfg.rbd_epd, cfg.rbd_dpn),
                       device)


def run_step(layer: PFTMoELayer, inp):
    layer.err.zero_()
    layer.step(inp.x, inp.wg, inp.bias, inp.w1, inp.w3, inp.w2, inp.dy)
    torch.cuda.synchronize()
    return layer.device_error()


def check_index_parity(layer: PFTMoELayer, cfg, O):
    """Routing, PFT and RBD must equal the oracle's bit for bit, given the GPU's float32 logits."""
    z = layer.logits.cpu().numpy()
    ids_ref, w_ref = O.route(z, cfg.k)
    ids = i64(layer.topk_ids)
    assert np.array_equal(ids, ids_ref), "top-k ids differ from the oracle on the same logits"
    w = layer.topk_w.cpu().numpy()
    assert np.abs(w - w_ref).max() <= 2e-6
    p = O.pft_build(ids, w, cfg.E)
    N = cfg.N
    assert np.array_equal(i64(layer.tokens_per_expert), p["tokens_per_expert"])
    assert np.array_equal(i64(layer.expert_offsets), p["expert_offsets"])
    assert np.array_equal(i64(layer.tile_offsets), p["tile_offsets"])
    if N:
        assert np.array_equal(i64(layer.token_ids[:N]), p["token_ids"])
        assert np.array_equal(i64(layer.expert_ids[:N]), p["expert_ids"])
        assert np.array_equal(layer.combine_weights[:N].cpu().numpy().astype(np.float64), p["combine_weights"])
        assert np.array_equal(i64(layer.pos), p["pos"])
    if layer.has_rbd:
        r = O.rbd_plan(ids, cfg.E, cfg.rbd_epd, cfg.rbd_dpn)
        P = r["num_pilots"]
        cnt = i64(layer.rbd_counts)
        assert cnt[0] == P and cnt[1] == r["num_token_device_pairs"]
        assert np.array_equal(i64(layer.pilots_per_node), r["pilots_per_node"])
        assert np.array_equal(i64(layer.node_offsets), r["node_offsets"])
        assert np.array_equal(i64(layer.pilot_token[:P]), r["pilot_token"])
        assert np.array_equal(i64(layer.pilot_node[:P]), r["pilot_node"])
        assert np.array_equal(i64(layer.pilot_device[:P]), r["pilot_device"])
        assert np.array_equal(i64(layer.replica_offsets[:P + 1]), r["replica_offsets"])
        assert np.array_equal(i64(layer.replica_expert[:N]), r["replica_expert"])
        assert np.array_equal(i64(layer.assign_pilot), r["assign_pilot"])
    return ids, w


class LazyExperts:
    """Stacked expert weights [E, r, c] kept on the GPU and handed to the oracle one
    expert at a time as float64 (a full-size stack would need tens of GB of host
    memory in float64).  The oracle only ever indexes experts that own rows."""

    def __init__(self, t):
        self.t = t
        self.shape = tuple(t.shape)

    def __len__(self):
        return self.shape[0]

    def __getitem__(self, e):
        return f64(self.t[int(e)])


def sampled_layer(O, S, z_gpu, x, wg, w1, w3, w2, dy, k):
    """The oracle's layer, forward and backward, on the token subset S (tokens are
    independent in y, dx and dlogits; dWg over S is complete in every column whose
    routed tokens all lie in S).  Routing uses the GPU's logits, which the tests
    compare with the oracle's separately.  The backward repeats the oracle's
    layer_backward step by step, but keeps only dX of each expert: its weight
    gradients over all E experts would not fit in host memory at full size.
    w1, w3, w2 are LazyExperts (or arrays); x, wg, dy are float64 arrays."""
    S = np.asarray(S)
    xs, dys = x[S], dy[S]
    fwd = O.layer_forward(xs, wg, None, w1, w3, w2, k, logits=z_gpu[S])
    pft = fwd["pft"]
    dO, g = O.combine_backward(dys, fwd["O"], pft["pos"], fwd["w"])
    offs = pft["expert_offsets"]
    dX = np.zeros_like(fwd["x_pft"])
    for e in range(len(offs) - 1):
        r0, r1 = int(offs[e]), int(offs[e + 1])
        if r1 > r0:
            gr = O.expert_backward(fwd["x_pft"][r0:r1], fwd["H1"][r0:r1], fwd["H3"][r0:r1], fwd["A"][r0:r1],
                                   dO[r0:r1], w1[e], w3[e], w2[e])
            dX[r0:r1] = gr["dX"]
    dz, dWg, dx_gate = O.gate_backward(xs, wg, fwd["ids"], fwd["w"], g, wg.shape[1])
    dx = O.token_grad(dX, pft["pos"]) + dx_gate
    return {"y": fwd["y"], "dx": dx, "dlogits": dz, "dWg": dWg, "ids": fwd["ids"]}
