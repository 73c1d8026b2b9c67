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
