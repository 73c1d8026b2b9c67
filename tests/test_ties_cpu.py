"""The tie layers of the GPU tie test really exercise the tie rule (CPU only).

For every case of tests/test_gpu_ties.py: the quantised logits are exact in
float32 (so the GPU sees the same values as the oracle), some tokens have equal
logits at the k-th / (k+1)-th boundary, and routing with the opposite tie rule
(equal logits to the HIGHER index) picks a different expert set or order on some
tokens.  A kernel that broke ties the wrong way, or compared with >= instead of
>, would therefore fail the GPU comparison.
"""
import numpy as np
import pytest
import torch

import oracle as O

from tests.test_gpu_ties import CASES, case_inputs


def _route_high_index_first(z, k):
    col = np.broadcast_to(np.arange(z.shape[1]), z.shape)
    order = np.lexsort((-col, -z), axis=-1)
    return order[:, :k]


def _f64(t):
    return None if t is None else t.to(torch.float64).numpy()


@pytest.mark.parametrize("name", sorted(CASES))
def test_tie_inputs_decide_selection(name):
    cfg, inp = case_inputs(name, "cpu")
    x, wg, bias = _f64(inp.x), _f64(inp.wg), _f64(inp.bias)
    z = O.gate_logits(x, wg, bias)
    # exact in float32: summing the float32-rounded products in float32 changes nothing
    z32 = (x.astype(np.float32) @ wg.astype(np.float32))
    if bias is not None:
        z32 = z32 + bias.astype(np.float32)
    assert np.array_equal(z32.astype(np.float64), z)
    ids, _ = O.route(z, cfg.k)
    s = -np.sort(-z, axis=1)
    boundary_ties = (s[:, cfg.k - 1] == s[:, cfg.k]).sum() if cfg.k < cfg.E else 0
    assert boundary_ties > 0, "no token ties at the selection boundary"
    other = _route_high_index_first(z, cfg.k)
    sel_diff = (np.sort(ids, axis=1) != np.sort(other, axis=1)).any(axis=1).sum()
    assert sel_diff > 0, "the opposite tie rule selects the same experts everywhere"
    assert (ids != other).any(axis=1).sum() >= sel_diff
