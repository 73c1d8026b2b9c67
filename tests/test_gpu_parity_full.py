"""CUDA path vs the CPU oracle at the full layer sizes.

Indices (routing, PFT, RBD) are compared in full, bit for bit.  Values are
compared on samples the oracle computes one by one:
  * logits of sampled tokens;
  * y, dx and dlogits of 64 sampled tokens, from the oracle's layer run on a token
    subset (tokens are independent in y, dx and dlogits);
  * dWg in the columns of two sampled experts (the heaviest and a random one),
    from the oracle's layer run on every token routed to either of them: no other
    token contributes to those columns;
  * PFT.x rows (exact copies);
  * H1, H3, A, O rows and the weight gradients dW1, dW3, dW2 of sampled experts
    (the heaviest, the lightest non-empty, an empty one when any, random ones),
    from the oracle run on that expert's rows.
Expert weights reach the oracle one expert at a time (LazyExperts): the largest
layers' float64 weights would not fit in host memory at once.
"""
import numpy as np
import pytest
import torch

import oracle as O
from workloads import CONFIGS, make_inputs

from tests.parity import (LOGIT_TOL, TOL, LazyExperts, check_index_parity, f64, i64, make_layer, rel_err, run_step,
                          sampled_layer)

FULL = ["dsmoe16b_bf16", "dsv3_bf16", "dsv3_zipf_bf16", "finegrained_bf16", "tiny_fp32"]


@pytest.mark.gpu
@pytest.mark.parametrize("name", FULL)
def test_full_size_sampled_parity(name):
    cfg = CONFIGS[name]
    tol = TOL[cfg.dtype]
    T, d, E, h, k, N = cfg.T, cfg.d, cfg.E, cfg.h, cfg.k, cfg.N
    inp = make_inputs(cfg, seed=0, device="cuda")
    layer = make_layer(cfg)
    assert run_step(layer, inp) == 0, "device error word set"
    rng = np.random.default_rng(0)

    # --- indices, in full
    ids, w = check_index_parity(layer, cfg, O)
    tpe = i64(layer.tokens_per_expert)
    if cfg.zipf_c > 0:   # the skewed layer really is skewed, and nothing was dropped
        assert tpe.max() / (N / E) >= 20 and (tpe == 0).sum() >= 4
    assert tpe.sum() == N

    # --- logits of sampled tokens
    x = f64(inp.x)
    wg = f64(inp.wg)
    bias = f64(inp.bias)
    z_gpu = layer.logits.cpu().numpy()
    toks = rng.choice(T, size=min(T, 64), replace=False)
    z_ref = O.gate_logits(x[toks], wg, bias)
    assert rel_err(z_gpu[toks], z_ref) <= LOGIT_TOL
    s = -np.sort(-z_ref, axis=1)
    if k < E:
        clear = (s[:, k - 1] - s[:, k]) > 1e-4 * np.abs(z_ref).max()
        ids_ref, _ = O.route(z_ref, k)
        assert np.array_equal(ids[toks][clear], ids_ref[clear])

    # --- y, dx, dlogits of 64 sampled tokens; dWg columns of two sampled experts
    dy = f64(inp.dy)
    tpe_nz = np.where(tpe > 0)[0]
    cols = sorted({int(tpe_nz[np.argmax(tpe[tpe_nz])]), int(rng.choice(tpe_nz))})
    col_toks = np.where(np.isin(ids, cols).any(axis=1))[0]
    S = np.union1d(toks, col_toks)
    ref = sampled_layer(O, S, z_gpu, x, wg, LazyExperts(inp.w1), LazyExperts(inp.w3), LazyExperts(inp.w2), dy, k)
    assert np.array_equal(ref["ids"], ids[S])
    at = np.searchsorted(S, toks)
    assert rel_err(f64(layer.y)[toks], ref["y"][at]) <= tol
    assert rel_err(f64(layer.dx)[toks], ref["dx"][at]) <= tol
    assert rel_err(layer.dlogits.cpu().numpy()[toks], ref["dlogits"][at]) <= tol
    assert rel_err(f64(layer.dwg)[:, cols], ref["dWg"][:, cols]) <= tol

    # --- PFT.x rows: exact copies of token rows
    rows = rng.choice(N, size=min(N, 2048), replace=False)
    tok_ids = i64(layer.token_ids[:N])
    assert np.array_equal(f64(layer.x_pft[torch.as_tensor(rows, device="cuda")]), x[tok_ids[rows]])

    # --- sampled experts: forward rows and weight gradients
    offs = i64(layer.expert_offsets)
    nz = np.where(tpe > 0)[0]
    experts = {int(nz[np.argmax(tpe[nz])]), int(nz[np.argmin(tpe[nz])])}
    if (tpe == 0).any():
        experts.add(int(np.where(tpe == 0)[0][0]))
    experts |= set(int(e) for e in rng.choice(E, size=2, replace=False))
    wts = layer.combine_weights[:N].cpu().numpy().astype(np.float64)
    for e in sorted(experts):
        r0, r1 = offs[e], offs[e + 1]
        dw_g = [f64(layer.dw1[e]), f64(layer.dw3[e]), f64(layer.dw2[e])]
        if r1 == r0:
            assert all(not g.any() for g in dw_g), f"empty expert {e} has non-zero weight gradients"
            continue
        X = x[tok_ids[r0:r1]]
        w1e, w3e, w2e = f64(inp.w1[e]), f64(inp.w3[e]), f64(inp.w2[e])
        H1, H3, A, Oe = O.expert_forward(X, w1e, w3e, w2e)
        for nm, t_gpu, want in (("H1", layer.h1, H1), ("H3", layer.h3, H3), ("A", layer.a, A), ("O", layer.out, Oe)):
            err = rel_err(f64(t_gpu[r0:r1]), want)
            assert err <= tol, (e, nm, err)
        dO = wts[r0:r1, None] * dy[tok_ids[r0:r1]]
        g = O.expert_backward(X, H1, H3, A, dO, w1e, w3e, w2e)
        for nm, got in zip(("dW1", "dW3", "dW2"), dw_g):
            err = rel_err(got, g[nm])
            assert err <= tol, (e, nm, err)

