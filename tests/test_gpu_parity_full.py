"""CUDA path vs the CPU oracle at the full layer sizes.

Indices (routing, PFT, RBD) are compared in full, bit for bit.  Values are
compared on samples the oracle computes one by one:
  * logits of sampled tokens;
  * y, dx and dlogits of sampled tokens, from a one-token oracle layer made of
    the token's k routed experts (tokens are independent in y and dx);
  * PFT.x rows (exact copies);
  * H1, H3, A, O rows and the weight gradients dW1, dW3, dW2 of sampled experts
    (the heaviest, the lightest non-empty, an empty one when any, random ones),
    from the oracle run on that expert's rows;
  * dWg through the identity dWg = x^T dlogits, with dlogits pinned above.
"""
import numpy as np
import pytest
import torch

import oracle as O
from workloads import CONFIGS, make_inputs

from tests.parity import LOGIT_TOL, TOL, check_index_parity, f64, i64, make_layer, rel_err, run_step

FULL = ["dsmoe16b_bf16", "dsv3_bf16", "dsv3_zipf_bf16", "finegrained_bf16", "tiny_fp32"]


def _token_layer(t, ids, z_gpu, x, wg, w1, w3, w2, dy, k):
    """Oracle forward + backward of one token, restricted to its k routed experts."""
    sel = np.sort(ids[t])
    xt = x[t:t + 1]
    w1s = np.stack([f64(w1[e]) for e in sel])
    w3s = np.stack([f64(w3[e]) for e in sel])
    w2s = np.stack([f64(w2[e]) for e in sel])
    fwd = O.layer_forward(xt, wg[:, sel], None, w1s, w3s, w2s, k, logits=z_gpu[t:t + 1, sel])
    bwd = O.layer_backward(fwd, dy[t:t + 1], xt, wg[:, sel], w1s, w3s, w2s)
    return sel, fwd["y"][0], bwd["dx"][0], bwd["dlogits"][0]


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

    # --- per-token y, dx, dlogits
    dy = f64(inp.dy)
    y_g, y_r, dx_g, dx_r, dz_g, dz_r = [], [], [], [], [], []
    y_gpu, dx_gpu, dl_gpu = f64(layer.y), f64(layer.dx), layer.dlogits.cpu().numpy()
    for t in toks[:6]:
        sel, yt, dxt, dzt = _token_layer(t, ids, z_gpu, x, wg, inp.w1, inp.w3, inp.w2, dy, k)
        y_g.append(y_gpu[t]); y_r.append(yt)
        dx_g.append(dx_gpu[t]); dx_r.append(dxt)
        full = np.zeros(E); full[sel] = dzt
        dz_g.append(dl_gpu[t]); dz_r.append(full)
    assert rel_err(y_g, y_r) <= tol
    assert rel_err(dx_g, dx_r) <= tol
    assert rel_err(dz_g, dz_r) <= tol

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
        for nm, t_gpu, ref in (("H1", layer.h1, H1), ("H3", layer.h3, H3), ("A", layer.a, A), ("O", layer.out, Oe)):
            err = rel_err(f64(t_gpu[r0:r1]), ref)
            assert err <= tol, (e, nm, err)
        dO = wts[r0:r1, None] * dy[tok_ids[r0:r1]]
        g = O.expert_backward(X, H1, H3, A, dO, w1e, w3e, w2e)
        for nm, got in zip(("dW1", "dW3", "dW2"), dw_g):
            err = rel_err(got, g[nm])
            assert err <= tol, (e, nm, err)

    # --- dWg = x^T dlogits (dlogits pinned per token above)
    assert rel_err(f64(layer.dwg), x.T @ dl_gpu.astype(np.float64)) <= tol
