"""Pins of the CPU oracle against things other than itself.

Every check here derives its expectation independently of the oracle's code:
hand-worked examples, closed forms, invariants, library routines (scipy
softmax/expit), brute force on tiny inputs and float64 finite differences.
"""
import itertools
import json
import math
import os

import numpy as np
import pytest
from scipy.special import expit, softmax

import oracle as O
from workloads import get_config, make_inputs
from workloads.generate import make_topk_ids


def rng(seed=0):
    return np.random.default_rng(seed)


# ------------------------------------------------------------------ gate / route
def test_route_hand_ties():
    # Hand cases: descending logit, equal logits go to the lower index.
    cases = [
        ([1.0, 3.0, 3.0, 2.0], 2, [1, 2], [0.5, 0.5]),
        ([0.0, 0.0, 0.0, 0.0], 3, [0, 1, 2], [1 / 3] * 3),
        ([2.0, 1.0], 1, [0], [1.0]),
        # logits ln3, ln2 -> weights proportional to 3 and 2
        ([0.0, math.log(3.0), math.log(2.0)], 2, [1, 2], [0.6, 0.4]),
        # two tied maxima, then a tie at the boundary: 2.0 at index 2 beats 2.0 at index 4
        ([-1.0, 5.0, 2.0, 5.0, 2.0], 3, [1, 3, 2],
         [1 / (2 + math.exp(-3)), 1 / (2 + math.exp(-3)), math.exp(-3) / (2 + math.exp(-3))]),
    ]
    for z, k, ids, w in cases:
        got_ids, got_w = O.route(np.array([z]), k)
        assert got_ids[0].tolist() == ids
        np.testing.assert_allclose(got_w[0], w, rtol=1e-15, atol=1e-15)


def test_route_selection_property_bruteforce():
    # The picked set S must dominate every unpicked expert under (value desc, index asc),
    # and S must be listed in that order.  Checked pair by pair on many tiny random cases,
    # with coarse values so that ties are frequent.
    r = rng(1)
    for _ in range(400):
        E = int(r.integers(1, 9)); k = int(r.integers(1, E + 1))
        z = r.integers(-3, 4, size=(1, E)).astype(np.float64)
        ids, _ = O.route(z, k)
        S = ids[0].tolist()
        assert len(set(S)) == k
        better = lambda i, j: z[0, i] > z[0, j] or (z[0, i] == z[0, j] and i < j)
        for i in S:
            for j in range(E):
                if j not in S:
                    assert better(i, j)
        for a, b in zip(S, S[1:]):
            assert better(a, b)


def test_route_weights_are_renormalised_softmax():
    r = rng(2)
    z = r.normal(size=(50, 12)) * 3
    for k in (1, 3, 12):
        ids, w = O.route(z, k)
        full = softmax(z, axis=1)                         # library softmax over all E
        picked = np.take_along_axis(full, ids.astype(np.int64), axis=1)
        np.testing.assert_allclose(w, picked / picked.sum(1, keepdims=True), rtol=1e-12)
        np.testing.assert_allclose(w.sum(1), 1.0, rtol=0, atol=1e-14)
    ids, w = O.route(z, 12)                               # k = E: the plain softmax, reordered
    np.testing.assert_allclose(np.take_along_axis(softmax(z, 1), ids.astype(np.int64), 1), w, rtol=1e-12)


def test_route_shift_invariance():
    r = rng(3)
    z = r.normal(size=(40, 9))
    shift = r.normal(size=(40, 1)) * 1000   # large enough that an unshifted exp overflows
    ids1, w1 = O.route(z, 4)
    ids2, w2 = O.route(z + shift, 4)
    # adding a per-token constant cannot change which experts win (barring rounding ties)
    assert (ids1 == ids2).all()
    np.testing.assert_allclose(w1, w2, rtol=1e-10)


def test_gate_logits_bias():
    x = np.array([[1.0, 2.0]]); wg = np.array([[1.0, 0.0, -1.0], [0.5, 1.0, 0.0]])
    np.testing.assert_array_equal(O.gate_logits(x, wg), [[2.0, 2.0, -1.0]])
    np.testing.assert_array_equal(O.gate_logits(x, wg, np.array([0.0, -0.5, 10.0])), [[2.0, 1.5, 9.0]])


def test_finegrained_combinations_golden(golden_dir):
    # The number of distinct expert sets a token can be routed to is C(E, k) ([A] §1).
    with open(os.path.join(golden_dir, "finegrained_combinations.json")) as f:
        g = json.load(f)
    c0, c1 = g["cases"]
    assert math.comb(c0["E"], c0["k"]) == c0["combinations"]
    assert abs(math.comb(c1["E"], c1["k"]) / c1["combinations_approx"] - 1) < c1["rel_tol"]
    # and the oracle's router reaches exactly the C(8, 2) = 28 sets
    z = rng(4).normal(size=(5000, c0["E"]))
    ids, _ = O.route(z, c0["k"])
    assert len({tuple(sorted(r)) for r in ids.tolist()}) == c0["combinations"]


# ------------------------------------------------------------------------- PFT
def test_pft_hand_example():
    # ids [[2,0],[2,3],[0,2]]: assignments a=t*k+j are (t0,e2) (t0,e0) (t1,e2) (t1,e3) (t2,e0) (t2,e2).
    # Stable by expert: e0 <- a1,a4; e2 <- a0,a2,a5; e3 <- a3.
    ids = np.array([[2, 0], [2, 3], [0, 2]])
    w = np.array([[.6, .4], [.7, .3], [.9, .1]])
    p = O.pft_build(ids, w, 4)
    assert p["tokens_per_expert"].tolist() == [2, 0, 3, 1]
    assert p["expert_offsets"].tolist() == [0, 2, 2, 5, 6]
    assert p["token_ids"].tolist() == [0, 2, 0, 1, 2, 1]
    assert p["expert_ids"].tolist() == [0, 0, 2, 2, 2, 3]
    np.testing.assert_array_equal(p["combine_weights"], [.4, .9, .6, .7, .1, .3])
    assert p["pos"].tolist() == [[2, 0], [3, 5], [1, 4]]
    assert p["tile_offsets"].tolist() == [0, 1, 1, 2, 3]


def _bucket_sort_reference(ids, E):
    # A different algorithm from the oracle's stable argsort: append to per-expert buckets
    # while walking the assignments in token-major order.
    buckets = [[] for _ in range(E)]
    T, k = ids.shape
    for t in range(T):
        for j in range(k):
            buckets[ids[t, j]].append((t, j))
    order = [a for b in buckets for a in b]
    return [len(b) for b in buckets], order


@pytest.mark.parametrize("seed", range(6))
def test_pft_against_buckets_and_invariants(seed):
    r = rng(10 + seed)
    T = int(r.integers(1, 60)); E = int(r.integers(1, 12)); k = int(r.integers(1, E + 1))
    ids = np.stack([r.permutation(E)[:k] for _ in range(T)])
    w = r.random((T, k))
    p = O.pft_build(ids, w, E)
    counts, order = _bucket_sort_reference(ids, E)
    assert p["tokens_per_expert"].tolist() == counts
    assert p["token_ids"].tolist() == [t for t, _ in order]
    assert p["expert_ids"].tolist() == [ids[t, j] for t, j in order]
    np.testing.assert_array_equal(p["combine_weights"], [w[t, j] for t, j in order])
    # invariants
    N = T * k
    assert p["tokens_per_expert"].sum() == N
    assert p["expert_offsets"][0] == 0 and p["expert_offsets"][-1] == N
    assert np.all(np.diff(p["expert_ids"]) >= 0)
    assert np.bincount(p["token_ids"], minlength=T).tolist() == [k] * T
    for e in range(E):
        seg = p["token_ids"][p["expert_offsets"][e]:p["expert_offsets"][e + 1]]
        assert np.all(np.diff(seg) > 0)          # ascending, each (t, e) at most once
    for t in range(T):
        for j in range(k):
            q = p["pos"][t, j]
            assert p["token_ids"][q] == t and p["expert_ids"][q] == ids[t, j]
    assert sorted(p["pos"].ravel().tolist()) == list(range(N))
    # tile list: expert e owns ceil(n_e / 128) tiles, counted row by row here
    tiles = [sum(1 for r0 in range(0, c, 128)) for c in counts]
    assert p["tile_offsets"].tolist() == [0] + list(np.cumsum(tiles))


@pytest.mark.parametrize("seed", range(4))
def test_pft_with_repeated_ids_keeps_slot_order(seed):
    # A token may name one expert in several slots (the entry points accept any ids in [0, E)):
    # the stable sort then keeps those slots in slot order, next to each other.
    r = rng(40 + seed)
    T = int(r.integers(1, 40)); E = int(r.integers(1, 6)); k = int(r.integers(2, 9))
    ids = r.integers(0, E, size=(T, k))
    ids[:, 1] = ids[:, 0]
    w = r.random((T, k))
    p = O.pft_build(ids, w, E)
    counts, order = _bucket_sort_reference(ids, E)
    assert p["tokens_per_expert"].tolist() == counts
    assert p["token_ids"].tolist() == [t for t, _ in order]
    np.testing.assert_array_equal(p["combine_weights"], [w[t, j] for t, j in order])
    for t in range(T):
        for j in range(k):
            q = p["pos"][t, j]
            assert p["token_ids"][q] == t and p["expert_ids"][q] == ids[t, j]
        for j in range(1, k):   # equal ids of one token: rows in slot order
            for i in range(j):
                if ids[t, i] == ids[t, j]:
                    assert p["pos"][t, i] < p["pos"][t, j]


def test_pft_rejects_bad_ids():
    with pytest.raises(ValueError):
        O.pft_build(np.array([[0, 5]]), np.ones((1, 2)), 4)


# ------------------------------------------------------------ dispatch / combine
def test_identity_experts_return_x():
    # With O := X_pft (identity experts), combine gives x * sum_j w = x.
    r = rng(20)
    T, d, E, k = 37, 8, 6, 3
    x = r.normal(size=(T, d))
    ids, w = O.route(r.normal(size=(T, E)), k)
    p = O.pft_build(ids, w, E)
    xp = O.dispatch(x, p["token_ids"])
    np.testing.assert_allclose(O.combine(xp, p["pos"], w), x, rtol=1e-13, atol=1e-13)
    # and the dispatched rows are exact copies
    np.testing.assert_array_equal(xp, x[p["token_ids"]])


def test_one_hot_weights_pick_rows():
    r = rng(21)
    T, d, E, k = 10, 5, 5, 2
    ids = np.stack([r.permutation(E)[:k] for _ in range(T)])
    w = np.zeros((T, k)); w[:, 1] = 1.0
    p = O.pft_build(ids, w, E)
    Ob = r.normal(size=(T * k, d))
    y = O.combine(Ob, p["pos"], w)
    np.testing.assert_array_equal(y, Ob[p["pos"][:, 1]])


# ---------------------------------------------------------------------- experts
def test_silu_matches_library():
    u = np.linspace(-30, 30, 1001)
    np.testing.assert_allclose(O.silu(u), u * expit(u), rtol=1e-14, atol=1e-300)


def test_hand_two_expert_layer():
    # d = h = 1, E = k = 2, x = 2, Wg = [0, ln3 / 2]  ->  z = [0, ln3]: expert 1 first, w = [3/4, 1/4].
    # Expert 0: W1=1, W3=3, W2=0.5 -> H1=2, H3=6, O0 = SiLU(2)*6*0.5.
    # Expert 1: W1=-1, W3=1, W2=2  -> H1=-2, H3=2, O1 = SiLU(-2)*2*2.
    sig = lambda u: 1 / (1 + math.exp(-u))
    silu = lambda u: u * sig(u)
    O0 = silu(2) * 6 * 0.5
    O1 = silu(-2) * 2 * 2
    y_exp = 0.75 * O1 + 0.25 * O0
    x = np.array([[2.0]]); wg = np.array([[0.0, math.log(3) / 2]])
    w1 = np.array([[[1.0]], [[-1.0]]]); w3 = np.array([[[3.0]], [[1.0]]]); w2 = np.array([[[0.5]], [[2.0]]])
    f = O.layer_forward(x, wg, None, w1, w3, w2, 2)
    assert f["ids"].tolist() == [[1, 0]]
    np.testing.assert_allclose(f["w"], [[0.75, 0.25]], rtol=1e-15)
    np.testing.assert_allclose(f["y"], [[y_exp]], rtol=1e-14)
    # backward with dY = 1, by hand: g = (O1, O0); dz_e = w_e (g_e - y);
    # expert e with slot weight we: dA = we*W2, dH1 = dA*H3*s(1+H1(1-s)), dH3 = dA*SiLU(H1)
    b = O.layer_backward(f, np.array([[1.0]]), x, wg, w1, w3, w2)
    dz1 = 0.75 * (O1 - y_exp); dz0 = 0.25 * (O0 - y_exp)
    np.testing.assert_allclose(b["dlogits"], [[dz0, dz1]], rtol=1e-13)
    np.testing.assert_allclose(b["dWg"], [[2 * dz0, 2 * dz1]], rtol=1e-13)

    def exp_grads(H1, H3, W1, W3, W2, we):
        dA = we * W2
        s = sig(H1)
        dH1 = dA * H3 * s * (1 + H1 * (1 - s)); dH3 = dA * silu(H1)
        return 2 * dH1, 2 * dH3, silu(H1) * H3 * we, dH1 * W1 + dH3 * W3
    g0 = exp_grads(2.0, 6.0, 1.0, 3.0, 0.5, 0.25)
    g1 = exp_grads(-2.0, 2.0, -1.0, 1.0, 2.0, 0.75)
    np.testing.assert_allclose(b["dW1"].ravel(), [g0[0], g1[0]], rtol=1e-13)
    np.testing.assert_allclose(b["dW3"].ravel(), [g0[1], g1[1]], rtol=1e-13)
    np.testing.assert_allclose(b["dW2"].ravel(), [g0[2], g1[2]], rtol=1e-13)
    np.testing.assert_allclose(b["dx"], [[g0[3] + g1[3] + dz1 * math.log(3) / 2]], rtol=1e-13)


def _dense_masked_layer(x, wg, bias, w1, w3, w2, k):
    """All-experts dense computation: y_t = sum_e [e in S_t] w_te FFN_e(x_t).

    No sorting, no gather, no PFT: every expert runs on every token and a mask
    keeps the routed ones.  The selection mask is derived independently here
    (per-token sort with Python's ``sorted`` on (-z, index)).
    """
    z = x @ wg + (0 if bias is None else bias[None, :])
    T, E = z.shape
    mask = np.zeros((T, E))
    for t in range(T):
        S = sorted(range(E), key=lambda i: (-z[t, i], i))[:k]
        ez = np.exp(z[t, S] - z[t, S].max())
        mask[t, S] = ez / ez.sum()
    H1 = np.einsum("td,edh->teh", x, w1)
    H3 = np.einsum("td,edh->teh", x, w3)
    A = H1 * expit(H1) * H3
    Oe = np.einsum("teh,ehd->ted", A, w2)
    return np.einsum("te,ted->td", mask, Oe)


@pytest.mark.parametrize("name", ["small_bf16", "small_ragged_bf16", "small_kE_bf16", "small_f32", "one_token_bf16"])
def test_ffn_against_dense_masked(name):
    cfg = get_config(name)
    inp = make_inputs(cfg, seed=5)
    f64 = lambda t: None if t is None else t.double().numpy()
    x, wg, bias, w1, w3, w2 = map(f64, (inp.x, inp.wg, inp.bias, inp.w1, inp.w3, inp.w2))
    f = O.layer_forward(x, wg, bias, w1, w3, w2, cfg.k)
    dense = _dense_masked_layer(x, wg, bias, w1, w3, w2, cfg.k)
    np.testing.assert_allclose(f["y"], dense, rtol=1e-10, atol=1e-12)


def test_ffn_homogeneity():
    # y is linear in W2 and in W3 (SwiGLU: O = (SiLU(XW1) * XW3) W2)
    r = rng(30)
    T, d, E, h, k = 20, 6, 5, 4, 2
    x = r.normal(size=(T, d)); wg = r.normal(size=(d, E))
    w1 = r.normal(size=(E, d, h)); w3 = r.normal(size=(E, d, h)); w2 = r.normal(size=(E, h, d))
    y = O.layer_forward(x, wg, None, w1, w3, w2, k)["y"]
    np.testing.assert_allclose(O.layer_forward(x, wg, None, w1, w3, 2.5 * w2, k)["y"], 2.5 * y, rtol=1e-12)
    np.testing.assert_allclose(O.layer_forward(x, wg, None, w1, -3 * w3, w2, k)["y"], -3 * y, rtol=1e-12)
    np.testing.assert_array_equal(O.layer_forward(x, wg, None, w1, 0 * w3, w2, k)["y"], 0 * y)


# --------------------------------------------------------------------- backward
def _fd_setup(seed, T=7, d=5, E=5, h=3, k=2, bias=True):
    r = rng(seed)
    p = dict(x=r.normal(size=(T, d)), wg=r.normal(size=(d, E)) * 0.7,
             w1=r.normal(size=(E, d, h)) / math.sqrt(d), w3=r.normal(size=(E, d, h)) / math.sqrt(d),
             w2=r.normal(size=(E, h, d)) / math.sqrt(h))
    b = r.normal(size=E) if bias else None
    dy = r.normal(size=(T, d))
    return p, b, dy, k


def _loss(p, b, dy, k):
    f = O.layer_forward(p["x"], p["wg"], b, p["w1"], p["w3"], p["w2"], k)
    return float((f["y"] * dy).sum()), f


def _margin_ok(z, k, eps=1e-3):
    s = -np.sort(-z, axis=1)
    return k >= z.shape[1] or np.all(s[:, k - 1] - s[:, k] > eps)


@pytest.mark.parametrize("seed", [0, 1, 2, 3])
def test_backward_finite_differences(seed):
    p, b, dy, k = _fd_setup(40 + seed)
    L0, f = _loss(p, b, dy, k)
    assert _margin_ok(f["logits"], k), "pick a seed whose selection is not near a tie"
    g = O.layer_backward(f, dy, p["x"], p["wg"], p["w1"], p["w3"], p["w2"])
    grads = {"x": g["dx"], "wg": g["dWg"], "w1": g["dW1"], "w3": g["dW3"], "w2": g["dW2"]}
    r = rng(99 + seed)
    eps = 1e-6
    for name, G in grads.items():
        v = r.normal(size=p[name].shape)
        pp = dict(p); pm = dict(p)
        pp[name] = p[name] + eps * v
        pm[name] = p[name] - eps * v
        fd = (_loss(pp, b, dy, k)[0] - _loss(pm, b, dy, k)[0]) / (2 * eps)
        an = float((G * v).sum())
        assert abs(fd - an) <= 1e-6 * max(1.0, abs(an)), (name, fd, an)


def test_gate_dz_finite_differences():
    # Perturb the logits directly: L(z) = sum_t dY_t . y_t with y built from the routed softmax.
    r = rng(50)
    T, E, k, d = 6, 7, 3, 4
    z = r.normal(size=(T, E)) * 2
    assert _margin_ok(z, k)
    Ob = r.normal(size=(T * k, d))
    dy = r.normal(size=(T, d))

    def L(zz):
        ids, w = O.route(zz, k)
        p = O.pft_build(ids, w, E)
        # experts fixed: per-assignment outputs Ob in (t, j) order, placed at pos
        Obuf = np.zeros_like(Ob)
        Obuf[p["pos"].ravel()] = Ob
        return float((O.combine(Obuf, p["pos"], w) * dy).sum()), ids, w, p, Obuf

    _, ids, w, p, Obuf = L(z)
    _, gcomb = O.combine_backward(dy, Obuf, p["pos"], w)
    dz, _, _ = O.gate_backward(np.zeros((T, 1)), np.zeros((1, E)), ids, w, gcomb, E)
    eps = 1e-6
    for t in range(T):
        for e in range(E):
            zp = z.copy(); zp[t, e] += eps
            zm = z.copy(); zm[t, e] -= eps
            fd = (L(zp)[0] - L(zm)[0]) / (2 * eps)
            assert abs(fd - dz[t, e]) < 1e-7, (t, e, fd, dz[t, e])
    # rows of dz sum to zero (softmax Jacobian) and are zero off the selection
    np.testing.assert_allclose(dz.sum(1), 0, atol=1e-13)
    mask = np.zeros((T, E), bool)
    np.put_along_axis(mask, ids.astype(np.int64), True, 1)
    assert np.all(dz[~mask] == 0)


def test_empty_experts_get_zero_grads():
    r = rng(60)
    T, d, E, h, k = 9, 4, 6, 3, 2
    x = r.normal(size=(T, d)); wg = np.zeros((d, E)); b = np.array([5.0, 4.0, 0, 0, 0, 0])
    w1 = r.normal(size=(E, d, h)); w3 = r.normal(size=(E, d, h)); w2 = r.normal(size=(E, h, d))
    f = O.layer_forward(x, wg, b, w1, w3, w2, k)     # every token picks experts 0 and 1
    assert f["pft"]["tokens_per_expert"].tolist() == [T, T, 0, 0, 0, 0]
    g = O.layer_backward(f, r.normal(size=(T, d)), x, wg, w1, w3, w2)
    for n in ("dW1", "dW3", "dW2"):
        assert np.all(g[n][2:] == 0) and np.any(g[n][:2] != 0)


# -------------------------------------------------------------------------- RBD
def test_rbd_hand_example():
    # E=8, 2 experts/device, 2 devices/node -> 4 experts/node, 2 nodes.
    # t0 -> experts 1,5,2 (nodes 0,1,0); t1 -> 0,3,2 (node 0); t2 -> 7,4,6 (node 1).
    ids = np.array([[1, 5, 2], [0, 3, 2], [7, 4, 6]])
    p = O.rbd_plan(ids, 8, 2, 2)
    assert p["num_pilots"] == 4
    assert p["pilot_node"].tolist() == [0, 0, 1, 1]
    assert p["pilot_token"].tolist() == [0, 1, 0, 2]
    assert p["pilots_per_node"].tolist() == [2, 2] and p["node_offsets"].tolist() == [0, 2, 4]
    assert p["replica_offsets"].tolist() == [0, 2, 5, 6, 9]
    assert p["replica_expert"].tolist() == [1, 2, 0, 2, 3, 5, 4, 6, 7]
    assert p["pilot_device"].tolist() == [0, 0, 2, 2]
    assert p["assign_pilot"].tolist() == [[0, 2, 0], [1, 1, 1], [3, 3, 3]]
    assert p["num_token_device_pairs"] == 7


def _rbd_bruteforce(ids, E, epd, dpn):
    epn = epd * dpn
    n_nodes = E // epn
    T, k = ids.shape
    pilots = []
    for node in range(n_nodes):
        for t in range(T):
            reps = sorted(e for e in ids[t] if e // epn == node)
            if reps:
                pilots.append((t, node, reps))
    assign = np.zeros((T, k), dtype=np.int64)
    for p, (t, node, reps) in enumerate(pilots):
        for j in range(k):
            if ids[t, j] in reps:
                assign[t, j] = p
    pairs = {(t, e // epd) for t in range(T) for e in ids[t]}
    return pilots, assign, len(pairs)


def test_rbd_bruteforce_tiny():
    r = rng(70)
    n_cases = 0
    for E in (1, 2, 4, 6, 8, 12, 16):
        for epd in (1, 2, 4):
            for dpn in (1, 2, 3):
                if E % (epd * dpn):
                    continue
                for k in range(1, E + 1):
                    T = int(r.integers(1, 9))
                    ids = np.stack([r.permutation(E)[:k] for _ in range(T)])
                    got = O.rbd_plan(ids, E, epd, dpn)
                    pilots, assign, npairs = _rbd_bruteforce(ids, E, epd, dpn)
                    assert got["num_pilots"] == len(pilots)
                    assert got["pilot_token"].tolist() == [p[0] for p in pilots]
                    assert got["pilot_node"].tolist() == [p[1] for p in pilots]
                    assert got["replica_expert"].tolist() == [e for p in pilots for e in p[2]]
                    assert got["replica_offsets"].tolist() == [0] + list(np.cumsum([len(p[2]) for p in pilots]))
                    assert got["pilot_device"].tolist() == [p[2][0] // epd for p in pilots]
                    assert got["assign_pilot"].tolist() == assign.tolist()
                    assert got["num_token_device_pairs"] == npairs
                    n_nodes = E // (epd * dpn)
                    cnt = [sum(1 for p in pilots if p[1] == n) for n in range(n_nodes)]
                    assert got["pilots_per_node"].tolist() == cnt
                    n_cases += 1
    assert n_cases > 100


def test_rbd_bruteforce_repeated_ids():
    # Ids drawn with repetition: one pilot per (token, node) still, the repeats listed as separate
    # replicas of it, every repeated slot assigned to that pilot, one (token, device) pair per device.
    r = rng(71)
    n_cases = 0
    for E in (2, 4, 8, 12):
        for epd in (1, 2):
            for dpn in (1, 2):
                if E % (epd * dpn):
                    continue
                for k in (2, 3, 5, 8):
                    T = int(r.integers(1, 9))
                    ids = r.integers(0, E, size=(T, k))
                    got = O.rbd_plan(ids, E, epd, dpn)
                    pilots, assign, npairs = _rbd_bruteforce(ids, E, epd, dpn)
                    assert got["num_pilots"] == len(pilots)
                    assert got["pilot_token"].tolist() == [p[0] for p in pilots]
                    assert got["pilot_node"].tolist() == [p[1] for p in pilots]
                    assert got["replica_expert"].tolist() == [e for p in pilots for e in p[2]]
                    assert got["replica_offsets"].tolist() == [0] + list(np.cumsum([len(p[2]) for p in pilots]))
                    assert got["pilot_device"].tolist() == [p[2][0] // epd for p in pilots]
                    assert got["assign_pilot"].tolist() == assign.tolist()
                    assert got["num_token_device_pairs"] == npairs
                    n_cases += 1
    assert n_cases > 40


@pytest.mark.parametrize("E,k,epd,dpn,expect", [
    (256, 8, 8, 4, 5.295),      # DeepSeek-V3-like map: 8 nodes of 32 experts
    (512, 16, 16, 8, 3.963),    # fine-grained map: 4 nodes of 128 experts
])
def test_rbd_expected_unique_nodes(E, k, epd, dpn, expect):
    # For uniformly random k-subsets, E[#distinct nodes] = n_nodes * (1 - C(E - epn, k) / C(E, k)).
    epn = epd * dpn
    n_nodes = E // epn
    closed = n_nodes * (1 - math.comb(E - epn, k) / math.comb(E, k))
    assert abs(closed - expect) < 1e-3
    T = 8192
    ids = make_topk_ids(T, E, k, seed=3).numpy()
    p = O.rbd_plan(ids, E, epd, dpn)
    mean = p["num_pilots"] / T
    per_tok = np.bincount(p["pilot_token"], minlength=T)
    se = per_tok.std() / math.sqrt(T)
    assert abs(mean - closed) < 5 * se + 1e-9, (mean, closed, se)


def test_rbd_rejects_bad_map():
    with pytest.raises(ValueError):
        O.rbd_plan(np.array([[0, 1]]), 6, 2, 2)
