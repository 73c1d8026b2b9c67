"""Float64 CPU oracle of the padding-free (PFT) MoE layer, forward and backward.

TEST INFRASTRUCTURE ONLY.  Nothing on the product path imports this module; only
``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s ``cpu_baseline`` leg do.

Sources (cited by page title and section):

* [A] X-MoE article, adg.csdn.net: §2.1.1 "PFT数据结构创新" (the PFT fields
  token_ids / expert_ids / tokens_per_expert / combine_weights / x, no capacity
  padding, no token dropping), §2.1.2 "跨平台核函数优化" (gather of PFT rows by
  token id; per-expert GEMM over the unpadded, expert-sorted rows),
  §2.2.1 "分层冗余消除算法" (RBD: expert->node map by integer division,
  per-token node dedup, pilot set {(token, node)}).
* [B] "5.4 MoE模型在分布式训练中的应用" (aiknowledge.cn), section 训练流程
  (gate scores -> dispatch -> local experts -> combine; backward along the
  reverse path) and 参数分布的不均匀性 (expert FFN parameters).
* [C] Reading notes "【论文】略读笔记90-前沿-可扩展 MoE 训练" (freshwlnd blog),
  sections 需求/创新 (fine-grained experts with large top-k; padding-free training).

Readings where the pages are silent:

* Gate: plain linear logits z = x Wg (+ an optional per-expert bias), no noise,
  no temperature.  Selection ranks the logits: descending value, equal values
  to the lower expert index.  Weights are the softmax over the *selected*
  logits (equivalently the full softmax renormalised over the k picks).
* Expert FFN: SwiGLU without biases, A = SiLU(X W1) * (X W3), O = A W2,
  SiLU(u) = u * sigmoid(u).
* PFT order: rows sorted by expert id ascending; inside an expert, the
  (token, slot) assignments keep their token-major order (a stable sort).
* Combine: y_t = sum_j w_tj O_pos(t,j), summed over j in slot order.
* RBD node of expert e: e // (experts_per_device * devices_per_node).  A pilot
  lands on the device of its lowest-id replica.

Everything is computed in float64 from inputs that are already rounded to their
storage type; no intermediate rounding is modelled.
"""
from __future__ import annotations

import numpy as np

__all__ = [
    "GEMM_TILE_ROWS", "gate_logits", "route", "pft_build", "gemm_tile_offsets", "dispatch",
    "silu", "expert_forward", "expert_ffn", "combine", "combine_backward", "expert_backward",
    "expert_ffn_backward", "token_grad", "gate_backward", "layer_forward", "layer_backward",
    "rbd_plan",
]

# Rows per grouped-GEMM M tile; an expert with n rows owns ceil(n / 128) tiles.
GEMM_TILE_ROWS = 128


def _f64(a):
    return np.asarray(a, dtype=np.float64)


# --------------------------------------------------------------------------- gate
def gate_logits(x, wg, bias=None):
    """Gate scores z = x @ Wg (+ bias per expert).  [B] 训练流程 step a (计算门控分数)."""
    z = _f64(x) @ _f64(wg)
    if bias is not None:
        z = z + _f64(bias)[None, :]
    return z


def route(z, k):
    """Top-k selection and renormalised weights from logits z [T, E].

    Ids per token are in descending logit order, equal logits ordered by the
    lower expert index.  The weights are softmax over the k selected logits.
    Large top-k routing: [C] 需求; combine weights: [A] §2.1.1.
    The logits are taken as given (any float type is widened exactly to float64,
    so comparisons are those of the given values).
    """
    z = _f64(z)
    T, E = z.shape
    if not (1 <= k <= E):
        raise ValueError("need 1 <= k <= E")
    col = np.broadcast_to(np.arange(E), z.shape)
    # lexsort: last key is primary -> sort by -z ascending (z descending), then index ascending
    order = np.lexsort((col, -z), axis=-1)
    ids = order[:, :k]
    zs = np.take_along_axis(z, ids, axis=1)
    ex = np.exp(zs - zs[:, :1])
    w = ex / ex.sum(axis=1, keepdims=True)
    return ids.astype(np.int32), w


# ---------------------------------------------------------------------------- PFT
def pft_build(ids, w, E):
    """The padding-free token buffer's index fields, [A] §2.1.1.

    The assignment list a = t*k + j (token-major) is sorted stably by expert id,
    so experts come in ascending order ([A] §2.1.2 iterates experts in sorted
    order) and inside an expert tokens keep ascending order (the boolean-mask
    slice x[mask] of [A] §2.1.2 preserves order).  No capacity, no padding,
    no dropping: every assignment appears exactly once.
    Returns a dict of int/float64 arrays; ``pos[t, j]`` is the buffer row that
    holds assignment (t, j) (the inverse of the sort).
    """
    ids = np.asarray(ids)
    T, k = ids.shape
    flat = ids.reshape(-1).astype(np.int64)
    if flat.size and (flat.min() < 0 or flat.max() >= E):
        raise ValueError("expert id out of range")
    order = np.argsort(flat, kind="stable")
    tokens_per_expert = np.bincount(flat, minlength=E).astype(np.int64)
    offsets = np.zeros(E + 1, dtype=np.int64)
    offsets[1:] = np.cumsum(tokens_per_expert)
    pos = np.empty(flat.size, dtype=np.int64)
    pos[order] = np.arange(flat.size)
    return {
        "tokens_per_expert": tokens_per_expert,
        "expert_offsets": offsets,
        "token_ids": order // k,
        "expert_ids": flat[order],
        "combine_weights": _f64(w).reshape(-1)[order],
        "pos": pos.reshape(T, k),
        "tile_offsets": gemm_tile_offsets(tokens_per_expert),
    }


def gemm_tile_offsets(tokens_per_expert, tile_rows=GEMM_TILE_ROWS):
    """Prefix over experts of ceil(n_e / tile_rows): expert e owns M tiles
    [tile_offsets[e], tile_offsets[e+1]).  Empty experts own none."""
    n = np.asarray(tokens_per_expert, dtype=np.int64)
    tiles = (n + tile_rows - 1) // tile_rows
    out = np.zeros(n.size + 1, dtype=np.int64)
    out[1:] = np.cumsum(tiles)
    return out


def dispatch(x, token_ids):
    """PFT.x: row r of the buffer is the token row x[token_ids[r]] ([A] §2.1.2 gather)."""
    return _f64(x)[np.asarray(token_ids)]


# --------------------------------------------------------------------- expert FFN
def silu(u):
    return u / (1.0 + np.exp(-u))


def expert_forward(X, w1e, w3e, w2e):
    """One expert's SwiGLU FFN on its rows X [n, d]: H1 = X W1, H3 = X W3, A = SiLU(H1) H3, O = A W2."""
    H1 = X @ _f64(w1e)
    H3 = X @ _f64(w3e)
    A = silu(H1) * H3
    return H1, H3, A, A @ _f64(w2e)


def expert_ffn(x_pft, offsets, w1, w3, w2):
    """Expert FFN over the expert-sorted buffer: expert e takes rows
    [offsets[e], offsets[e+1]) with no padding ([A] §2.1.2 per-expert GEMM loop)."""
    x_pft = _f64(x_pft)
    E = len(offsets) - 1
    N = x_pft.shape[0]
    h = np.shape(w1)[2]
    d = np.shape(w2)[2]
    H1 = np.zeros((N, h)); H3 = np.zeros((N, h)); A = np.zeros((N, h)); O = np.zeros((N, d))
    for e in range(E):
        r0, r1 = int(offsets[e]), int(offsets[e + 1])
        if r1 > r0:
            H1[r0:r1], H3[r0:r1], A[r0:r1], O[r0:r1] = expert_forward(x_pft[r0:r1], w1[e], w3[e], w2[e])
    return H1, H3, A, O


def combine(o, pos, w):
    """y_t = sum_j w_tj * O[pos(t, j)], j in slot order ([A] §2.1.1 combine_weights; [B] 训练流程 step d)."""
    o = _f64(o)
    pos = np.asarray(pos)
    w = _f64(w)
    y = np.zeros((pos.shape[0], o.shape[1]))
    for j in range(pos.shape[1]):
        y += w[:, j:j + 1] * o[pos[:, j]]
    return y


# ----------------------------------------------------------------------- backward
def combine_backward(dy, o, pos, w):
    """Backward of the combine ([B] 训练流程: gradients along the reverse path).

    dO[pos(t, j)] = w_tj * dY_t;  g_tj = <dY_t, O[pos(t, j)]> (gradient w.r.t. w_tj).
    """
    dy = _f64(dy); o = _f64(o); w = _f64(w); pos = np.asarray(pos)
    T, k = pos.shape
    dO = np.zeros_like(o)
    g = np.zeros((T, k))
    for j in range(k):
        dO[pos[:, j]] = w[:, j:j + 1] * dy
        g[:, j] = np.einsum("td,td->t", dy, o[pos[:, j]])
    return dO, g


def expert_backward(X, H1, H3, A, dO, w1e, w3e, w2e):
    """Gradients of one expert's SwiGLU FFN.

    dA = dO W2^T;  dH1 = dA * H3 * s * (1 + H1 (1 - s)) with s = sigmoid(H1);  dH3 = dA * SiLU(H1);
    dW2 = A^T dO;  dW1 = X^T dH1;  dW3 = X^T dH3;  dX = dH1 W1^T + dH3 W3^T.
    """
    w1e = _f64(w1e); w3e = _f64(w3e); w2e = _f64(w2e)
    dA = dO @ w2e.T
    s = 1.0 / (1.0 + np.exp(-H1))
    dH1 = dA * H3 * s * (1.0 + H1 * (1.0 - s))
    dH3 = dA * (H1 * s)
    return {
        "dX": dH1 @ w1e.T + dH3 @ w3e.T,
        "dW1": X.T @ dH1, "dW3": X.T @ dH3, "dW2": A.T @ dO,
        "dH1": dH1, "dH3": dH3,
    }


def expert_ffn_backward(x_pft, H1, H3, A, dO, offsets, w1, w3, w2):
    """Expert backward over the expert-sorted buffer; empty experts get zero weight gradients."""
    x_pft = _f64(x_pft)
    E = len(offsets) - 1
    d, h = np.shape(w1)[1], np.shape(w1)[2]
    dX = np.zeros_like(x_pft)
    dW1 = np.zeros((E, d, h)); dW3 = np.zeros((E, d, h)); dW2 = np.zeros((E, h, d))
    for e in range(E):
        r0, r1 = int(offsets[e]), int(offsets[e + 1])
        if r1 > r0:
            g = expert_backward(x_pft[r0:r1], H1[r0:r1], H3[r0:r1], A[r0:r1], dO[r0:r1], w1[e], w3[e], w2[e])
            dX[r0:r1] = g["dX"]; dW1[e] = g["dW1"]; dW3[e] = g["dW3"]; dW2[e] = g["dW2"]
    return dX, dW1, dW3, dW2


def token_grad(dx_pft, pos):
    """dx_t = sum_j dX_pft[pos(t, j)], j in slot order (the transpose of the dispatch gather)."""
    dx_pft = _f64(dx_pft)
    pos = np.asarray(pos)
    out = np.zeros((pos.shape[0], dx_pft.shape[1]))
    for j in range(pos.shape[1]):
        out += dx_pft[pos[:, j]]
    return out


def gate_backward(x, wg, ids, w, g, E):
    """Backward through the renormalised top-k softmax and the linear gate.

    Only the selected logits receive gradient (the selection is piecewise
    constant).  With w = softmax over the selected logits and g_j = dL/dw_j:
    dz_{t, ids[t,j]} = w_j * (g_j - sum_l w_l g_l).  Then dWg = x^T dz and the
    gate's contribution to dx is dz Wg^T.
    """
    x = _f64(x); wg = _f64(wg); w = _f64(w); g = _f64(g)
    T, k = np.shape(ids)
    dz = np.zeros((T, E))
    inner = (w * g).sum(axis=1, keepdims=True)
    np.put_along_axis(dz, np.asarray(ids, dtype=np.int64), w * (g - inner), axis=1)
    return dz, x.T @ dz, dz @ wg.T


# --------------------------------------------------------------------- full layer
def layer_forward(x, wg, bias, w1, w3, w2, k, logits=None):
    """Forward of the whole layer: gate -> route -> PFT -> dispatch -> experts -> combine.

    ``logits`` (optional): route from these logits instead of the oracle's own
    (used to compare indices bit-exactly against a given logits buffer).
    """
    E = np.shape(wg)[1]
    z = gate_logits(x, wg, bias) if logits is None else _f64(logits)
    ids, w = route(z, k)
    pft = pft_build(ids, w, E)
    x_pft = dispatch(x, pft["token_ids"])
    H1, H3, A, O = expert_ffn(x_pft, pft["expert_offsets"], w1, w3, w2)
    y = combine(O, pft["pos"], w)
    return {"logits": z, "ids": ids, "w": w, "pft": pft, "x_pft": x_pft,
            "H1": H1, "H3": H3, "A": A, "O": O, "y": y}


def layer_backward(fwd, dy, x, wg, w1, w3, w2):
    """Backward of the whole layer given the forward record and dY."""
    E = np.shape(wg)[1]
    pft = fwd["pft"]
    dO, g = combine_backward(dy, fwd["O"], pft["pos"], fwd["w"])
    dX_pft, dW1, dW3, dW2 = expert_ffn_backward(fwd["x_pft"], fwd["H1"], fwd["H3"], fwd["A"], dO,
                                                 pft["expert_offsets"], w1, w3, w2)
    dx = token_grad(dX_pft, pft["pos"])
    dz, dWg, dx_gate = gate_backward(x, wg, fwd["ids"], fwd["w"], g, E)
    return {"dO": dO, "g": g, "dX_pft": dX_pft, "dW1": dW1, "dW3": dW3, "dW2": dW2,
            "dx": dx + dx_gate, "dlogits": dz, "dWg": dWg}


# ---------------------------------------------------------------------------- RBD
def rbd_plan(ids, E, experts_per_device, devices_per_node):
    """Redundancy-bypassing dispatch plan ([A] §2.2.1), indexing only.

    node(e) = e // (experts_per_device * devices_per_node).  Each token sends one
    pilot per distinct node among its k experts; pilots are ordered by node,
    then token.  Pilot p's replicas are the token's experts on that node in
    ascending id (CSR ``replica_offsets`` / ``replica_expert``); the pilot lands
    on the device (e // experts_per_device) of its lowest-id replica.
    ``assign_pilot[t, j]`` is the pilot that carries assignment (t, j).
    """
    ids = np.asarray(ids, dtype=np.int64)
    T, k = ids.shape
    epn = experts_per_device * devices_per_node
    if epn <= 0 or E % epn != 0:
        raise ValueError("E must be a multiple of experts_per_device * devices_per_node")
    n_nodes = E // epn
    tok = np.repeat(np.arange(T, dtype=np.int64), k)
    e = ids.reshape(-1)
    node = e // epn
    keys, inv = np.unique(node * T + tok, return_inverse=True)   # sorted by (node, token)
    inv = inv.reshape(-1)
    P = keys.size
    pilot_node = keys // T
    pilot_token = keys % T
    pilots_per_node = np.bincount(pilot_node, minlength=n_nodes)
    node_offsets = np.zeros(n_nodes + 1, dtype=np.int64)
    node_offsets[1:] = np.cumsum(pilots_per_node)
    grouped = np.lexsort((e, inv))                                # by pilot, then expert id
    replica_expert = e[grouped]
    replica_offsets = np.zeros(P + 1, dtype=np.int64)
    replica_offsets[1:] = np.cumsum(np.bincount(inv, minlength=P))
    pilot_device = replica_expert[replica_offsets[:-1]] // experts_per_device
    n_dev_pairs = np.unique((e // experts_per_device) * T + tok).size
    return {
        "n_nodes": n_nodes,
        "pilots_per_node": pilots_per_node, "node_offsets": node_offsets,
        "pilot_token": pilot_token, "pilot_node": pilot_node, "pilot_device": pilot_device,
        "replica_offsets": replica_offsets, "replica_expert": replica_expert,
        "assign_pilot": inv.reshape(T, k),
        "num_pilots": int(P), "num_token_device_pairs": int(n_dev_pairs),
    }
