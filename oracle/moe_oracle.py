"""fp64 CPU oracle for the DiT-MoE sparse expert layer: the forward, the
adaLN pieces around it, per-image statistics, and the backward.

TEST INFRASTRUCTURE.  This module is the checker, not the product: only the
test suite, the smoke check and the benchmark's CPU-baseline leg may import
it.  It shares no code with the CUDA path and imports nothing from it.

Every function restates one step of the method as the pages define it, in
plain numpy on float64, with a library primitive (matmul, exp, tanh, a
stable sort) as a step where one fits and no blocking, fusion or reordering
beyond the definition.  Sources, by page title and section:

* "Scaling Diffusion Transformers to 16 Billion Parameters" (reading note)
  - "MOE 回顾", eq. MoE(x): MoE(x) = sum_i g(x)_i e_i(x); g sparse with k of
    E weights non-zero, so unused experts are not computed.
  - "MOE-DIT", eq. MLP: MLP(x) = W2 gelu(W1 x); every expert is such an MLP.
  - "MOE-DIT", shared-expert routing: n_s extra experts that every token is
    assigned to, whatever the router says.
  - "MOE-DIT", expert-level balance loss, eq. L_balance.
* "DiT-MoE" hub page, section 1 "MoE Gate 路由机制": MoEGate with
  weight (n_routed_experts, gating_dim), softmax scoring, top_k =
  num_experts_per_tok, aux_loss_alpha.
* "Scalable Diffusion Models with Transformers (DiT)", "DiT block 实现细节":
  the core transformer uses the tanh approximation of GELU; adaLN-Zero
  scales each residual branch by a per-sample gate alpha.
* "Diffusion Transformer (DiT) 技术全景解析" 2.2.3 (AdaLN): a plain
  layer_norm over the features, then a per-sample scale and shift.
* "Scaling Diffusion Transformers to 16 Billion Parameters", expert
  specialisation analysis: expert-selection frequency by class, spatial
  position and denoising step.
* "Expert Race: A Flexible Routing Strategy for Scaling Diffusion
  Transformer with Mixture of Experts", abstract: tokens and experts compete
  together and the top candidates are selected.

Readings where the pages are silent (each is listed in the design notes):
g is the softmax score of a selected expert, not renormalised; shared
experts are summed with weight 1; top-K order is descending score, ties to
the lower expert id; Expert-Race takes the S = K*T largest of the T x E
softmax scores, ties to the lower flat index t*E+i; the balance loss's T is
every token of the call and its n is E; expert biases (nn.Linear) are applied
inside e_i, before gating.  For the backward: the selection and the counts
are discrete and carry no gradient; the gates g = P of the selected experts
and the balance loss's p_i carry it back through the softmax.

Parity status: every function here is pinned by a CPU test (closed forms,
brute force, library special cases, invariants, a hand-worked example; the
backward functions against float64 torch autograd through the layer written
with torch library ops, the selection held fixed).  The
full-layer numeric output has no worked example on the pages, so beyond those
pins it is "parity unpinned" against the pages themselves.
"""
from __future__ import annotations

import math
from typing import Optional

import numpy as np

F64 = np.float64


def as_f64(a):
    return None if a is None else np.asarray(a, dtype=F64)


# ---------------------------------------------------------------- router

def gate_logits(x, wg, router_bias=None):
    """l[t,i] = x_t . Wg[i] (+ b_i).

    MoEGate keeps a weight of shape (n_routed_experts, gating_dim) and scores
    hidden states against it ("DiT-MoE" hub page, section 1).  The router bias
    is a synthetic load-skew device of the workloads, not on the pages.
    """
    l = as_f64(x) @ as_f64(wg).T
    if router_bias is not None:
        l = l + as_f64(router_bias)[None, :]
    return l


def softmax_scores(logits):
    """P[t,i] = exp(l_i - m) / sum_j exp(l_j - m), m = max_j l_j.

    MoEGate's scoring_func is 'softmax' (hub page, section 1); P(t,i) is the
    probability of expert i for token t in the balance loss ("MOE-DIT").
    """
    l = as_f64(logits)
    m = l.max(axis=1, keepdims=True)
    e = np.exp(l - m)
    return e / e.sum(axis=1, keepdims=True)


def topk_route(P, K):
    """Per token, the K largest scores, in descending score, ties to the lower id.

    Returns (idx [T,K] int64, g [T,K] fp64) with g the selected scores themselves
    (g sparse with K non-zeros, "MOE 回顾"; MoEGate picks top_k experts).
    """
    P = as_f64(P)
    T, E = P.shape
    idx = np.empty((T, K), dtype=np.int64)
    for t in range(T):
        # stable sort on -P keeps equal scores in ascending expert order
        order = np.argsort(-P[t], kind="stable")
        idx[t] = order[:K]
    g = np.take_along_axis(P, idx, axis=1)
    return idx, g


def race_route(P, S):
    """Expert-Race: the S largest entries of the flattened T x E score matrix.

    Tokens and experts compete together and the top candidates win (Expert
    Race abstract).  Ties go to the lower flat index t*E+i.  Each token keeps
    its winners in descending score, ties to the lower expert id.
    Returns (idx [T,E] int64 padded with -1, g [T,E] fp64 padded with 0,
    n_sel [T] int64).
    """
    P = as_f64(P)
    T, E = P.shape
    flat = P.reshape(-1)
    order = np.argsort(-flat, kind="stable")       # ties: ascending flat index
    chosen = np.zeros(T * E, dtype=bool)
    chosen[order[:S]] = True
    chosen = chosen.reshape(T, E)
    idx = np.full((T, E), -1, dtype=np.int64)
    g = np.zeros((T, E), dtype=F64)
    n_sel = chosen.sum(axis=1).astype(np.int64)
    for t in range(T):
        ids = np.nonzero(chosen[t])[0]
        if ids.size:
            o = ids[np.argsort(-P[t, ids], kind="stable")]
            idx[t, :o.size] = o
            g[t, :o.size] = P[t, o]
    return idx, g, n_sel


def expert_counts(idx, E):
    """counts[i] = sum_t I(t,i): how many (token, expert) pairs chose expert i."""
    idx = np.asarray(idx).reshape(-1)
    idx = idx[idx >= 0]
    return np.bincount(idx, minlength=E).astype(np.int64)


def balance_loss(counts, P, K, alpha):
    """L = alpha * sum_i (n/(K T) sum_t I(t,i)) * (1/T sum_t P(t,i)), n = E.

    "MOE-DIT", expert-level balance loss; T is the number of tokens of the
    call, K the experts per token, n the number of routed experts.
    """
    P = as_f64(P)
    T, E = P.shape
    f = (E / (K * T)) * np.asarray(counts, dtype=F64)
    p = P.sum(axis=0) / T
    return float(alpha * np.sum(f * p))


def balance_stats(idx, P, E):
    """[counts_0..counts_{E-1}, s_0..s_{E-1}] with s_i = sum_t P(t,i): the two per-expert
    token sums eq. L_balance ("MOE-DIT") is made of; both add over disjoint token sets."""
    return np.concatenate([expert_counts(idx, E).astype(F64), as_f64(P).sum(axis=0)])


def balance_loss_from_stats(stats, K, T, alpha):
    """L_balance of T tokens from their statistics: alpha sum_i (n/(K T)) counts_i (s_i / T)."""
    stats = as_f64(stats)
    E = stats.size // 2
    if T == 0:
        return 0.0
    return float(alpha * np.sum((E / (K * T)) * stats[:E] * (stats[E:] / T)))


def balance_loss_per_sequence(idx, P, K, alpha, seq_len):
    """Mean over images of L_balance with T read as one image's patch count.

    "MOE-DIT", eq. L_balance calls T "the length of the image-patch
    sequence".  A call holding B = T_call / seq_len images of seq_len tokens
    each then has one loss per image, counts and score means taken over that
    image's tokens only; this returns their mean.  seq_len = T_call gives
    balance_loss over the whole call.
    """
    P = as_f64(P)
    T, E = P.shape
    if seq_len <= 0 or T % seq_len:
        raise ValueError("seq_len must divide the token count")
    idx = np.asarray(idx).reshape(T, -1)
    per_image = []
    for b in range(T // seq_len):
        rows = slice(b * seq_len, (b + 1) * seq_len)
        per_image.append(balance_loss(expert_counts(idx[rows], E), P[rows], K, alpha))
    return float(np.mean(per_image))


def expert_frequency(idx, E, labels, n_labels):
    """hist[b, i] = number of selected pairs (t, i) whose token carries label b.

    "Scaling Diffusion Transformers to 16 Billion Parameters", expert
    specialisation analysis: expert-selection frequency counted by image
    class, by spatial position and by denoising timestep.  labels[t] is the
    label of token t: its patch position inside the image, or the class or
    timestep of the image it belongs to.
    """
    idx = np.asarray(idx)
    T = idx.shape[0]
    idx = idx.reshape(T, -1)
    labels = np.asarray(labels).reshape(T)
    hist = np.zeros((n_labels, E), dtype=np.int64)
    for t in range(T):
        for i in idx[t]:
            if i >= 0:
                hist[labels[t], i] += 1
    return hist


def position_labels(T, seq_len):
    """Label of token t by its patch position inside its image: t mod seq_len."""
    return np.arange(T) % seq_len


def image_labels(T, seq_len, per_image):
    """Label of token t from the label of the image holding it (class or timestep)."""
    return np.repeat(np.asarray(per_image), seq_len)[:T]


# ---------------------------------------------------------------- balance loss backward

def balance_loss_grad_logits(P, counts, K, alpha):
    """dL_balance / dl[t,i] for the logits l of the router (counts held constant).

    "MOE-DIT", eq. L_balance: L = alpha sum_i f_i p_i with f_i = (n/(K T))
    counts_i from the discrete selection (no gradient) and p_i = (1/T) sum_t
    P[t,i], so dL/dP[t,i] = alpha f_i / T =: c_i for every token.  Through the
    softmax: dl[t,i] = P[t,i] (c_i - sum_j P[t,j] c_j).
    """
    P = as_f64(P)
    T, E = P.shape
    c = alpha * (E / (K * T)) * np.asarray(counts, dtype=F64) / T
    return P * (c[None, :] - (P @ c)[:, None])


def router_backward(x, wg, dlogits):
    """Gradients of l = x Wg^T + b: dWg = dl^T x [E,D], db = sum_t dl [E], dx = dl Wg [T,D]."""
    x, wg, dl = as_f64(x), as_f64(wg), as_f64(dlogits)
    return dl.T @ x, dl.sum(axis=0), dl @ wg


# ---------------------------------------------------------------- layer backward

def gelu_tanh_grad(u):
    """d/du of the tanh GELU: 0.5 (1 + th) + 0.5 u (1 - th^2) c (1 + 3 * 0.044715 u^2),
    th = tanh(c (u + 0.044715 u^3)), c = sqrt(2/pi)."""
    u = as_f64(u)
    c = math.sqrt(2.0 / math.pi)
    th = np.tanh(c * (u + 0.044715 * u ** 3))
    return 0.5 * (1.0 + th) + 0.5 * u * (1.0 - th * th) * c * (1.0 + 3.0 * 0.044715 * u * u)


def _expert_backward(x, w1, b1, w2, b2, dz):
    """Rows x [n,D] through e(x) = W2 gelu(W1 x + b1) + b2, given dz = dJ/de [n,D]:
    returns z = e(x) and the gradients (dx, dW1, db1, dW2, db2)."""
    u = as_f64(x) @ as_f64(w1).T
    if b1 is not None:
        u = u + as_f64(b1)[None, :]
    h = gelu_tanh(u)
    z = h @ as_f64(w2).T
    if b2 is not None:
        z = z + as_f64(b2)[None, :]
    dw2 = dz.T @ h
    db2 = dz.sum(axis=0)
    du = (dz @ as_f64(w2)) * gelu_tanh_grad(u)
    dw1 = du.T @ as_f64(x)
    db1 = du.sum(axis=0)
    dx = du @ as_f64(w1)
    return z, dx, dw1, db1, dw2, db2


def layer_backward(inp, idx, dout, K, alpha, aux_scale=1.0):
    """Gradients of J = <dout, MoE(x)> + aux_scale * L_balance for the tanh-GELU layer.

    The selection idx (-1 padded) and the counts are discrete (no gradient);
    the gates g[t,i] = P[t,i] of the selected experts carry the routing
    gradient: dP[t,i] = <dout_t, e_i(x_t)> on the selection plus the balance
    loss's alpha f_i / T on every entry ("MOE 回顾" eq. MoE(x), "MOE-DIT" eq.
    MLP and eq. L_balance), then back through the softmax and l = x Wg^T + b.
    Returns a dict of dx, dwg, dbias, dw1, db1, dw2, db2, dws1, dbs1, dws2, dbs2.
    """
    x = as_f64(inp["x"])
    dout = as_f64(dout)
    T, D = x.shape
    E = inp["w1"].shape[0]
    P = softmax_scores(gate_logits(x, inp["wg"], inp.get("router_bias")))
    idx = np.asarray(idx).reshape(T, -1)
    grads = {k: np.zeros_like(as_f64(inp[w])) for k, w in
             (("dw1", "w1"), ("dw2", "w2"), ("dws1", "ws1"), ("dws2", "ws2"))}
    H = inp["w1"].shape[1]
    grads["db1"] = np.zeros((E, H))
    grads["db2"] = np.zeros((E, D))
    ns = inp["ws1"].shape[0]
    grads["dbs1"] = np.zeros((ns, H))
    grads["dbs2"] = np.zeros((ns, D))
    dx = np.zeros((T, D))
    dP = np.zeros((T, E))
    for e in range(E):
        rows, slots = np.nonzero(idx == e)
        if rows.size == 0:
            continue
        g = P[rows, e][:, None]
        z, dxe, dw1, db1, dw2, db2 = _expert_backward(x[rows], inp["w1"][e], _bias_row(inp.get("b1"), e),
                                                      inp["w2"][e], _bias_row(inp.get("b2"), e), g * dout[rows])
        np.add.at(dx, rows, dxe)
        grads["dw1"][e] += dw1
        grads["db1"][e] += db1
        grads["dw2"][e] += dw2
        grads["db2"][e] += db2
        dP[rows, e] += np.sum(dout[rows] * z, axis=1)
    for j in range(ns):
        _, dxj, dw1, db1, dw2, db2 = _expert_backward(x, inp["ws1"][j], _bias_row(inp.get("bs1"), j),
                                                      inp["ws2"][j], _bias_row(inp.get("bs2"), j), dout)
        dx += dxj
        grads["dws1"][j] += dw1
        grads["dbs1"][j] += db1
        grads["dws2"][j] += dw2
        grads["dbs2"][j] += db2
    counts = expert_counts(idx, E)
    dP += aux_scale * alpha * (E / (K * T)) * counts[None, :].astype(F64) / T
    dl = P * (dP - np.sum(P * dP, axis=1, keepdims=True))
    dwg, dbias, dxr = router_backward(x, inp["wg"], dl)
    grads.update(dx=dx + dxr, dwg=dwg, dbias=dbias)
    return grads


# ---------------------------------------------------------------- adaLN-Zero around the layer

def layer_norm(x, eps=1e-5):
    """(x - mean) / sqrt(var + eps) over the last dimension, biased variance, no affine.

    "Diffusion Transformer (DiT) 技术全景解析" 2.2.3 (AdaLN): the adaptive norm
    normalises with a plain layer_norm over the feature dimension (library
    default epsilon) before the conditional scale and shift.
    """
    x = as_f64(x)
    mu = x.mean(axis=-1, keepdims=True)
    var = ((x - mu) ** 2).mean(axis=-1, keepdims=True)
    return (x - mu) / np.sqrt(var + eps)


def adaln(x, gamma, beta, img_len, eps=1e-5):
    """gamma_b * LayerNorm(x_t) + beta_b for token t of image b = t // img_len.

    "Diffusion Transformer (DiT) 技术全景解析" 2.2.3: gamma and beta are
    regressed from the conditioning per sample and broadcast over its tokens.
    """
    x = as_f64(x)
    T = x.shape[0]
    b = np.arange(T) // img_len
    return as_f64(gamma)[b] * layer_norm(x, eps) + as_f64(beta)[b]


def gated_residual(x_res, y, alpha, img_len):
    """x_res_t + alpha_b * y_t: the adaLN-Zero gate on a residual branch.

    "Scalable Diffusion Models with Transformers (DiT)", DiT block details
    (adaLN-Zero): a per-dimension scale alpha, regressed per sample, multiplies
    the branch before each residual connection; zero alpha makes the block the
    identity.
    """
    x_res = as_f64(x_res)
    b = np.arange(x_res.shape[0]) // img_len
    return x_res + as_f64(alpha)[b] * as_f64(y)


# ---------------------------------------------------------------- experts

def gelu_tanh(u):
    """0.5 u (1 + tanh(sqrt(2/pi) (u + 0.044715 u^3))): the tanh GELU of the DiT core."""
    u = as_f64(u)
    return 0.5 * u * (1.0 + np.tanh(math.sqrt(2.0 / math.pi) * (u + 0.044715 * u ** 3)))


def gelu_erf(u):
    """0.5 u (1 + erf(u / sqrt 2)): exact GELU (nn.GELU default), kept only as an option."""
    u = as_f64(u)
    erf = np.vectorize(math.erf, otypes=[F64])
    return 0.5 * u * (1.0 + erf(u / math.sqrt(2.0)))


def expert_mlp(x, w1, b1, w2, b2, act="tanh"):
    """e(x) = W2 gelu(W1 x + b1) + b2 for a batch of rows x [n,D].

    "MOE-DIT", eq. MLP: two linear layers with a GELU between; each expert is
    such an MLP.  Weights are nn.Linear style: w1 [H,D], w2 [D,H].
    """
    sigma = gelu_tanh if act == "tanh" else gelu_erf
    u = as_f64(x) @ as_f64(w1).T
    if b1 is not None:
        u = u + as_f64(b1)[None, :]
    y = sigma(u) @ as_f64(w2).T
    if b2 is not None:
        y = y + as_f64(b2)[None, :]
    return y


# ---------------------------------------------------------------- layer

def route(inp, K, routing="topk", alpha=0.01):
    """Router half of the layer: logits, scores, selection, counts, balance loss."""
    P = softmax_scores(gate_logits(inp["x"], inp["wg"], inp.get("router_bias")))
    T, E = P.shape
    if routing == "race":
        idx, g, n_sel = race_route(P, K * T)
    else:
        idx, g = topk_route(P, K)
        n_sel = np.full(T, K, dtype=np.int64)
    counts = expert_counts(idx, E)
    return {"P": P, "idx": idx, "g": g, "n_sel": n_sel, "counts": counts,
            "aux": balance_loss(counts, P, K, alpha)}


def _bias_row(b, j):
    return None if b is None else b[j]


def layer_output(inp, idx, g, n_sel=None, tokens=None, act="tanh"):
    """MoE(x_t) = sum_{i in sel_t} g_{t,i} e_i(x_t) + sum_j s_j(x_t).

    "MOE 回顾", eq. MoE(x), with the sparse g (only selected experts are
    evaluated), plus the shared experts of "MOE-DIT" with weight 1.
    ``idx``/``g`` hold each token's selection (-1 padded); ``tokens`` restricts
    the evaluation to a subset of rows (the others are not computed).
    """
    x = as_f64(inp["x"])
    T = x.shape[0]
    tok = np.arange(T) if tokens is None else np.asarray(tokens)
    idx = np.asarray(idx)[tok]
    g = as_f64(g)[tok]
    xs = x[tok]
    out = np.zeros((tok.size, x.shape[1]), dtype=F64)
    E = inp["w1"].shape[0]
    for e in range(E):
        rows, slots = np.nonzero(idx == e)
        if rows.size == 0:
            continue
        y = expert_mlp(xs[rows], inp["w1"][e], _bias_row(inp.get("b1"), e),
                       inp["w2"][e], _bias_row(inp.get("b2"), e), act)
        np.add.at(out, rows, g[rows, slots][:, None] * y)
    for j in range(inp["ws1"].shape[0]):
        out += expert_mlp(xs, inp["ws1"][j], _bias_row(inp.get("bs1"), j),
                          inp["ws2"][j], _bias_row(inp.get("bs2"), j), act)
    return out


def layer(inp, K, routing="topk", alpha=0.01, act="tanh"):
    """Whole layer: route, evaluate the selected and the shared experts, combine."""
    r = route(inp, K, routing, alpha)
    r["out"] = layer_output(inp, r["idx"], r["g"], r["n_sel"], act=act)
    return r


def dense_masked_output(inp, g_dense, act="tanh"):
    """MoE(x) = sum_{i=1..E} g(x)_i e_i(x) evaluated densely over all E experts.

    The un-sparsified form of "MOE 回顾": every expert runs on every token and
    is multiplied by a gate vector that is zero off the selection.
    """
    x = as_f64(inp["x"])
    out = np.zeros_like(x)
    for e in range(inp["w1"].shape[0]):
        y = expert_mlp(x, inp["w1"][e], _bias_row(inp.get("b1"), e),
                       inp["w2"][e], _bias_row(inp.get("b2"), e), act)
        out += as_f64(g_dense)[:, e:e + 1] * y
    for j in range(inp["ws1"].shape[0]):
        out += expert_mlp(x, inp["ws1"][j], _bias_row(inp.get("bs1"), j),
                          inp["ws2"][j], _bias_row(inp.get("bs2"), j), act)
    return out


def dense_gate(idx, g, T, E):
    """Scatter a (-1 padded) selection into a dense [T,E] gate matrix."""
    gd = np.zeros((T, E), dtype=F64)
    idx = np.asarray(idx)
    for t in range(T):
        for k in range(idx.shape[1]):
            if idx[t, k] >= 0:
                gd[t, idx[t, k]] = g[t, k]
    return gd


# ---------------------------------------------------------------- permutation

def canonical_permutation(idx, E, tile=128):
    """Expert-contiguous order of the selected (token, expert) pairs.

    Computing only the selected experts ("MOE 回顾": unused experts need not
    be computed) means gathering each expert's tokens into one block.  The
    canonical order: expert segments in ascending expert id, tokens ascending
    inside a segment; segment i starts at padded_offsets[i], the sum of the
    earlier segment lengths rounded up to ``tile`` rows.
    Returns counts [E], offsets [E+1] (unpadded), padded_offsets [E+1],
    pos [T,Kmax] (-1 where unselected) and row_token [R] (-1 on pad rows),
    row_slot [R] (which of the token's slots the row serves, -1 on pad).
    """
    idx = np.asarray(idx)
    T, Kmax = idx.shape
    counts = expert_counts(idx, E)
    offsets = np.zeros(E + 1, dtype=np.int64)
    offsets[1:] = np.cumsum(counts)
    padded = np.zeros(E + 1, dtype=np.int64)
    padded[1:] = np.cumsum((counts + tile - 1) // tile * tile)
    R = int(padded[-1])
    pos = np.full((T, Kmax), -1, dtype=np.int64)
    row_token = np.full(R, -1, dtype=np.int64)
    row_slot = np.full(R, -1, dtype=np.int64)
    fill = padded[:-1].copy()
    for t in range(T):                      # ascending tokens inside each segment
        for k in range(Kmax):
            e = idx[t, k]
            if e < 0:
                continue
            r = fill[e]
            fill[e] += 1
            pos[t, k] = r
            row_token[r] = t
            row_slot[r] = k
    return {"counts": counts, "offsets": offsets, "padded_offsets": padded,
            "pos": pos, "row_token": row_token, "row_slot": row_slot}
