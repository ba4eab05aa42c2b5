"""Pins of the fp64 oracle against what the pages and the mathematics fix.

None of these compares the oracle with itself: each check is a closed form, a
hand-worked example from tests/golden (with its citation), a brute force on a
tiny input, a library routine for a special case, or an invariant.  The
mutation tests at the end plant a plausible mistake in the oracle and check
that some pin catches it.
"""
import itertools
import json
import math
import os

import numpy as np
import pytest
import torch

from oracle import moe_oracle as O
from sparse_moe_layer_03_b200 import inputs as I
from sparse_moe_layer_03_b200 import metrics as M

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _rand_scores(T, E, seed):
    rng = np.random.default_rng(seed)
    return O.softmax_scores(rng.standard_normal((T, E)) * 2.0)


# ------------------------------------------------------------------ softmax

def test_softmax_rows_sum_to_one_and_argmax():
    rng = np.random.default_rng(0)
    l = rng.standard_normal((300, 16)) * 5
    P = O.softmax_scores(l)
    assert np.all(P >= 0)
    assert np.max(np.abs(P.sum(1) - 1.0)) < 1e-12
    assert np.array_equal(P.argmax(1), l.argmax(1))


def test_softmax_matches_library_and_shift_invariance():
    rng = np.random.default_rng(1)
    l = rng.standard_normal((64, 8)) * 3
    ref = torch.softmax(torch.from_numpy(l), dim=1).numpy()
    assert np.max(np.abs(O.softmax_scores(l) - ref)) < 1e-14
    assert np.max(np.abs(O.softmax_scores(l + 7.25) - O.softmax_scores(l))) < 1e-14


def test_gate_logits_library():
    rng = np.random.default_rng(2)
    x, wg, b = rng.standard_normal((10, 12)), rng.standard_normal((4, 12)), rng.standard_normal(4)
    ref = torch.nn.functional.linear(torch.from_numpy(x), torch.from_numpy(wg), torch.from_numpy(b))
    assert np.allclose(O.gate_logits(x, wg, b), ref.numpy(), rtol=0, atol=1e-13)


# ------------------------------------------------------------------ top-K

@pytest.mark.parametrize("K", [1, 2, 3, 8])
def test_topk_equals_brute_force(K):
    E = 8
    P = _rand_scores(120, E, 3 + K)
    idx, g = O.topk_route(P, K)
    for t in range(P.shape[0]):
        best = max(itertools.combinations(range(E), K), key=lambda c: sum(P[t, i] for i in c))
        assert set(idx[t]) == set(best)
        assert all(P[t, idx[t, k]] >= P[t, idx[t, k + 1]] for k in range(K - 1))
        assert np.array_equal(g[t], P[t, idx[t]])
    if K == E:
        assert all(sorted(r) == list(range(E)) for r in idx.tolist())


def test_topk_ties_take_lower_id():
    P = np.array([[0.25, 0.25, 0.25, 0.25], [0.1, 0.4, 0.4, 0.1]])
    idx, _ = O.topk_route(P, 2)
    assert idx.tolist() == [[0, 1], [1, 2]]


# ------------------------------------------------------------------ race

def test_race_single_token_equals_topk():
    P = _rand_scores(1, 16, 7)
    idx, g, n = O.race_route(P, 2)
    idk, gk = O.topk_route(P, 2)
    assert n.tolist() == [2] and idx[0, :2].tolist() == idk[0].tolist()


def test_race_all_selected_when_k_equals_e():
    P = _rand_scores(9, 4, 8)
    idx, g, n = O.race_route(P, 9 * 4)
    assert n.tolist() == [4] * 9
    assert all(sorted(r) == [0, 1, 2, 3] for r in idx.tolist())


@pytest.mark.parametrize("T,E,K", [(4, 3, 1), (3, 4, 2), (5, 2, 1)])
def test_race_brute_force_tiny(T, E, K):
    P = _rand_scores(T, E, 10 * T + E)
    S = K * T
    idx, g, n = O.race_route(P, S)
    flat = [(P[t, i], t, i) for t in range(T) for i in range(E)]
    best = max(itertools.combinations(range(T * E), S), key=lambda c: sum(flat[f][0] for f in c))
    want = {(flat[f][1], flat[f][2]) for f in best}
    got = {(t, int(idx[t, k])) for t in range(T) for k in range(n[t])}
    assert got == want and n.sum() == S
    for t in range(T):
        sel = idx[t, :n[t]]
        assert all(P[t, sel[k]] >= P[t, sel[k + 1]] for k in range(len(sel) - 1))
        assert np.all(idx[t, n[t]:] == -1)


# ------------------------------------------------------------------ counts and loss

def test_counts_sum_and_histogram():
    P = _rand_scores(333, 8, 11)
    idx, _ = O.topk_route(P, 2)
    c = O.expert_counts(idx, 8)
    assert c.sum() == 2 * 333
    brute = [0] * 8
    for row in idx.tolist():
        for e in row:
            brute[e] += 1
    assert c.tolist() == brute


def test_balance_loss_uniform_scores_gives_alpha():
    # Wg = 0 and no bias: every P = 1/E, so p_i = 1/E and sum_i f_i = E -> L = alpha
    T, D, E, K = 64, 16, 8, 2
    x = np.random.default_rng(0).standard_normal((T, D))
    r = O.route({"x": x, "wg": np.zeros((E, D))}, K, "topk", 0.05)
    assert abs(r["aux"] - 0.05) < 1e-15
    r = O.route({"x": x, "wg": np.zeros((E, D))}, K, "race", 0.05)
    assert abs(r["aux"] - 0.05) < 1e-15


def test_balance_loss_single_expert_gives_alpha():
    x = np.random.default_rng(1).standard_normal((17, 8))
    r = O.route({"x": x, "wg": np.random.default_rng(2).standard_normal((1, 8))}, 1, "topk", 0.01)
    assert r["counts"].tolist() == [17] and abs(r["aux"] - 0.01) < 1e-16


def test_balance_loss_uniform_counts_gives_alpha():
    # hand-built router: token t points along expert (t mod E) -> counts all T*K/E
    E, T = 4, 40
    x = np.zeros((T, E))
    for t in range(T):
        x[t, t % E] = 3.0 + 0.01 * t
    r = O.route({"x": x, "wg": np.eye(E)}, 1, "topk", 0.01)
    assert r["counts"].tolist() == [T // E] * E
    assert abs(r["aux"] - 0.01) < 1e-15


def test_balance_loss_partial_sums():
    P = _rand_scores(50, 8, 12)
    idx, _ = O.topk_route(P, 2)
    c = O.expert_counts(idx, 8)
    f = 8 / (2 * 50) * c
    assert abs(f.sum() - 8) < 1e-12 and abs(P.sum(0).sum() / 50 - 1) < 1e-12


def _golden_x(a_list):
    a = {"ln3": math.log(3.0), "-ln3": -math.log(3.0), "0": 0.0}
    return np.array([[a[s], 0.0] for s in a_list])


def test_worked_example_balance_and_race():
    g = json.load(open(os.path.join(GOLDEN, "balance_worked_example.json")))
    wg = np.array([[1.0, 0.0], [0.0, 0.0]])
    for case in g["cases"]:
        x = _golden_x(case["a"])
        inp = {"x": x, "wg": wg}
        for mode in ("topk", "race"):
            r = O.route(inp, case["K"], mode, g["alpha"])
            want = case[mode]
            assert np.allclose(r["P"], case["P"], atol=1e-15)
            assert r["idx"].tolist() == want["idx"], (case["name"], mode)
            assert r["counts"].tolist() == want["counts"]
            if mode == "race":
                assert r["n_sel"].tolist() == want["n_sel"]
            assert abs(r["aux"] - want["loss"]) < 1e-15


def test_balance_stats_of_parts_give_the_whole_batch_loss():
    # counts and score sums add over disjoint token sets, so the loss from summed statistics
    # of the parts is the loss of the whole batch: the hand-worked values, then a random case
    g = json.load(open(os.path.join(GOLDEN, "balance_worked_example.json")))
    wg = np.array([[1.0, 0.0], [0.0, 0.0]])
    for case in g["cases"]:
        r = O.route({"x": _golden_x(case["a"]), "wg": wg}, case["K"], "topk", g["alpha"])
        parts = [slice(0, 2), slice(2, 4)]
        st = sum(O.balance_stats(r["idx"][p], r["P"][p], 2) for p in parts)
        assert abs(O.balance_loss_from_stats(st, case["K"], 4, g["alpha"]) - case["topk"]["loss"]) < 1e-15
    rng = np.random.default_rng(61)
    T, E, K, alpha = 97, 8, 2, 0.01
    P = O.softmax_scores(rng.standard_normal((T, E)) * 1.5 + np.linspace(-1, 1, E))
    idx, _ = O.topk_route(P, K)
    whole = O.balance_loss(O.expert_counts(idx, E), P, K, alpha)
    cuts = [0, 13, 60, 97]
    st = sum(O.balance_stats(idx[a:b], P[a:b], E) for a, b in zip(cuts[:-1], cuts[1:]))
    assert abs(O.balance_loss_from_stats(st, K, T, alpha) - whole) <= 1e-15 * abs(whole) * 10
    assert np.array_equal(st[:E], O.expert_counts(idx, E))
    assert O.balance_loss_from_stats(np.zeros(2 * E), K, 0, alpha) == 0.0


def test_balance_stats_uniform_scores_give_alpha_for_any_split():
    # uniform P: every p_i = 1/E and sum_i f_i = E, so L = alpha whatever the selection or split
    T, E, K, alpha = 30, 4, 2, 0.05
    P = np.full((T, E), 1.0 / E)
    idx, _ = O.topk_route(P, K)
    st = O.balance_stats(idx[:7], P[:7], E) + O.balance_stats(idx[7:], P[7:], E)
    assert abs(O.balance_loss_from_stats(st, K, T, alpha) - alpha) < 1e-15


def test_planted_mean_of_rank_losses_is_caught():
    # averaging the parts' own losses is not the whole-batch loss: worked case A split in two
    # halves gives 1.5 alpha and 1.0 alpha (mean 1.25 alpha) against 1.125 alpha for the batch
    g = json.load(open(os.path.join(GOLDEN, "balance_worked_example.json")))
    case = g["cases"][0]
    r = O.route({"x": _golden_x(case["a"]), "wg": np.array([[1.0, 0.0], [0.0, 0.0]])}, 1, "topk", g["alpha"])
    halves = [O.balance_loss(O.expert_counts(r["idx"][p], 2), r["P"][p], 1, g["alpha"])
              for p in (slice(0, 2), slice(2, 4))]
    assert abs(halves[0] - 1.5 * g["alpha"]) < 1e-15 and abs(halves[1] - g["alpha"]) < 1e-15
    assert abs(np.mean(halves) - case["topk"]["loss"]) > 0.1 * g["alpha"]


def test_worked_example_per_image_loss_and_frequencies():
    g = json.load(open(os.path.join(GOLDEN, "balance_per_image_example.json")))
    inp = {"x": _golden_x(g["a"]), "wg": np.array([[1.0, 0.0], [0.0, 0.0]])}
    L, K, alpha = g["seq_len"], g["K"], g["alpha"]
    for mode in ("topk", "race"):
        r = O.route(inp, K, mode, alpha)
        assert np.allclose(r["P"], g["P"], atol=1e-15)
        idx = r["idx"][:, :1] if mode == "race" else r["idx"]
        assert idx.tolist() == g["idx"], mode
        assert abs(O.balance_loss_per_sequence(r["idx"], r["P"], K, alpha, L) - g["per_image"]["loss"]) < 1e-15
        assert abs(r["aux"] - g["whole_call"]["loss"]) < 1e-15
        T = r["P"].shape[0]
        hp = O.expert_frequency(r["idx"], 2, O.position_labels(T, L), L)
        assert hp.tolist() == g["position_hist"]["hist"]
        ih = g["image_hist"]
        hi = O.expert_frequency(r["idx"], 2, O.image_labels(T, L, ih["image_labels"]), ih["n_labels"])
        want = np.zeros((ih["n_labels"], 2), dtype=np.int64)
        for row, v in ih["rows"].items():
            want[int(row)] = v
        assert np.array_equal(hi, want)


def test_per_image_loss_closed_forms():
    # one image spanning the call is the whole-call loss
    P = _rand_scores(48, 8, 21)
    idx, _ = O.topk_route(P, 2)
    whole = O.balance_loss(O.expert_counts(idx, 8), P, 2, 0.01)
    assert abs(O.balance_loss_per_sequence(idx, P, 2, 0.01, 48) - whole) < 1e-15
    # uniform scores: every image's loss is alpha, whatever the selection
    Pu = np.full((64, 8), 1 / 8)
    idx_u, _ = O.topk_route(Pu, 2)
    assert abs(O.balance_loss_per_sequence(idx_u, Pu, 2, 0.01, 16) - 0.01) < 1e-15
    # every image routes each expert equally often: alpha again, whatever the scores
    E, K, L = 4, 1, 8
    idx_b = np.tile(np.arange(E).repeat(L // E), 3).reshape(-1, 1)
    Pb = _rand_scores(3 * L, E, 22)
    assert abs(O.balance_loss_per_sequence(idx_b, Pb, K, 0.05, L) - 0.05) < 1e-15
    with pytest.raises(ValueError):
        O.balance_loss_per_sequence(idx, P, 2, 0.01, 5)


@pytest.mark.parametrize("routing", ["topk", "race"])
def test_frequency_marginals_and_relabelling(routing):
    P = _rand_scores(96, 8, 23)
    if routing == "race":
        idx, _, _ = O.race_route(P, 2 * 96)
    else:
        idx, _ = O.topk_route(P, 2)
    counts = O.expert_counts(idx, 8)
    hp = O.expert_frequency(idx, 8, O.position_labels(96, 32), 32)
    assert np.array_equal(hp.sum(0), counts)
    img = [5, 0, 2]
    hi = O.expert_frequency(idx, 8, O.image_labels(96, 32, img), 6)
    assert np.array_equal(hi.sum(0), counts)
    assert hi[1].sum() == 0 and hi[3].sum() == 0 and hi[4].sum() == 0
    for b, lab in enumerate(img):   # an image's row is its own selection histogram
        assert np.array_equal(hi[lab], O.expert_counts(idx[b * 32:(b + 1) * 32], 8))
    # renaming the labels permutes the rows
    perm = np.array([3, 1, 0, 2, 5, 4])
    hi2 = O.expert_frequency(idx, 8, perm[O.image_labels(96, 32, img)], 6)
    assert np.array_equal(hi2[perm], hi)


# ------------------------------------------------------------------ balance loss backward

@pytest.mark.parametrize("routing", ["topk", "race"])
def test_balance_loss_gradient_matches_autograd(routing):
    # torch autograd (float64) differentiates the loss written with library ops; the counts come
    # from the discrete selection and carry no gradient
    rng = np.random.default_rng(51)
    T, D, E, K, alpha = 40, 24, 8, 2, 0.01
    x = rng.standard_normal((T, D))
    wg = rng.standard_normal((E, D)) / np.sqrt(D)
    b = rng.standard_normal(E) * 0.3
    inp = {"x": x, "wg": wg, "router_bias": b}
    r = O.route(inp, K, routing, alpha)
    xt = torch.tensor(x, requires_grad=True)
    wt = torch.tensor(wg, requires_grad=True)
    bt = torch.tensor(b, requires_grad=True)
    Pt = torch.softmax(torch.nn.functional.linear(xt, wt, bt), dim=1)
    counts = torch.tensor(r["counts"], dtype=torch.float64)
    loss = alpha * torch.sum((E / (K * T)) * counts * Pt.mean(0))
    loss.backward()
    assert abs(loss.item() - r["aux"]) < 1e-15
    dl = O.balance_loss_grad_logits(r["P"], r["counts"], K, alpha)
    dwg, db, dx = O.router_backward(x, wg, dl)
    assert np.max(np.abs(dwg - wt.grad.numpy())) < 1e-15
    assert np.max(np.abs(db - bt.grad.numpy())) < 1e-15
    assert np.max(np.abs(dx - xt.grad.numpy())) < 1e-15


def test_gelu_tanh_grad_matches_autograd():
    u = torch.linspace(-6, 6, 2001, dtype=torch.float64, requires_grad=True)
    torch.nn.functional.gelu(u, approximate="tanh").sum().backward()
    assert np.max(np.abs(O.gelu_tanh_grad(u.detach().numpy()) - u.grad.numpy())) < 1e-14


@pytest.mark.parametrize("routing", ["topk", "race"])
def test_layer_backward_matches_autograd(routing):
    # the whole layer written with library ops in float64, the selection held fixed
    rng = np.random.default_rng(53)
    T, D, H, E, K, ns, alpha, lam = 24, 16, 32, 4, 2, 2, 0.05, 0.7
    inp = {"x": rng.standard_normal((T, D)), "wg": rng.standard_normal((E, D)) / 4,
           "router_bias": rng.standard_normal(E) * 0.2,
           "w1": rng.standard_normal((E, H, D)) / 4, "b1": rng.standard_normal((E, H)) * 0.1,
           "w2": rng.standard_normal((E, D, H)) / 6, "b2": rng.standard_normal((E, D)) * 0.1,
           "ws1": rng.standard_normal((ns, H, D)) / 4, "bs1": rng.standard_normal((ns, H)) * 0.1,
           "ws2": rng.standard_normal((ns, D, H)) / 6, "bs2": rng.standard_normal((ns, D)) * 0.1}
    r = O.route(inp, K, routing, alpha)
    idx = r["idx"]
    dout = rng.standard_normal((T, D))
    got = O.layer_backward(inp, idx, dout, K, alpha, aux_scale=lam)
    t = {k: torch.tensor(v, requires_grad=True) for k, v in inp.items()}
    F = torch.nn.functional
    P = torch.softmax(F.linear(t["x"], t["wg"], t["router_bias"]), dim=1)
    out = torch.zeros(T, D, dtype=torch.float64)
    for e in range(E):
        rows, slots = np.nonzero(idx == e)
        if rows.size == 0:
            continue
        rr = torch.as_tensor(rows)
        y = F.linear(F.gelu(F.linear(t["x"][rr], t["w1"][e], t["b1"][e]), approximate="tanh"), t["w2"][e], t["b2"][e])
        out = out.index_add(0, rr, P[rr, e][:, None] * y)
    for j in range(ns):
        out = out + F.linear(F.gelu(F.linear(t["x"], t["ws1"][j], t["bs1"][j]), approximate="tanh"), t["ws2"][j],
                             t["bs2"][j])
    counts = torch.tensor(O.expert_counts(idx, E), dtype=torch.float64)
    loss = alpha * torch.sum((E / (K * T)) * counts * P.mean(0))
    J = (torch.tensor(dout) * out).sum() + lam * loss
    J.backward()
    pairs = [("dx", "x"), ("dwg", "wg"), ("dbias", "router_bias"), ("dw1", "w1"), ("db1", "b1"), ("dw2", "w2"),
             ("db2", "b2"), ("dws1", "ws1"), ("dbs1", "bs1"), ("dws2", "ws2"), ("dbs2", "bs2")]
    for g, k in pairs:
        ref = t[k].grad.numpy()
        assert np.max(np.abs(got[g] - ref)) <= 1e-12 * max(1.0, np.max(np.abs(ref))), g


def test_balance_loss_gradient_vanishes_for_uniform_counts():
    # with every expert equally loaded, L = alpha sum_i p_i = alpha whatever the scores: zero gradient
    P = _rand_scores(32, 4, 52)
    dl = O.balance_loss_grad_logits(P, np.full(4, 16), 2, 0.05)
    assert np.max(np.abs(dl)) < 1e-18
    assert np.max(np.abs(dl.sum(1))) < 1e-18   # every row of a softmax gradient sums to zero


# ------------------------------------------------------------------ adaLN-Zero

def test_layer_norm_matches_library_and_moments():
    rng = np.random.default_rng(41)
    x = rng.standard_normal((64, 96)) * 3 + 1.5
    ref = torch.nn.functional.layer_norm(torch.from_numpy(x), (96,)).numpy()
    assert np.max(np.abs(O.layer_norm(x) - ref)) < 1e-12
    y = O.layer_norm(x, eps=0.0)
    assert np.max(np.abs(y.mean(1))) < 1e-12 and np.max(np.abs(y.var(1) - 1)) < 1e-12


def test_adaln_special_cases():
    rng = np.random.default_rng(42)
    x = rng.standard_normal((48, 32))
    ones, zeros = np.ones((3, 32)), np.zeros((3, 32))
    assert np.max(np.abs(O.adaln(x, ones, zeros, 16) - O.layer_norm(x))) < 1e-15
    g, b = rng.standard_normal((3, 32)), rng.standard_normal((3, 32))
    m = O.adaln(x, g, b, 16)
    for i in range(3):   # each image uses its own gamma and beta
        rows = slice(16 * i, 16 * i + 16)
        ref = torch.nn.functional.layer_norm(torch.from_numpy(x[rows]), (32,), weight=torch.from_numpy(g[i]),
                                             bias=torch.from_numpy(b[i])).numpy()
        assert np.max(np.abs(m[rows] - ref)) < 1e-12


def test_gated_residual_identity_at_zero_gate():
    rng = np.random.default_rng(43)
    x, y = rng.standard_normal((40, 24)), rng.standard_normal((40, 24))
    assert np.array_equal(O.gated_residual(x, y, np.zeros((5, 24)), 8), x)          # adaLN-Zero at init
    assert np.max(np.abs(O.gated_residual(np.zeros_like(x), y, np.ones((5, 24)), 8) - y)) == 0
    a = rng.standard_normal((5, 24))
    out = O.gated_residual(x, y, a, 8)
    assert np.max(np.abs(out[17] - (x[17] + a[2] * y[17]))) < 1e-15                 # token 17 is in image 2


# ------------------------------------------------------------------ experts

def test_gelu_tanh_matches_library_and_identity():
    u = np.linspace(-8, 8, 4001)
    ref = torch.nn.functional.gelu(torch.from_numpy(u), approximate="tanh").numpy()
    assert np.max(np.abs(O.gelu_tanh(u) - ref)) < 1e-14
    assert np.max(np.abs(O.gelu_tanh(u) - O.gelu_tanh(-u) - u)) < 1e-13
    assert O.gelu_tanh(np.array([0.0]))[0] == 0.0


def test_gelu_erf_matches_library_and_differs_from_tanh():
    u = np.linspace(-6, 6, 1201)
    ref = torch.nn.functional.gelu(torch.from_numpy(u)).numpy()
    assert np.max(np.abs(O.gelu_erf(u) - ref)) < 1e-14
    assert np.max(np.abs(O.gelu_erf(u) - O.gelu_tanh(u))) > 1e-4


def test_expert_mlp_matches_library():
    rng = np.random.default_rng(5)
    D, H = 24, 96
    x = rng.standard_normal((13, D))
    w1, b1 = rng.standard_normal((H, D)) / 5, rng.standard_normal(H)
    w2, b2 = rng.standard_normal((D, H)) / 10, rng.standard_normal(D)
    tt = lambda a: torch.from_numpy(a)
    ref = torch.nn.functional.linear(
        torch.nn.functional.gelu(torch.nn.functional.linear(tt(x), tt(w1), tt(b1)), approximate="tanh"),
        tt(w2), tt(b2)).numpy()
    assert np.max(np.abs(O.expert_mlp(x, w1, b1, w2, b2) - ref)) < 1e-12


def _small_inputs(T=40, D=32, H=64, E=4, K=2, ns=2, bias=0.3, seed=9, routing="topk"):
    w = I.small_workload(T, D, H, E, K, ns, "f32", routing, seed)
    return w, I.make_inputs(w, bias_std=bias)


def test_single_expert_reduces_to_dense_mlp():
    w, inp = _small_inputs(E=1, K=1, ns=0)
    r = O.layer(inp, 1)
    tt = lambda a: torch.from_numpy(np.asarray(a, dtype=np.float64))
    ref = torch.nn.functional.linear(
        torch.nn.functional.gelu(torch.nn.functional.linear(tt(inp["x"]), tt(inp["w1"][0]), tt(inp["b1"][0])),
                                 approximate="tanh"), tt(inp["w2"][0]), tt(inp["b2"][0])).numpy()
    assert np.all(r["g"] == 1.0)
    assert np.max(np.abs(r["out"] - ref)) < 1e-12


@pytest.mark.parametrize("routing", ["topk", "race"])
def test_sparse_equals_dense_masked(routing):
    w, inp = _small_inputs(T=48, E=8, K=2, routing=routing)
    r = O.layer(inp, 2, routing)
    gd = O.dense_gate(r["idx"], r["g"], 48, 8)
    dense = O.dense_masked_output(inp, gd)
    assert np.max(np.abs(r["out"] - dense)) < 1e-12


@pytest.mark.parametrize("routing", ["topk", "race"])
def test_layer_output_on_a_token_subset_equals_those_rows(routing):
    # the sampled full-size parity checks evaluate the oracle on a subset of tokens: the subset's
    # rows must be the full evaluation's rows, in the order asked, repeats included
    w, inp = _small_inputs(T=48, E=8, K=2, routing=routing)
    r = O.layer(inp, 2, routing)
    for tok in ([0], [47, 3, 19, 3], list(range(0, 48, 5)), []):
        tok = np.asarray(tok, dtype=np.int64)
        sub = O.layer_output(inp, r["idx"], r["g"], tokens=tok)
        assert sub.shape == (len(tok), inp["x"].shape[1])
        assert np.max(np.abs(sub - r["out"][tok]), initial=0.0) < 1e-13


def test_shared_concat_identity():
    w, inp = _small_inputs(E=2, ns=3)
    x = torch.from_numpy(inp["x"].astype(np.float64))
    w1c = torch.from_numpy(np.concatenate(list(inp["ws1"]), 0).astype(np.float64))
    b1c = torch.from_numpy(np.concatenate(list(inp["bs1"]), 0).astype(np.float64))
    w2c = torch.from_numpy(np.concatenate(list(inp["ws2"]), 1).astype(np.float64))
    b2c = torch.from_numpy(inp["bs2"].astype(np.float64).sum(0))
    cat = torch.nn.functional.linear(
        torch.nn.functional.gelu(torch.nn.functional.linear(x, w1c, b1c), approximate="tanh"), w2c, b2c).numpy()
    zero = dict(inp)
    zero["w2"] = np.zeros_like(inp["w2"])
    zero["b2"] = None
    r = O.layer(zero, 2)
    assert np.max(np.abs(r["out"] - cat)) < 1e-12


def test_token_permutation_and_expert_relabelling():
    w, inp = _small_inputs(T=30, E=6, K=2)
    base = O.layer(inp, 2)["out"]
    perm = np.random.default_rng(0).permutation(30)
    p_inp = dict(inp)
    p_inp["x"] = inp["x"][perm]
    assert np.max(np.abs(O.layer(p_inp, 2)["out"] - base[perm])) < 1e-12
    lab = np.random.default_rng(1).permutation(6)
    r_inp = dict(inp)
    for k in ("wg", "w1", "w2", "b1", "b2"):
        r_inp[k] = inp[k][lab]
    assert np.max(np.abs(O.layer(r_inp, 2)["out"] - base)) < 1e-12


# ------------------------------------------------------------------ permutation

@pytest.mark.parametrize("routing", ["topk", "race"])
def test_canonical_permutation_properties(routing):
    P = _rand_scores(300, 8, 21)
    idx = O.topk_route(P, 2)[0] if routing == "topk" else O.race_route(P, 600)[0]
    cp = O.canonical_permutation(idx, 8)
    po = cp["padded_offsets"]
    assert np.all(po % 128 == 0)
    # independent construction: sort the (expert, token) pairs
    t_of, k_of = np.nonzero(idx >= 0)
    e_of = idx[t_of, k_of]
    order = np.lexsort((t_of, e_of))
    for e in range(8):
        seg = cp["row_token"][po[e]:po[e] + cp["counts"][e]]
        assert np.all(np.diff(seg) > 0)
        assert set(seg.tolist()) == set(np.nonzero((idx == e).any(1))[0].tolist())
        assert np.all(cp["row_token"][po[e] + cp["counts"][e]:po[e + 1]] == -1)
    rows = cp["pos"][t_of[order], k_of[order]]
    assert np.array_equal(cp["row_token"][rows], t_of[order])
    assert np.array_equal(cp["offsets"][1:], np.cumsum(cp["counts"]))


# ------------------------------------------------------------------ accounting and inputs

def test_flop_convention_reproduces_dit_gflops():
    g = json.load(open(os.path.join(GOLDEN, "dit_xl2_gflops.json")))
    D, L, p, C = g["hidden"], g["depth"], g["patch"], g["latent_channels"]
    H = g["mlp_ratio"] * D
    for case in g["cases"]:
        N = case["tokens"]
        per_block = N * M.mlp_macs_per_token(D, H) + N * 4 * D * D + 2 * N * N * D + 6 * D * D
        embed = N * p * p * C * D + g["frequency_embedding"] * D + D * D
        final = N * D * p * p * 2 * C + 2 * D * D
        gmacs = (L * per_block + embed + final) / 1e9
        assert abs(gmacs / case["printed_gflops"] - 1) < 2e-3, gmacs


def test_layer_flops_xl():
    w = I.WORKLOADS["xl2_8e2a_512"]
    f = M.gemm_flops(w.T, w.D, w.H, w.K, w.n_shared)
    assert abs(f / 2.7831e12 - 1) < 1e-4


def test_inputs_seeded_and_bf16_exact():
    w = I.small_workload(20, 16, 32, 4, 2, 1, "bf16", seed=3)
    a, b = I.make_inputs(w), I.make_inputs(w)
    assert np.array_equal(a["w1"], b["w1"])
    t = torch.from_numpy(np.random.default_rng(0).standard_normal(10000).astype(np.float32))
    assert torch.equal(torch.from_numpy(I.round_to_bf16(t.numpy())), t.to(torch.bfloat16).float())
    assert torch.equal(torch.from_numpy(a["x"]).to(torch.bfloat16).float(), torch.from_numpy(a["x"]))


# ------------------------------------------------------------------ planted mistakes

def test_planted_gelu_sign_is_caught(monkeypatch):
    bad = lambda u: 0.5 * u * (1.0 - np.tanh(math.sqrt(2 / math.pi) * (u + 0.044715 * u ** 3)))
    monkeypatch.setattr(O, "gelu_tanh", bad)
    with pytest.raises(AssertionError):
        test_gelu_tanh_matches_library_and_identity()


def test_planted_loss_factor_is_caught(monkeypatch):
    def bad(counts, P, K, alpha):
        T, E = P.shape
        return float(alpha * np.sum((1 / (K * T)) * counts * P.sum(0) / T))
    monkeypatch.setattr(O, "balance_loss", bad)
    with pytest.raises(AssertionError):
        test_balance_loss_uniform_scores_gives_alpha()


def test_planted_dropped_bias_is_caught(monkeypatch):
    def bad(x, w1, b1, w2, b2, act="tanh"):
        u = np.asarray(x, np.float64) @ np.asarray(w1, np.float64).T     # b1 dropped
        y = O.gelu_tanh(u) @ np.asarray(w2, np.float64).T
        return y if b2 is None else y + b2
    monkeypatch.setattr(O, "expert_mlp", bad)
    with pytest.raises(AssertionError):
        test_expert_mlp_matches_library()


def test_planted_race_tie_order_is_caught(monkeypatch):
    def bad(P, S):
        P = np.asarray(P, np.float64)
        T, E = P.shape
        order = np.lexsort((-np.arange(T * E), -P.reshape(-1)))   # ties to the higher flat index
        chosen = np.zeros(T * E, bool)
        chosen[order[:S]] = True
        chosen = chosen.reshape(T, E)
        idx = np.full((T, E), -1, np.int64)
        for t in range(T):
            ids = np.nonzero(chosen[t])[0]
            idx[t, :ids.size] = ids[np.argsort(-P[t, ids], kind="stable")]
        g = np.where(idx >= 0, np.take_along_axis(P, np.maximum(idx, 0), 1), 0.0)
        return idx, g, chosen.sum(1)
    monkeypatch.setattr(O, "race_route", bad)
    with pytest.raises(AssertionError):
        test_worked_example_balance_and_race()


def test_planted_per_image_token_count_is_caught(monkeypatch):
    # a per-image loss that keeps the whole call's T in f and p
    def wrong(idx, P, K, alpha, seq_len):
        P = np.asarray(P, dtype=np.float64)
        T, E = P.shape
        idx = np.asarray(idx).reshape(T, -1)
        out = []
        for b in range(T // seq_len):
            rows = slice(b * seq_len, (b + 1) * seq_len)
            c = O.expert_counts(idx[rows], E)
            out.append(alpha * np.sum((E / (K * T)) * c * P[rows].sum(0) / T))
        return float(np.mean(out))
    monkeypatch.setattr(O, "balance_loss_per_sequence", wrong)
    with pytest.raises(AssertionError):
        test_worked_example_per_image_loss_and_frequencies()


def test_planted_gelu_derivative_is_caught(monkeypatch):
    # a GELU derivative missing the tanh-slope term
    def wrong(u):
        c = math.sqrt(2.0 / math.pi)
        return 0.5 * (1.0 + np.tanh(c * (u + 0.044715 * u ** 3)))
    monkeypatch.setattr(O, "gelu_tanh_grad", wrong)
    with pytest.raises(AssertionError):
        test_layer_backward_matches_autograd("topk")
