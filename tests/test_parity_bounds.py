"""The gate bound of the parity harness, checked on the CPU against fp32 evaluations.

``parity.score_error_bound`` bounds how far softmax scores computed in fp32 from the
stored inputs can lie from the oracle's fp64 scores, for any summation order of the
logits.  Here the scores are evaluated in fp32 (numpy) in several orders, with
round-to-nearest and with truncating accumulation, on XL-like rows (D = 1152, E = 8,
bf16 inputs, router bias of variance 0.5), and every score must stay inside the bound;
a planted mistake (three dropped products) must not.
"""
import numpy as np
import pytest

from oracle import moe_oracle as O
from sparse_moe_layer_03_b200 import inputs as I
from tests import parity as PA


def _inputs(T=48, D=1152, E=8, seed=5):
    # the expert widths do not enter the router: a narrow H keeps the draw small (x, Wg come first)
    w = I.small_workload(T, D, 64, E, 2, 0, "bf16", "topk", seed=seed, router_bias="normal")
    inp = I.make_inputs(w)
    return inp


def _trunc32(v64):
    """fp64 -> fp32 rounded toward zero (a truncating accumulator)."""
    f = v64.astype(np.float32)
    over = np.abs(f.astype(np.float64)) > np.abs(v64)
    f[over] = np.nextafter(f[over], np.float32(0))
    return f


def _logits32(inp, order, truncate=False, drop=None):
    """[T,E] logits summed in fp32 in the given order of the D products (exact in fp32 for bf16)."""
    x = np.asarray(inp["x"], np.float32)
    wg = np.asarray(inp["wg"], np.float32)
    T, D = x.shape
    prods = (x[:, None, :].astype(np.float64) * wg[None, :, :].astype(np.float64)).astype(np.float32)
    if drop is not None:
        prods[:, :, drop] = 0.0
    add = (lambda a, b: _trunc32(a.astype(np.float64) + b.astype(np.float64))) if truncate else \
        (lambda a, b: (a + b).astype(np.float32))
    if order == "chains4":
        # four chains, chain g summing the 16-column slices g, g+4, ... ; each slice summed first
        chains = [np.zeros(prods.shape[:2], np.float32) for _ in range(4)]
        for s in range(D // 16):
            part = np.zeros(prods.shape[:2], np.float32)
            for d in range(16):
                part = add(part, prods[:, :, s * 16 + d])
            chains[s % 4] = add(chains[s % 4], part)
        acc = add(add(chains[0], chains[1]), add(chains[2], chains[3]))
    else:
        idx = range(D) if order == "forward" else range(D - 1, -1, -1)
        acc = np.zeros(prods.shape[:2], np.float32)
        for d in idx:
            acc = add(acc, prods[:, :, d])
    b = inp.get("router_bias")
    if b is not None:
        acc = add(acc, np.broadcast_to(np.asarray(b, np.float32), acc.shape))
    return acc


def _softmax32(l):
    l = l.astype(np.float32)
    e = np.exp((l - l.max(axis=1, keepdims=True)).astype(np.float32)).astype(np.float32)
    z = np.zeros(l.shape[0], np.float32)
    for i in range(l.shape[1]):
        z = (z + e[:, i]).astype(np.float32)
    inv = (np.float32(1.0) / z).astype(np.float32)
    return (e * inv[:, None]).astype(np.float32)


@pytest.mark.parametrize("order,truncate", [("forward", False), ("reverse", False), ("chains4", False),
                                            ("forward", True), ("chains4", True)])
def test_fp32_scores_stay_inside_the_bound(order, truncate):
    inp = _inputs()
    P = O.softmax_scores(O.gate_logits(inp["x"], inp["wg"], inp.get("router_bias")))
    bound = PA.score_error_bound(inp)
    P32 = _softmax32(_logits32(inp, order, truncate)).astype(np.float64)
    err = np.abs(P32 - P)
    assert np.all(err <= bound), (err.max(), bound[err > bound])
    # the bound is not vacuous: it stays well below the scores themselves
    assert np.all(bound <= 0.02 * P)


def test_a_dropped_product_leaves_the_bound():
    inp = _inputs()
    P = O.softmax_scores(O.gate_logits(inp["x"], inp["wg"], inp.get("router_bias")))
    bound = PA.score_error_bound(inp)
    bad = _softmax32(_logits32(inp, "forward", drop=[7, 500, 901])).astype(np.float64)
    assert np.any(np.abs(bad - P) > bound)


def test_bound_on_an_fp32_workload_row():
    # fp32 inputs: products are rounded too (covered by n = D + 2)
    w = I.small_workload(32, 384, 64, 8, 2, 0, "f32", "topk", seed=9)
    inp = I.make_inputs(w)
    P = O.softmax_scores(O.gate_logits(inp["x"], inp["wg"], inp.get("router_bias")))
    x = np.asarray(inp["x"], np.float32)
    wg = np.asarray(inp["wg"], np.float32)
    acc = np.zeros((32, 8), np.float32)
    for d in range(384):
        acc = (acc + (x[:, d:d + 1] * wg[None, :, d]).astype(np.float32)).astype(np.float32)
    err = np.abs(_softmax32(acc).astype(np.float64) - P)
    assert np.all(err <= PA.score_error_bound(inp))
